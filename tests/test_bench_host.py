"""Host-side logic of bench.py that decides what a reported number means,
checked on CPU: which measured peak a fraction divides by, the step's
roofline time, the DRAM traffic attached to the dominant kernel (and its
invalidation when the kernel source changes), and the clock summary that
accepts or rejects a run."""
import json
import os
import shutil

import pytest

import bench
import synth

PK = dict(hbm=6551.0, bf16=1633.1, bf16_sust=1358.1, burst_mhz=1965.0, sust_mhz=1305.0, src="measured")


def test_peak_choice_follows_the_sampled_clock():
    assert bench.pick_peak(PK, 1965.0) == "burst"
    assert bench.pick_peak(PK, 1900.0) == "burst"
    assert bench.pick_peak(PK, 1417.0) == "sustained"
    assert bench.pick_peak(PK, 1305.0) == "sustained"
    # exactly half way goes to the burst figure; no clock record means sustained
    assert bench.pick_peak(PK, (1965.0 + 1305.0) / 2) == "burst"
    assert bench.pick_peak(PK, None) == "sustained"


def test_step_roofline_is_the_sum_of_the_three_products():
    ls = synth.layer_set("qwen2.5-3b")
    T = 32768
    i8 = 3084.0
    P = ls.params
    want_burst = (2 * T * P / (i8 * 1e12) + 2 * 2 * T * P / (PK["bf16"] * 1e12)) * 1e3
    want_sust = (2 * T * P / (i8 * PK["bf16_sust"] / PK["bf16"] * 1e12)
                 + 2 * 2 * T * P / (PK["bf16_sust"] * 1e12)) * 1e3
    assert bench.step_roofline_ms(ls, T, PK, "burst", i8) == pytest.approx(want_burst, rel=1e-12)
    assert bench.step_roofline_ms(ls, T, PK, "sustained", i8) == pytest.approx(want_sust, rel=1e-12)
    assert want_burst < want_sust
    # the 3B set's dense roofline at these peaks: about 7.8 ms burst, 9.4 ms sustained
    assert 7.5 < want_burst < 8.1 and 9.1 < want_sust < 9.7


def _fake_root(tmp_path):
    root = tmp_path / "root"
    csrc = root / "semi_structured_sparsity_step_b200" / "csrc"
    csrc.mkdir(parents=True)
    for f in ("gemm_tc.cu", "sbl_device.cuh"):
        shutil.copy(os.path.join(bench.ROOT, "semi_structured_sparsity_step_b200", "csrc", f), csrc / f)
    (root / "profiles").mkdir()
    return root


def test_traffic_is_reported_only_for_the_source_it_was_captured_on(tmp_path, monkeypatch):
    root = _fake_root(tmp_path)
    monkeypatch.setattr(bench, "ROOT", str(root))
    assert bench.traffic_for("backward_dw_bf16") is None  # no capture file
    h = bench._kernel_source_hash()
    entry = {"bytes_per_launch": 782914286.0, "launches": 7, "source_hash": h}
    (root / "profiles" / "traffic.json").write_text(json.dumps({"backward_dw_bf16": entry}))
    assert bench.traffic_for("backward_dw_bf16") == 782914286.0
    assert bench.traffic_for("forward_i8") is None  # no entry for that family
    # any change to the kernel source voids the figure
    p = root / "semi_structured_sparsity_step_b200" / "csrc" / "gemm_tc.cu"
    p.write_text(p.read_text() + "\n// edited\n")
    assert bench._kernel_source_hash() != h
    assert bench.traffic_for("backward_dw_bf16") is None


def test_clock_summary_decodes_reasons_and_takes_the_median():
    c = bench.ClockSampler(0)
    assert c.summary()["samples"] == 0 and c.summary()["sm_mhz"] is None
    c.sm_max = 1965.0
    c.how = "test"
    c.samples = [(1400.0, 0x4), (1420.0, 0x4), (1965.0, 0x0), (1380.0, 0x4 | 0x40)]
    s = c.summary()
    assert s["sm_mhz"] == pytest.approx(1410.0)
    assert s["sm_min_mhz"] == 1380.0 and s["sm_max_mhz"] == 1965.0 and s["samples"] == 4
    assert s["reasons"] == ["hw_thermal_slowdown", "sw_power_cap"]


def test_smi_lines_parse_into_samples():
    c = bench.ClockSampler(0)

    class _P:
        stdout = ["0, 1410, 1965, 812.5, 0x4, Not Active, Not Active, Not Active, Active\n",
                  "0, 1395, 1965, 990.1, 0x4, Active, Not Active, Not Active, Active\n",
                  "garbage\n"]
    c.proc = _P()
    c._read_smi()
    assert c.samples == [(1410.0, 0x4), (1395.0, 0x4 | 0x8)]
    assert c.sm_max == 1965.0
