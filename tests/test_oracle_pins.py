"""Pins for the CPU oracle: checks against what the pages and the mathematics
fix, never against the oracle itself.

Each test names the passage it follows (page title, section).  A plausible
slip in the oracle (a wrong tie order, a dropped epsilon, a transposed
operand, a wrong scale) fails at least one of them.
"""
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _bf16(values) -> np.ndarray:
    return synth.bits(torch.tensor(values, dtype=torch.float32).to(torch.bfloat16))


def _read_kv(path):
    rows = []
    for line in open(path, encoding="utf-8"):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        key, *vals = line.split()
        rows.append((key, vals))
    return rows


# ---------------------------------------------------------------- mask (a1)
def test_worked_example_mask():
    """Explainer, "N:M 半結構化稀疏性的運作機制": the 2:4 example (reading:
    top-N by magnitude; the page's first printed group is a typo)."""
    kv = dict(_read_kv(os.path.join(GOLDEN, "worked_example_2of4.txt")))
    N, M = int(kv["N"][0]), int(kv["M"][0])
    w = _bf16([float(v) for v in kv["input"]]).reshape(1, -1)
    keep = oracle.nm_mask(w, N, M)
    assert keep.astype(int).ravel().tolist() == [int(v) for v in kv["keep"]]
    kept = np.where(keep, oracle.bf16_to_f32(w), 0.0).ravel()
    want = oracle.bf16_to_f32(_bf16([float(v) for v in kv["kept"]]))
    assert np.array_equal(kept, want)


def _stable_topn(a, N):
    return set(sorted(range(len(a)), key=lambda j: (-a[j], j))[:N])


def test_mask_bruteforce_m4_all_tuples():
    """Summary, "半结构化 N:M 稀疏": every tuple of {0, +-1, +-2} at M = 4,
    every N, against a stable sort (ties -> lowest index)."""
    vals = [0.0, 1.0, -1.0, 2.0, -2.0]
    tuples = np.array(np.meshgrid(*[vals] * 4, indexing="ij")).reshape(4, -1).T
    w = _bf16(tuples)
    mags = np.abs(tuples)
    for N in range(1, 5):
        keep = oracle.nm_mask(w, N, 4)
        for r in range(tuples.shape[0]):
            want = _stable_topn(list(mags[r]), N)
            assert set(np.nonzero(keep[r])[0].tolist()) == want, (tuples[r], N)


def test_mask_bruteforce_m8_magnitude_patterns():
    """All 3^8 magnitude patterns over {0, 1, 2} at M = 8 with random signs
    (including -0.0), every N, against a stable sort."""
    rng = np.random.default_rng(7)
    levels = np.array(np.meshgrid(*[[0.0, 1.0, 2.0]] * 8, indexing="ij")).reshape(8, -1).T
    signs = np.where(rng.random(levels.shape) < 0.5, -1.0, 1.0)
    w = _bf16(levels * signs)          # 0 * -1 gives -0.0
    for N in range(1, 9):
        keep = oracle.nm_mask(w, N, 8)
        # vectorised stable-sort reference: lexsort by (index, -magnitude)
        order = np.lexsort((np.broadcast_to(np.arange(8), levels.shape), -levels), axis=1)
        want = np.zeros_like(keep)
        np.put_along_axis(want, order[:, :N], True, axis=1)
        assert np.array_equal(keep, want), N
        # and a few rows through the plain Python sort
        for r in range(0, levels.shape[0], 997):
            assert set(np.nonzero(keep[r])[0].tolist()) == _stable_topn(list(levels[r]), N)


@pytest.mark.parametrize("N,M", [(8, 8), (6, 8), (4, 8), (2, 8), (2, 4), (1, 4)])
def test_mask_exactly_n_per_group(N, M):
    """Summary, "半结构化 N:M 稀疏": ||M_group||_0 = N exactly; 6:8 keeps 75%."""
    w = synth.trimodal_weight(64, 256, seed=1, tensor_id=3)
    if N < M:
        w = synth.with_boundary_ties(w, N, M, seed=1, frac=0.05)
    keep = oracle.nm_mask(synth.bits(w), N, M)
    assert (keep.reshape(-1, M).sum(axis=1) == N).all()
    assert keep.mean() == N / M


def test_mask_ties_and_all_equal_groups():
    """Tie-straddling groups built by construction keep the lower-index twin;
    all-equal groups keep the first N positions."""
    N, M = 6, 8
    w = synth.with_boundary_ties(synth.normal_weight(8, 64, seed=2), N, M, seed=2, frac=0.5,
                                 all_equal_groups=2)
    a = np.abs(oracle.bf16_to_f32(synth.bits(w))).reshape(-1, M)
    keep = oracle.nm_mask(synth.bits(w), N, M).reshape(-1, M)
    n_checked = 0
    for g in range(a.shape[0]):
        if np.unique(a[g]).size == 1:
            assert keep[g].tolist() == [True] * N + [False] * (M - N)
            n_checked += 1
            continue
        want = _stable_topn(list(a[g]), N)
        assert set(np.nonzero(keep[g])[0].tolist()) == want
    assert n_checked == 2


def test_mask_from_master_not_quantised():
    """Summary, 核心方法 (first difference) / gist 2.2: the mask ranks the
    continuous master weights.  All eight weights here quantise to +1, so a
    mask taken from W_q would keep the first six; the master-weight mask keeps
    the six largest."""
    vals = [0.50, 0.90, 0.55, 0.95, 0.60, 0.85, 0.65, 0.80]
    w = _bf16(vals).reshape(1, 8)
    weff, gamma, keep = oracle.effective_weight(w, 6, 8)
    assert (oracle.ternary(w, gamma) == 1).all()
    assert keep.ravel().tolist() == [False, True, False, True, True, True, True, True]
    assert weff.ravel().tolist() == [0, 1, 0, 1, 1, 1, 1, 1]


# ---------------------------------------------------------------- gamma (a2)
def _gamma_rational(w_bits):
    """Independent route: exact rational sum, then the stated roundings."""
    f = oracle.bf16_to_f32(w_bits).astype(np.float64).ravel()
    s = sum((Fraction(abs(float(v))) for v in f), Fraction(0))
    return np.float32(float(s) / float(f.size))


def test_gamma_constant_tensor():
    """Summary, 前置知识: gamma = ||W||_1 / (d_out d_in); a tensor of +-c
    has gamma = c."""
    for c in [0.02, 0.3, 1.5, 7.0]:
        w = torch.full((16, 32), c).to(torch.bfloat16)
        w[::2] *= -1
        assert oracle.absmean_gamma(synth.bits(w)) == np.float32(float(w[0, 0].abs()))


def test_gamma_worked_example_and_random():
    kv = dict(_read_kv(os.path.join(GOLDEN, "worked_example_2of4.txt")))
    w = _bf16([float(v) for v in kv["input"]]).reshape(1, -1)
    assert oracle.absmean_gamma(w) == _gamma_rational(w)
    assert abs(float(oracle.absmean_gamma(w)) - 0.625) < 2e-3
    for seed in range(3):
        w = synth.bits(synth.normal_weight(17, 40, seed=seed))
        assert oracle.absmean_gamma(w) == _gamma_rational(w)


def test_gamma_sum_is_exact():
    """The sum is exact and rounded once: 1 + 2^-53 + 2^-53 in that order
    loses both small terms under left-to-right fp64 addition."""
    w = _bf16([1.0, 2.0 ** -53, 2.0 ** -53, 0.0]).reshape(1, 4)
    g = oracle.absmean_gamma(w)
    assert g == np.float32((1.0 + 2.0 ** -52) / 4.0)
    assert g == _gamma_rational(w)


# ---------------------------------------------------------------- ternary (a3)
def test_ternary_threshold_form():
    """Explainer, "1.58 位元量化的技術原理": -1 below -gamma/2, 0 within
    +-gamma/2 (inclusive), +1 above; the fp32 rounding of w/den may only
    move values that sit within half an ulp of the 0.5 threshold."""
    w = synth.bits(synth.normal_weight(64, 512, seed=4))
    gamma = oracle.absmean_gamma(w)
    q = oracle.ternary(w, gamma)
    assert set(np.unique(q).tolist()) <= {-1, 0, 1}
    den = Fraction(float(np.float32(gamma + np.float32(1e-5))))
    f = oracle.bf16_to_f32(w).ravel()
    r32 = np.divide(f, np.float32(den), dtype=np.float32)
    for v, qq, rr in zip(f.tolist(), q.ravel().tolist(), r32.tolist()):
        ratio = Fraction(v) / den
        want = -1 if ratio < Fraction(-1, 2) else (1 if ratio > Fraction(1, 2) else 0)
        if want != qq:
            assert abs(rr) == 0.5, (v, qq, want)


def test_ternary_exact_half_rounds_to_zero():
    """|w / den| = 0.5 exactly maps to 0 (round half to even); 1.5 clips to 1."""
    gamma = np.float32(0.5) - np.float32(1e-5)
    assert np.float32(gamma + np.float32(1e-5)) == np.float32(0.5)
    w = _bf16([0.25, -0.25, 0.75, -0.75, 0.2, 1.0, -3.0, 0.0]).reshape(1, 8)
    assert oracle.ternary(w, gamma).ravel().tolist() == [0, 0, 1, -1, 0, 1, -1, 0]


def test_ternary_odd_symmetry_and_worked_example():
    w = synth.normal_weight(32, 64, seed=5)
    g = oracle.absmean_gamma(synth.bits(w))
    assert np.array_equal(oracle.ternary(synth.bits(-w), g), -oracle.ternary(synth.bits(w), g))
    kv = dict(_read_kv(os.path.join(GOLDEN, "worked_example_2of4.txt")))
    wb = _bf16([float(v) for v in kv["input"]]).reshape(1, -1)
    weff, _, _ = oracle.effective_weight(wb, int(kv["N"][0]), int(kv["M"][0]))
    assert weff.ravel().tolist() == [int(v) for v in kv["weff"]]


def _zero_share_analytic(weights, means, sd):
    """P(|w| <= gamma/2) for a Gaussian mixture with gamma = E|w| (closed form)."""
    from scipy.stats import norm

    def e_abs(mu, s):
        return s * math.sqrt(2 / math.pi) * math.exp(-mu * mu / (2 * s * s)) + mu * (1 - 2 * norm.cdf(-mu / s))

    gamma = sum(p * e_abs(m, sd) for p, m in zip(weights, means))
    t = gamma / 2
    return sum(p * (norm.cdf((t - m) / sd) - norm.cdf((-t - m) / sd)) for p, m in zip(weights, means))


def test_zero_share_normal():
    """N(0, s) weights: P(q = 0) = 2 Phi(sqrt(2/pi)/2) - 1 = 0.3101."""
    q = oracle.ternary(synth.bits(synth.normal_weight(1024, 1024, seed=6)),
                       oracle.absmean_gamma(synth.bits(synth.normal_weight(1024, 1024, seed=6))))
    want = _zero_share_analytic([1.0], [0.0], 0.02)
    assert abs(want - 0.3101) < 1e-3
    assert abs((q == 0).mean() - want) < 3e-3


def test_zero_share_trimodal():
    """Summary, 论文图表 Figure 1 reports about 42.2% zeros for a trained
    BitNet; for the synthetic trimodal mixture used here the closed form is
    0.356 (the 42% is the weight of its centre component)."""
    w = synth.bits(synth.trimodal_weight(1024, 2048, seed=0))
    q = oracle.ternary(w, oracle.absmean_gamma(w))
    want = _zero_share_analytic([0.42, 0.29, 0.29], [0.0, 0.026, -0.026], 0.006)
    assert abs(want - 0.356) < 2e-3
    assert abs((q == 0).mean() - want) < 5e-3


# ---------------------------------------------------------------- act quant (a4)
def test_act_quant_pins():
    """Summary, 前置知识 / Algorithm 1 step (3): per-token absmax to int8."""
    x = synth.activations(33, 200, seed=8, outlier_frac=0.01)
    xb = synth.bits(x)
    xq, amax = oracle.act_quant(xb)
    xf = oracle.bf16_to_f32(xb)
    assert np.array_equal(amax, np.abs(xf).max(axis=1))
    assert np.abs(xq.astype(int)).max() <= 127
    arg = np.abs(xf).argmax(axis=1)
    peak = xq[np.arange(33), arg].astype(int)
    assert np.array_equal(np.abs(peak), np.full(33, 127))
    assert np.array_equal(np.sign(peak), np.sign(xf[np.arange(33), arg]).astype(int))
    # dequantisation error bound: |x - xq * amax / 127| <= amax / 254 (+ fp32 slack)
    err = np.abs(xf.astype(np.float64) - xq.astype(np.float64) * amax[:, None].astype(np.float64) / 127)
    assert (err <= amax[:, None] / 254 * (1 + 1e-5)).all()


def test_act_quant_zero_row_and_scale_invariance():
    x = synth.activations(4, 64, seed=9).to(torch.float32)
    x[1] = 0.0
    xq, amax = oracle.act_quant(synth.bits(x.to(torch.bfloat16)))
    assert (xq[1] == 0).all() and amax[1] == np.float32(1e-5)
    for k in (-3, 5):
        xq2, amax2 = oracle.act_quant(synth.bits((x * 2.0 ** k).to(torch.bfloat16)))
        assert np.array_equal(xq2[[0, 2, 3]], xq[[0, 2, 3]])
        assert np.array_equal(amax2[[0, 2, 3]], amax[[0, 2, 3]] * np.float32(2.0 ** k))


def test_act_quant_empty():
    xq, amax = oracle.act_quant(np.zeros((0, 16), np.uint16))
    assert xq.shape == (0, 16) and amax.shape == (0,)


# ---------------------------------------------------------------- forward (a5)
def test_forward_acc_bruteforce():
    rng = np.random.default_rng(10)
    xq = rng.integers(-128, 128, (5, 24)).astype(np.int8)
    w = rng.integers(-1, 2, (7, 24)).astype(np.int8)
    acc = oracle.forward_acc(xq, w)
    for t in range(5):
        for o in range(7):
            assert acc[t, o] == sum(int(xq[t, j]) * int(w[o, j]) for j in range(24))
    # extreme magnitudes stay exact
    xq = np.full((1, 11008), -128, np.int8)
    w = np.full((1, 11008), -1, np.int8)
    assert oracle.forward_acc(xq, w)[0, 0] == 128 * 11008


def test_forward_output_error_bound():
    """Summary, Algorithm 1 step (6): y approximates x . (gamma W_eff)^T up
    to the activation quantisation error, which is at most
    amax/254 * gamma * sum_j |W_eff[o, j]| per output."""
    x = synth.activations(16, 256, seed=11)
    w = synth.normal_weight(48, 256, seed=11)
    r = oracle.forward(synth.bits(x), synth.bits(w), 6, 8)
    xt = x.to(torch.float64)
    wdq = float(r["gamma"]) * torch.from_numpy(r["weff"].astype(np.float64))
    ref = (xt @ wdq.T).numpy()
    bound = (r["amax"][:, None].astype(np.float64) / 254) * float(r["gamma"]) * \
        np.abs(r["weff"]).sum(axis=1)[None, :].astype(np.float64)
    assert (np.abs(r["y"] - ref) <= bound * (1 + 1e-4) + 1e-6).all()
    # and the bound is not vacuous: y tracks the reference closely
    assert np.abs(r["y"] - ref).max() < 0.05 * np.abs(ref).max()


U32 = Fraction(1, 1 << 24)   # unit roundoff of fp32, round to nearest


def _ulp_close(got: float, want: Fraction, n_roundings: int) -> bool:
    """|got - want| <= n rounding errors of fp32 relative to |want|."""
    return abs(Fraction(float(got)) - want) <= n_roundings * U32 * abs(want)


def test_forward_out_is_the_exact_scaled_product():
    """Summary, Algorithm 1 step (6) ("s absorbs the quantisation scales")
    with 前置知识's absmax scale 127/max|x|: y = acc * gamma * amax / 127.
    Checked against exact rationals: the oracle's three fp32 roundings
    (amax/127, gamma*(.), acc*(.)) leave at most 3 ulps.  A slip of the
    level (128 for 127), a dropped or squared gamma, or an inverted amax is
    off by far more than that."""
    rng = np.random.default_rng(21)
    T, d_out = 40, 24
    acc = rng.integers(-(1 << 20), 1 << 20, size=(T, d_out)).astype(np.int32)
    acc[0, :3] = [0, 1, -1]
    amax = np.exp(rng.uniform(np.log(1e-5), np.log(60.0), size=T)).astype(np.float32)
    amax[:4] = [np.float32(1e-5), 3.0, 0.3125, 2.75]     # floor and non-powers of two
    for gamma in [np.float32(0.0234375), np.float32(rng.uniform(1e-3, 0.1)), np.float32(0.0)]:
        y = oracle.forward_out(acc, gamma, amax)
        assert y.dtype == np.float32
        for t in range(T):
            for o in range(d_out):
                want = Fraction(int(acc[t, o])) * Fraction(float(gamma)) * Fraction(float(amax[t])) / 127
                assert _ulp_close(y[t, o], want, 3), (t, o, y[t, o], float(want))


def test_forward_hand_built_layer_exact():
    """The whole forward on inputs whose every intermediate is known by hand
    (summary, Algorithm 1 steps (2)-(6); 前置知识).  W has one magnitude
    c = 3/128 with hand-set signs, so gamma = c exactly, every code is the
    sign, and at 6:8 the first six positions of each group are kept (all
    ties).  The int8 codes are round-half-even of x * 127 / amax in exact
    arithmetic (the inputs avoid .5 boundaries), and the expected y is the
    exact rational sum(xq * W_eff) * c * amax / 127."""
    c = Fraction(3, 128)
    d_in = 16
    signs = np.array([[1, -1, 1, 1, -1, -1, 1, -1, -1, 1, 1, -1, 1, 1, -1, 1],
                      [-1, -1, -1, 1, 1, 1, -1, 1, 1, 1, -1, -1, 1, -1, 1, 1],
                      [1, 1, 1, 1, 1, 1, 1, 1, -1, -1, -1, -1, -1, -1, -1, -1]], np.int64)
    w = _bf16((signs * float(c)).tolist())
    xs = [[3.0, -1.25, 0.5, 2.0, -0.75, 0.0, 1.75, -2.5, 0.25, -3.0, 1.0, 0.125, -1.625, 2.25, -0.375, 0.625],
          [0.3125, -0.1875, 0.0625, 0.25, -0.3125, 0.125, 0.0, -0.09375, 0.140625, 0.03125, -0.21875, 0.28125,
           -0.046875, 0.1875, -0.25, 0.109375],
          [2.75, 1.4375, -0.6875, 2.0, -2.75, 0.5, 1.125, -1.875, 0.875, -0.25, 2.5, -1.0, 0.1875, -2.125, 1.625,
           0.75]]
    x = _bf16(xs)
    r = oracle.forward(x, w, 6, 8)
    assert Fraction(float(r["gamma"])) == c
    keep = np.tile(np.array([1, 1, 1, 1, 1, 1, 0, 0], np.int64), d_in // 8)
    weff = signs * keep[None, :]
    assert np.array_equal(r["weff"], weff)
    for t, row in enumerate(xs):
        amax = max(abs(Fraction(v)) for v in row)
        assert Fraction(float(r["amax"][t])) == amax
        xq = []
        for v in row:
            q = Fraction(v) * 127 / amax
            fl = math.floor(q)
            assert abs((q - fl) - Fraction(1, 2)) > Fraction(1, 1000), "hand input sits on a rounding tie"
            xq.append(fl + 1 if q - fl > Fraction(1, 2) else fl)
        assert r["xq"][t].tolist() == xq
        for o in range(weff.shape[0]):
            acc = sum(int(a) * int(b) for a, b in zip(xq, weff[o]))
            assert int(r["acc"][t, o]) == acc
            want = Fraction(acc) * c * amax / 127
            assert _ulp_close(r["y"][t, o], want, 3), (t, o, float(r["y"][t, o]), float(want))


def test_dense_8of8_is_plain_bitlinear():
    """Summary, 前置知识: with N = M nothing is masked (plain BitNet b1.58)."""
    w = synth.bits(synth.normal_weight(16, 64, seed=12))
    weff, gamma, keep = oracle.effective_weight(w, 8, 8)
    assert keep.all()
    assert np.array_equal(weff, oracle.ternary(w, gamma))


# ---------------------------------------------------------------- backward (a6, a7)
def test_backward_matches_autograd_of_ste_surrogate():
    """Summary, "Straight-Through Estimator (STE)" and Algorithm 1 step (7):
    the backward treats the quantisers and the N:M selector as the identity,
    so dX and dW are torch autograd gradients of the linear map with the
    dequantised weight gamma W_eff (for dX) and of X W^T (for dW)."""
    T, d_in, d_out = 12, 64, 40
    x = synth.activations(T, d_in, seed=13)
    w = synth.normal_weight(d_out, d_in, seed=13)
    dy = synth.grad_output(T, d_out, seed=13)
    weff, gamma, keep = oracle.effective_weight(synth.bits(w), 6, 8)

    xv = x.to(torch.float64).requires_grad_(True)
    wdq = float(gamma) * torch.from_numpy(weff.astype(np.float64))
    (xv @ wdq.T).backward(dy.to(torch.float64))
    dx = oracle.backward_dx(synth.bits(dy), weff, gamma)
    np.testing.assert_allclose(dx, xv.grad.numpy(), rtol=1e-6, atol=1e-6)

    wv = w.to(torch.float64).requires_grad_(True)
    (x.to(torch.float64) @ wv.T).backward(dy.to(torch.float64))
    dw = oracle.backward_dw(synth.bits(dy), synth.bits(x))
    np.testing.assert_allclose(dw, wv.grad.numpy(), rtol=1e-6, atol=1e-6)
    # Dual STE: masked positions still receive their (nonzero) gradient
    assert (np.abs(dw[~keep]) > 0).mean() > 0.99


# ---------------------------------------------------------------- pack (a9, a10)
def test_pack_hand_packed_rows():
    lines = _read_kv(os.path.join(GOLDEN, "packed_rows.txt"))
    cases = []
    for key, vals in lines:
        if key == "case":
            cases.append({"N": int(vals[0]), "M": int(vals[1])})
        else:
            cases[-1][key] = vals
    assert len(cases) == 4
    for c in cases:
        N, M = c["N"], c["M"]
        weff = np.array([int(v) for v in c["weff"]], np.int8).reshape(1, -1)
        p = oracle.pack(weff, N, M)
        crow, irow, total = oracle.packed_layout(1, weff.shape[1], N, M)
        assert (crow, irow, total) == (16, 16, 32)
        want = np.zeros(32, np.uint8)
        for i, b in enumerate(c["codes"]):
            want[i] = int(b, 16)
        for i, b in enumerate(c["index"]):
            want[16 + i] = int(b, 16)
        assert np.array_equal(p, want), (p, want)
        assert np.array_equal(oracle.unpack(p, 1, weff.shape[1], N, M), weff)


@pytest.mark.parametrize("N,M", [(6, 8), (2, 4), (8, 8), (2, 8), (3, 8), (5, 8), (1, 4), (3, 4), (4, 4)])
def test_pack_roundtrip(N, M):
    w = synth.bits(synth.trimodal_weight(6, 96, seed=14))
    weff, _, _ = oracle.effective_weight(w, N, M)
    p = oracle.pack(weff, N, M)
    crow, irow, total = oracle.packed_layout(6, 96, N, M)
    assert p.size == total and crow % 16 == 0 and irow % 16 == 0
    assert np.array_equal(oracle.unpack(p, 6, 96, N, M), weff)
    # every slot mask has exactly N bits; bits per weight = (2N + M) / M
    assert (2 * N + M) * 96 // M <= 8 * (crow + irow)


def test_pack_rejects_too_many_nonzeros():
    with pytest.raises(ValueError):
        oracle.pack(np.ones((1, 8), np.int8), 6, 8)


def test_gemv_packed_equals_forward():
    x = synth.activations(3, 128, seed=15)
    w = synth.bits(synth.trimodal_weight(20, 128, seed=15))
    weff, gamma, _ = oracle.effective_weight(w, 6, 8)
    xq, amax = oracle.act_quant(synth.bits(x))
    y = oracle.gemv_packed(xq, amax, oracle.pack(weff, 6, 8), gamma, 128, 20, 6, 8)
    assert np.array_equal(y, oracle.forward_out(oracle.forward_acc(xq, weff), gamma, amax))


# ---------------------------------------------------------------- dense 2-bit layout
def test_dense2_hand_packed_rows():
    cases = []
    for key, vals in _read_kv(os.path.join(GOLDEN, "dense2_rows.txt")):
        if key == "case":
            cases.append({})
        else:
            cases[-1][key] = vals
    assert len(cases) == 2
    for c in cases:
        weff = np.array([int(v) for v in c["weff"]], np.int8).reshape(1, -1)
        p = oracle.pack_dense2(weff)
        want = np.zeros(16, np.uint8)
        for i, b in enumerate(c["codes"]):
            want[i] = int(b, 16)
        assert np.array_equal(p, want), (p, want)
        assert np.array_equal(oracle.unpack_dense2(p, 1, 8), weff)


@pytest.mark.parametrize("N,M", [(6, 8), (2, 4), (8, 8)])
def test_dense2_roundtrip_and_8of8_codes_plane(N, M):
    """Round trip, and the dense layout equals the codes plane of the 8:8
    packed format (every position a slot)."""
    w = synth.bits(synth.trimodal_weight(5, 96, seed=16))
    weff, _, _ = oracle.effective_weight(w, N, M)
    d = oracle.pack_dense2(weff)
    assert np.array_equal(oracle.unpack_dense2(d, 5, 96), weff)
    crow, _, _ = oracle.packed_layout(5, 96, 8, 8)
    assert np.array_equal(d, oracle.pack(weff, 8, 8)[:5 * crow])


# ---------------------------------------------------------------- 2:4 sparse operand (a8)
def test_sparse24_hand_compressed_row():
    kv = dict(_read_kv(os.path.join(GOLDEN, "sparse24_row.txt")))
    d_out, d_in = int(kv["d_out"][0]), int(kv["d_in"][0])
    weff = np.array([int(v) for v in kv["weff"]], np.int8).reshape(d_out, d_in)
    buf = oracle.compress24(weff)
    vrow, meta_off, total, KB, MB = oracle.sparse24_layout(d_out, d_in)
    assert total == int(kv["total"][0]) and meta_off == int(kv["meta_off"][0]) and buf.size == total
    assert [f"{b:02x}" for b in buf[:vrow]] == kv["values"]
    assert np.all(buf[vrow:meta_off] == 0)
    meta = buf[meta_off:]
    assert [f"{b:02x}" for b in meta[:2]] == kv["meta"]
    assert np.all(meta[2:] == 0x44)
    assert np.array_equal(oracle.decompress24(buf, d_out, d_in), weff)


def test_sparse24_every_group_pattern():
    """All 81 ternary groups of four: two or fewer nonzeros compress to the
    slots the definition names, anything more is rejected."""
    import itertools
    for grp in itertools.product((-1, 0, 1), repeat=4):
        w = np.array(list(grp) + [0] * 12, np.int8).reshape(1, 16)
        nz = [p for p in range(4) if grp[p] != 0]
        if len(nz) > 2:
            with pytest.raises(ValueError):
                oracle.compress24(w)
            continue
        slots = sorted(nz + [p for p in range(4) if grp[p] == 0][: 2 - len(nz)])
        buf = oracle.compress24(w)
        assert buf[0] == np.uint8(grp[slots[0]] & 0xFF) and buf[1] == np.uint8(grp[slots[1]] & 0xFF)
        _, meta_off, _, _, _ = oracle.sparse24_layout(1, 16)
        assert buf[meta_off] & 0xF == slots[0] | (slots[1] << 2)
        assert np.array_equal(oracle.decompress24(buf, 1, 16), w)


def test_sparse24_block_placement():
    """The selector of one group lands at the byte worked out by hand:
    row 300, weights 388..391 of a 520 x 520 weight.  Row blocks of 128:
    mb = 2, r = 44; weight blocks of 256: kb = 1, offset 132 -> half 1,
    weight 4 of the half -> group 1 -> byte 0, high nibble.  KB = 3, so the
    half starts at ((2 * 3 + 1) * 2 + 1) * 2048 = 30720 and the byte is
    30720 + 44 * 16 = 31424 bytes into the selector plane."""
    w = np.zeros((520, 520), np.int8)
    w[300, 388 + 1] = 1
    w[300, 388 + 3] = -1
    buf = oracle.compress24(w)
    vrow, meta_off, total, KB, MB = oracle.sparse24_layout(520, 520)
    assert (vrow, KB, MB) == (260 + 12, 3, 6)
    meta = buf[meta_off:]
    assert meta[31424] == (0x4 | ((1 | 3 << 2) << 4))
    meta2 = meta.copy()
    meta2[31424] = 0x44
    assert np.all(meta2 == 0x44)
    assert buf[300 * vrow + 2 * 97] == 1 and buf[300 * vrow + 2 * 97 + 1] == 0xFF


def test_sparse24_product_and_roundtrip_ragged():
    """On 2:4 weights from the full weight step (ragged in both dimensions),
    the product formed from kept values and selected activations equals the
    dense product of W_eff, including the int8 extremes."""
    w = synth.bits(synth.trimodal_weight(392, 784, seed=21))
    weff, _, _ = oracle.effective_weight(w, 2, 4)
    buf = oracle.compress24(weff)
    assert np.array_equal(oracle.decompress24(buf, 392, 784), weff)
    rng = np.random.default_rng(21)
    xq = rng.integers(-128, 128, size=(19, 784)).astype(np.int8)
    xq[0] = -128
    xq[1] = 127
    assert np.array_equal(oracle.forward_acc_sparse24(xq, buf, 392, 784), oracle.forward_acc(xq, weff))


# ---------------------------------------------------------------- Norm before Q_a (NEXT: fused norm + quant)
def test_f32_to_bf16_matches_torch():
    rng = np.random.default_rng(21)
    v = np.concatenate([rng.normal(0, 3, 4000).astype(np.float32),
                        # exact halfway points between neighbouring bf16 values
                        ((np.arange(1, 200, dtype=np.uint32) << 16) | 0x8000).view(np.float32)])
    want = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(oracle.f32_to_bf16(v), want)


def test_rms_norm_hand_row():
    """x = [3, 4, 0, 0], g = 1, eps = 0: ss = 25, v = 6.25, r = 0.4;
    xn = bf16(1.2), bf16(1.6), 0, 0 = 0x3F9A (1.203125), 0x3FCD (1.6015625);
    Q_a: amax 1.6015625, codes rint(1.203125 * 127 / 1.6015625) = 95, 127."""
    x = synth.bits(torch.tensor([[3.0, 4.0, 0.0, 0.0]]).to(torch.bfloat16))
    g = synth.bits(torch.ones(4).to(torch.bfloat16))
    xn, xq, amax = oracle.rms_norm_act_quant(x, g, 0.0)
    assert xn.tolist() == [[0x3F9A, 0x3FCD, 0, 0]]
    assert xq.tolist() == [[95, 127, 0, 0]]
    assert amax.tolist() == [1.6015625]


def test_rms_norm_matches_torch_fp64():
    x = synth.activations(64, 896, seed=22, outlier_frac=0.01)
    g = (torch.rand(896, generator=torch.Generator().manual_seed(5)) + 0.5).to(torch.bfloat16)
    xn, _ = oracle.rms_norm(synth.bits(x), synth.bits(g), 1e-6)
    ref = torch.nn.functional.rms_norm(x.double(), (896,), g.double(), eps=1e-6)
    got = oracle.bf16_to_f32(xn).astype(np.float64)
    # within one bf16 ulp of the fp64 result, and equal to its bf16 rounding almost everywhere
    ulp = np.abs(ref.float().to(torch.bfloat16).float().numpy()) * 2.0 ** -7
    assert np.all(np.abs(got - ref.numpy()) <= ulp + 1e-30)
    assert (xn == synth.bits(ref.float().to(torch.bfloat16))).mean() > 0.99


def test_rms_norm_special_rows():
    g = synth.bits(torch.ones(16).to(torch.bfloat16))
    zero = np.zeros((1, 16), np.uint16)
    xn, xq, amax = oracle.rms_norm_act_quant(zero, g, 1e-6)
    assert not xn.any() and not xq.any() and amax.tolist() == [np.float32(1e-5)]
    const = synth.bits(torch.full((1, 16), -0.75).to(torch.bfloat16))
    xn, xq, _ = oracle.rms_norm_act_quant(const, g, 0.0)
    assert np.all(oracle.bf16_to_f32(xn) == -1.0) and np.all(xq == -127)
    # eps = 0: scaling x by a power of two leaves xn unchanged, bit for bit
    x = synth.bits(synth.activations(8, 64, seed=23))
    x2 = synth.bits(torch.from_numpy(oracle.bf16_to_f32(x) * 8.0).to(torch.bfloat16))
    assert np.array_equal(oracle.rms_norm(x, synth.bits(torch.ones(64).to(torch.bfloat16)), 0.0)[0],
                          oracle.rms_norm(x2, synth.bits(torch.ones(64).to(torch.bfloat16)), 0.0)[0])


# ---------------------------------------------------------------- ablations (NEXT rank 3)
@pytest.mark.parametrize("N,M", [(6, 8), (2, 4), (4, 8)])
def test_mask_from_quantised_keeps_nonzeros_first(N, M):
    """Pi_N:M(|W_q|): per group the kept positions are the nonzero ternary
    positions in ascending order, then the lowest zero positions, N in all
    (a direct restatement, checked against the rank rule)."""
    w = synth.bits(synth.trimodal_weight(12, 64, seed=31))
    weff, gamma, keep = oracle.effective_weight_mask_from_quantised(w, N, M)
    wq = oracle.ternary(w, gamma)
    for row in range(12):
        for g in range(64 // M):
            grp = wq[row, g * M:(g + 1) * M]
            order = [p for p in range(M) if grp[p] != 0] + [p for p in range(M) if grp[p] == 0]
            want = np.zeros(M, bool)
            want[order[:N]] = True
            assert np.array_equal(keep[row, g * M:(g + 1) * M], want)
    # it keeps at least as many nonzero codes as the mask from |W| does
    weff_w, _, _ = oracle.effective_weight(w, N, M)
    assert (weff != 0).sum() >= (weff_w != 0).sum()


def test_masked_grad_equals_autograd_of_masked_weight():
    """dW (.) M is the gradient of y = x (W (.) M)^T with M held constant."""
    x = synth.activations(6, 32, seed=32)
    dy = synth.grad_output(6, 16, seed=32)
    w = synth.bits(synth.normal_weight(16, 32, seed=32))
    keep = oracle.nm_mask(w, 6, 8)
    wv = torch.from_numpy(oracle.bf16_to_f32(w).astype(np.float64)).requires_grad_(True)
    xm = torch.from_numpy(oracle.bf16_to_f32(synth.bits(x)).astype(np.float64))
    (xm @ (wv * torch.from_numpy(keep)).T).backward(
        torch.from_numpy(oracle.bf16_to_f32(synth.bits(dy)).astype(np.float64)))
    got = oracle.masked_grad(oracle.backward_dw(synth.bits(dy), synth.bits(x)), keep)
    np.testing.assert_allclose(got, wv.grad.numpy(), rtol=1e-6, atol=1e-6)
    assert not got[~keep].any()
