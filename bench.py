#!/usr/bin/env python
"""Sparse-BitLinear training-step benchmark (forward + Dual-STE backward).

One step = the whole hot path over one batch of the Qwen2.5-3B-shaped layer
set (q/o 2048x2048, k/v 256x2048, gate/up 11008x2048, down 2048x11008),
32768 tokens (16 x 2048), 6:8:

  for every projection:  sbl_mask_quant   (mask, gamma, ternary, quant-then-mask;
                                           on three side streams)
  for every input:       sbl_act_quant    (attn_in, o_in, mlp_in, down_in; main
                                           stream, overlapped with the above)
  for every projection:  sbl_forward      (int8 tcgen05 product; at N:M = 2:4,
                                           sbl_compress24 + the sparse MMA)
                         sbl_backward     (bf16 tcgen05 dX, then dW)

Inputs are seeded synthetic tensors (synth): trimodal bf16 master weights,
X ~ N(0, 1) with 0.1% outlier channels x10, dY ~ N(0, 1).  The per-step
working set (about 11 GB) is far larger than the 126 MB L2, so no L2 flush
is needed between steps.

Prints ONE JSON line (rank 0).  ``--impl reference`` times the CPU oracle on
a bounded sample of the same workload instead.  Under torchrun (N > 1) each
rank runs an independent batch (weak scaling); there is no collective on the
data path.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

WORKLOADS = {
    # name: (default tokens, weight distribution, outlier fraction of X channels, boundary-tie groups)
    "qwen2.5-3b": (32768, "trimodal", 0.001, 0.0),
    "qwen2.5-0.5b": (4096, "normal", 0.0, 0.0),
    "qwen2.5-3b-up": (8192, "trimodal", 0.001, 0.01),
}
N_KEEP, M_GROUP = 6, 8
SPARSE24 = False  # --sparse24: 2:4 layers use the sparse tensor core
METRIC = "Sparse-BitLinear fwd+bwd tokens/s (3B-shape, 6:8)"

NOMINAL_I8_OVER_BF16 = 2.0  # dense int8 / dense bf16 tensor throughput (4.5 / 2.25 PFLOP/s)


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(hbm=d["hbm_gbs"], bf16=d["bf16_tflops"], bf16_sust=d.get("bf16_tflops_sustained",
                    d["bf16_tflops"]), src="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sust=1400.0, src="fallback")


# ----------------------------------------------------------------- inputs
def make_weight(ls, i, p):
    _, dist, _, ties = WORKLOADS[ls.name]
    if dist == "trimodal":
        w = synth.trimodal_weight(p.d_out, p.d_in, seed=0, tensor_id=i)
    else:
        w = synth.normal_weight(p.d_out, p.d_in, seed=0, tensor_id=i)
    if ties > 0 and N_KEEP < M_GROUP:
        w = synth.with_boundary_ties(w, N_KEEP, M_GROUP, seed=0, tensor_id=300 + i, frac=ties)
    return w


def make_inputs(ls, T, seed, device):
    """Seeded synthetic tensors for one step, on `device` (CPU pinned or cuda)."""
    W, X, dY = {}, {}, {}
    outl = WORKLOADS[ls.name][2]
    for i, p in enumerate(ls.projections):
        W[p.name] = make_weight(ls, i, p)  # replicated across ranks
    for j, (name, d_in) in enumerate(ls.inputs.items()):
        X[name] = synth.activations(T, d_in, seed=seed, tensor_id=100 + j, outlier_frac=outl)
    for i, p in enumerate(ls.projections):
        dY[p.name] = synth.grad_output(T, p.d_out, seed=seed, tensor_id=200 + i)
    if device == "pinned":
        f = lambda t: t.pin_memory()  # noqa: E731
    else:
        f = lambda t: t.to(device)  # noqa: E731
    return ({k: f(v) for k, v in W.items()}, {k: f(v) for k, v in X.items()},
            {k: f(v) for k, v in dY.items()})


class Step:
    """Device buffers for one step and the sequence of C-ABI calls."""

    def __init__(self, ls, T, W, X, dY):
        import semi_structured_sparsity_step_b200 as sbl
        from semi_structured_sparsity_step_b200.layer import SparseBitLinearLayer
        self.sbl, self.ls, self.T = sbl, ls, T
        self.W, self.X, self.dY = W, X, dY
        dev = "cuda"
        self.layers = {p.name: SparseBitLinearLayer(W[p.name], N_KEEP, M_GROUP, sparse24=SPARSE24)
                       for p in ls.projections}
        self.Xq = {n: torch.empty(T, d, dtype=torch.int8, device=dev) for n, d in ls.inputs.items()}
        self.amax = {n: torch.empty(T, dtype=torch.float32, device=dev) for n in ls.inputs}
        self.Y = {p.name: torch.empty(T, p.d_out, dtype=torch.float32, device=dev) for p in ls.projections}
        self.dX = {p.name: torch.empty(T, p.d_in, dtype=torch.float32, device=dev) for p in ls.projections}
        self.dW = {p.name: torch.empty(p.d_out, p.d_in, dtype=torch.float32, device=dev) for p in ls.projections}
        n_p, n_x = len(ls.projections), len(ls.inputs)
        # the weight steps (mask, gamma, ternary) of the projections are
        # independent of the activation quantisation: they run on side streams,
        # overlapped with act_quant on the main stream, and join before the
        # forward products
        self.side = [torch.cuda.Stream() for _ in range(3)]
        self.sparse24 = SPARSE24 and (N_KEEP, M_GROUP) == (2, 4)  # compress + sparse tensor-core forward
        self.kernels_per_step = 2 * n_p + n_x + 3 * n_p + (n_p if self.sparse24 else 0)

    def run(self, stream, ev=None):
        """Enqueue one step.  With `ev` (dict name -> list), record event pairs per call."""
        sbl, ls, T = self.sbl, self.ls, self.T

        def timed(name, fn):
            if ev is None:
                fn()
                return
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            ev.setdefault(name, []).append((a, b))

        def weight_and_act_quant():
            fork = torch.cuda.Event()
            fork.record(stream)
            for sd in self.side:
                sd.wait_event(fork)
            for i, p in enumerate(ls.projections):
                self.layers[p.name].weight_step(self.side[i % len(self.side)])
            for n, d in ls.inputs.items():
                sbl.sbl_act_quant(self.X[n], T, d, self.Xq[n], self.amax[n], stream)
            for sd in self.side:
                join = torch.cuda.Event()
                join.record(sd)
                stream.wait_event(join)

        timed("weight_and_act_quant", weight_and_act_quant)
        for p in ls.projections:
            L = self.layers[p.name]
            timed("forward_i8", lambda p=p, L=L: L.forward(self.Xq[p.input_name], self.amax[p.input_name],
                                                           self.Y[p.name], stream=stream))
        for p in ls.projections:
            L = self.layers[p.name]
            timed("backward_dx_bf16", lambda p=p, L=L: L.backward(self.dY[p.name], self.X[p.input_name],
                                                                  self.dX[p.name], None, stream=stream))
            timed("backward_dw_bf16", lambda p=p, L=L: L.backward(self.dY[p.name], self.X[p.input_name],
                                                                  None, self.dW[p.name], stream=stream))


def algorithmic_work(ls, T):
    P = ls.params
    fwd_ops = 2.0 * T * P          # dense-equivalent int8 ops
    dx_flops = 2.0 * T * P
    dw_flops = 2.0 * T * P
    return fwd_ops, dx_flops, dw_flops


# ----------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.lines = []
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except (OSError, ValueError):
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for nm, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------- CPU oracle timing
def oracle_sample(ls, T_full, tokens=128, seed=0):
    """Time the oracle as it stands on a bounded sample of the workload and
    extrapolate to one full step: the weight side of the q projection scaled
    by parameter count, the token side of all projections on `tokens` tokens
    scaled to T_full tokens."""
    import oracle
    q = ls.projections[0]
    wq = synth.bits(make_weight(ls, 0, q))
    t0 = time.perf_counter()
    oracle.effective_weight(wq, N_KEEP, M_GROUP)
    t_w = time.perf_counter() - t0
    weight_side = t_w * ls.params / (q.d_out * q.d_in)
    outl = WORKLOADS[ls.name][2]
    xs = {n: synth.bits(synth.activations(tokens, d, seed=seed, tensor_id=100 + j, outlier_frac=outl))
          for j, (n, d) in enumerate(ls.inputs.items())}
    t_tok = 0.0
    weffs = {}
    for i, p in enumerate(ls.projections):
        weffs[p.name] = oracle.effective_weight(synth.bits(make_weight(ls, i, p)), N_KEEP, M_GROUP)
    for n in ls.inputs:
        t0 = time.perf_counter()
        oracle.act_quant(xs[n])
        t_tok += time.perf_counter() - t0
    for i, p in enumerate(ls.projections):
        weff, gamma, _ = weffs[p.name]
        dy = synth.bits(synth.grad_output(tokens, p.d_out, seed=seed, tensor_id=200 + i))
        xq, amax = oracle.act_quant(xs[p.input_name])
        t0 = time.perf_counter()
        oracle.forward_out(oracle.forward_acc(xq, weff), gamma, amax)
        oracle.backward_dx(dy, weff, gamma)
        oracle.backward_dw(dy, xs[p.input_name])
        t_tok += time.perf_counter() - t0
    token_side = t_tok * T_full / tokens
    step_s = weight_side + token_side
    try:
        from threadpoolctl import threadpool_info
        cores = max([1] + [d.get("num_threads", 1) for d in threadpool_info()])
    except Exception:  # pragma: no cover
        cores = 1
    sample = (f"oracle weight side on {q.name} ({q.d_out}x{q.d_in}) scaled x{ls.params / (q.d_out * q.d_in):.2f} "
              f"by parameter count + token side of all {len(ls.projections)} projections on {tokens} tokens "
              f"scaled x{T_full // tokens}; extrapolated")
    return step_s, cores, sample, t_w + t_tok


# ----------------------------------------------------------------- traffic (ncu)
def _kernel_source_hash():
    h = hashlib.sha256()
    for f in ("gemm_tc.cu", "sbl_device.cuh"):
        h.update(open(os.path.join(ROOT, "semi_structured_sparsity_step_b200", "csrc", f), "rb").read())
    return h.hexdigest()[:16]


def traffic_for(kernel_key):
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p))
    e = d.get(kernel_key)
    if not e or e.get("source_hash") != _kernel_source_hash():
        return None
    return e.get("bytes_per_launch")


# ----------------------------------------------------------------- decode
def run_decode(args):
    """Decode GEMV on the packed 6:8 format: a stack of `layers` distinct 3B
    layer sets (each projection packed separately), batch 1 / 8 / 16 tokens,
    int8 activations (absmax-quantised N(0, 1)).  One pass over the stack is
    captured in a CUDA graph; bytes = packed weights + int8 activations +
    fp32 outputs actually touched.  The stack (~0.87 GB at 36 layers) is far
    larger than L2, so every pass streams the weights from HBM."""
    import semi_structured_sparsity_step_b200 as sbl
    from semi_structured_sparsity_step_b200.layer import act_quant
    torch.cuda.set_device(0)
    sbl.sbl_set_gemv_variant(args.gemv_variant)
    ls = synth.layer_set("qwen2.5-3b")
    layers = args.layers
    g = torch.Generator(device="cuda")
    g.manual_seed(7)
    # Distinct random ternary 6:8 weights per layer, packed on the device: the
    # weight side (mask_quant) runs once per projection on random bf16 master
    # weights drawn on the device, then sbl_pack.
    packs, dense = [], []  # the packed 6:8 format, and the dense 2-bit layout of the same weights
    for l in range(layers):
        for p in ls.projections:
            w = (torch.randn(p.d_out, p.d_in, generator=g, device="cuda") * 0.02).to(torch.bfloat16)
            from semi_structured_sparsity_step_b200.layer import SparseBitLinearLayer
            L = SparseBitLinearLayer(w, N_KEEP, M_GROUP)
            L.weight_step()
            nbytes = sbl.sbl_packed_bytes(p.d_out, p.d_in, N_KEEP, M_GROUP)
            pk = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
            sbl.sbl_pack(L.W_eff, p.d_out, p.d_in, N_KEEP, M_GROUP, pk, nbytes)
            nb2 = sbl.sbl_dense2_bytes(p.d_out, p.d_in)
            d2 = torch.empty(nb2, dtype=torch.uint8, device="cuda")
            sbl.sbl_pack_dense2(L.W_eff, p.d_out, p.d_in, d2, nb2)
            packs.append((p, pk, L.gamma.clone(), nbytes))
            dense.append((d2, nb2))
            del L, w
    sbl.sbl_check()
    torch.cuda.empty_cache()
    pk_bytes = sum(x[3] for x in packs)
    d2_bytes = sum(x[1] for x in dense)
    results, results_d2 = {}, {}
    pkk = peaks()
    for batch in (1, 8, 16):
        xs = {}
        for n, d in ls.inputs.items():
            x = torch.randn(batch, d, generator=g, device="cuda").to(torch.bfloat16)
            xq = torch.empty(batch, d, dtype=torch.int8, device="cuda")
            am = torch.empty(batch, dtype=torch.float32, device="cuda")
            act_quant(x, xq, am)
            xs[n] = (xq, am)
        ys = [torch.empty(batch, p.d_out, dtype=torch.float32, device="cuda") for (p, _, _, _) in packs]
        stream = torch.cuda.Stream()

        per_layer = len(ls.projections)
        groups, groups_d2 = [], []
        for l in range(layers):
            probs, probs_d2 = [], []
            sl = slice(l * per_layer, (l + 1) * per_layer)
            for (p, pk, gm, _), (d2, _), y in zip(packs[sl], dense[sl], ys[sl]):
                xq, am = xs[p.input_name]
                probs.append((pk, xq, am, gm, y, p.d_in, p.d_out))
                probs_d2.append((d2, xq, am, gm, y, p.d_in, p.d_out))
            groups.append(probs)
            groups_d2.append(probs_d2)

        for variant in ("packed", "dense2"):
            ms = _decode_pass_ms(sbl, stream, groups if variant == "packed" else groups_d2, batch, variant, args)
            act_bytes = sum(batch * p.d_in + 4 * batch for (p, _, _, _) in packs)
            out_bytes = sum(4 * batch * p.d_out for (p, _, _, _) in packs)
            wb = pk_bytes if variant == "packed" else d2_bytes
            tot = wb + act_bytes + out_bytes
            gbs = tot / (ms / 1e3) / 1e9
            (results if variant == "packed" else results_d2)[str(batch)] = {
                "ms_per_pass": ms, "bytes_per_pass": tot, "weight_bytes": wb, "achieved_gbs": gbs,
                "frac_hbm": gbs / pkk["hbm"], "tokens_per_s_36_layers": batch / (ms / 1e3),
                "gemv_launches_per_pass": layers}
    print(json.dumps({"metric": "Sparse-BitLinear packed decode GEMV, HBM bytes/s", "unit": "GB/s",
                      "workload": f"{layers} distinct qwen2.5-3b layer sets, packed 6:8 (2.5 bit/weight), "
                                  f"batch 1/8/16, one grouped GEMV launch per layer (7 projections), CUDA graph per pass",
                      "gemv_kernel": ["per-warp streaming", "block-wide TMA ring"][args.gemv_variant],
                      "peak_hbm_gbs": pkk["hbm"], "peak_source": pkk["src"], "results": results,
                      "dense2": {"layout": "dense 2-bit codes of the same weights (2.0 bit/weight, no index plane)",
                                 "results": results_d2}}))


def _decode_pass_ms(sbl, stream, groups, batch, variant, args):
    """ms per pass over the layer stack (one grouped GEMV launch per layer),
    captured in a CUDA graph and replayed."""
    def one_pass():
        for probs in groups:
            if variant == "packed":
                sbl.sbl_gemv_packed_group(probs, batch, N_KEEP, M_GROUP, stream)
            else:
                sbl.sbl_gemv_dense2_group(probs, batch, stream)

    with torch.cuda.stream(stream):
        for _ in range(2):
            one_pass()
    stream.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        one_pass()
    for _ in range(args.warmup):
        graph.replay()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    reps = max(args.steps, 5)
    e0.record(stream)
    with torch.cuda.stream(stream):
        for _ in range(reps):
            graph.replay()
    e1.record(stream)
    stream.synchronize()
    sbl.sbl_check()
    del graph
    return e0.elapsed_time(e1) / reps


# ----------------------------------------------------------------- prefill
def run_prefill(args):
    """Prefill forward on the packed 6:8 format of the 3B layer set: per
    projection, int8 activations (absmax-quantised N(0, 1)) times the packed
    weight: expanded in shared memory for every token tile
    (sbl_forward_packed), unpacked once per pass and multiplied by the dense
    int8 kernel (sbl_unpack + sbl_forward_group), and from an int8 W_eff that
    is already resident (sbl_forward per projection, and sbl_forward_group,
    which runs short batches in one launch).  Shapes: 512 tokens (1 x 512), 8192
    (8 x 1024) and 32768 (16 x 2048).  One pass = the seven projections;
    passes are captured in a CUDA graph (16 passes per replay at 512 tokens,
    2 at 8192, 1 at 32768); int8 ops = 2 T P (dense-equivalent)."""
    import semi_structured_sparsity_step_b200 as sbl
    from semi_structured_sparsity_step_b200.layer import SparseBitLinearLayer, act_quant
    torch.cuda.set_device(0)
    ls = synth.layer_set("qwen2.5-3b")
    g = torch.Generator(device="cuda")
    g.manual_seed(11)
    layers = []
    for i, p in enumerate(ls.projections):
        w = make_weight(ls, i, p).cuda()
        L = SparseBitLinearLayer(w, N_KEEP, M_GROUP)
        L.weight_step()
        nbytes = sbl.sbl_packed_bytes(p.d_out, p.d_in, N_KEEP, M_GROUP)
        pk = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
        sbl.sbl_pack(L.W_eff, p.d_out, p.d_in, N_KEEP, M_GROUP, pk, nbytes)
        layers.append((p, L, pk))
    unpacked = [torch.empty(p.d_out, p.d_in, dtype=torch.int8, device="cuda") for (p, _, _) in layers]
    sbl.sbl_check()
    pk_peak = peaks()
    i8_peak = pk_peak["bf16"] * NOMINAL_I8_OVER_BF16  # burst: each pass is timed on its own
    results = {}
    stream = torch.cuda.Stream()
    for T in (512, 8192, 32768):
        xs = {}
        for n, d in ls.inputs.items():
            x = torch.randn(T, d, generator=g, device="cuda").to(torch.bfloat16)
            xq = torch.empty(T, d, dtype=torch.int8, device="cuda")
            am = torch.empty(T, dtype=torch.float32, device="cuda")
            act_quant(x, xq, am)
            xs[n] = (xq, am)
        ys = [torch.empty(T, p.d_out, dtype=torch.float32, device="cuda") for (p, _, _) in layers]

        def one_pass(variant):
            for (p, L, pk), y, wk in zip(layers, ys, unpacked):
                xq, am = xs[p.input_name]
                if variant == "packed":      # weight decoded in shared memory for every token tile
                    sbl.sbl_forward_packed(xq, am, pk, L.gamma, T, p.d_in, p.d_out, N_KEEP, M_GROUP, y, None, stream)
                elif variant == "unpack_int8":  # decoded once per pass, then the dense int8 products
                    sbl.sbl_unpack(pk, p.d_out, p.d_in, N_KEEP, M_GROUP, wk, stream)
                elif variant == "int8_weff":  # int8 W_eff already resident (training layout)
                    sbl.sbl_forward(xq, am, L.W_eff, L.gamma, T, p.d_in, p.d_out, y, None, stream)
            if variant in ("unpack_int8", "int8_weff_grouped"):  # the seven products through sbl_forward_group
                weights = unpacked if variant == "unpack_int8" else [L.W_eff for (_, L, _) in layers]
                sbl.sbl_forward_group([(xs[p.input_name][0], xs[p.input_name][1], w, L.gamma, T, p.d_in, p.d_out,
                                        y, None) for (p, L, _), y, w in zip(layers, ys, weights)], stream)

        row = {}
        for variant in ("packed", "unpack_int8", "int8_weff", "int8_weff_grouped"):
            with torch.cuda.stream(stream):
                for _ in range(2):
                    one_pass(variant)
            stream.synchronize()
            # several passes per replay for short passes, so the host's cost of
            # a replay never shows in the device timing
            per_graph = 16 if T <= 1024 else (2 if T <= 8192 else 1)
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph, stream=stream):
                for _ in range(per_graph):
                    one_pass(variant)
            for _ in range(args.warmup):
                graph.replay()
            stream.synchronize()
            reps = max(args.steps, 5)
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            with torch.cuda.stream(stream):
                for _ in range(reps):
                    graph.replay()
            e1.record(stream)
            stream.synchronize()
            del graph
            ms = e0.elapsed_time(e1) / (reps * per_graph)
            tops = 2.0 * T * ls.params / (ms / 1e3) / 1e12
            row[variant] = {"ms_per_pass": ms, "tokens_per_s": T / (ms / 1e3), "int8_tops": tops,
                            "frac_int8_peak": tops / i8_peak}
        sbl.sbl_check()
        results[str(T)] = row
        del xs, ys
        torch.cuda.empty_cache()
    print(json.dumps({"metric": "Sparse-BitLinear prefill forward on the packed 6:8 format (3B layer set)",
                      "unit": "tokens/s", "peak_int8_tops": i8_peak,
                      "peak_source": f"{pk_peak['src']} bf16 burst x2 nominal int8/bf16",
                      "workload": "qwen2.5-3b layer set, 6:8 packed (2.5 bit/weight), T = 512 / 8192 / 32768, "
                                  "Xq from absmax-quantised N(0,1), fp32 outputs",
                      "results": results}))


# ----------------------------------------------------------------- fused norm + act quant
def run_normquant(args):
    """Q_a(RMSNorm(x)) on the four distinct inputs of the 3B step (attn_in,
    o_in, mlp_in, down_in; T = 32768, X ~ N(0, 1) with 0.1% outlier channels,
    gain ~ U(0.5, 1.5)): the fused kernel (reads X, writes Xn and Xq; and
    without the optional Xn) against sbl_act_quant alone on the same X (reads
    X, writes Xq).  CUDA events, inputs far larger than L2."""
    import semi_structured_sparsity_step_b200 as sbl
    torch.cuda.set_device(0)
    ls = synth.layer_set("qwen2.5-3b")
    T = args.tokens or 32768
    g_gen = torch.Generator().manual_seed(3)
    bufs = []
    for j, (name, d) in enumerate(ls.inputs.items()):
        x = synth.activations(T, d, seed=0, tensor_id=100 + j, outlier_frac=0.001).cuda()
        g = (torch.rand(d, generator=g_gen) + 0.5).to(torch.bfloat16).cuda()
        bufs.append((x, g, d, torch.empty(T, d, dtype=torch.bfloat16, device="cuda"),
                     torch.empty(T, d, dtype=torch.int8, device="cuda"), torch.empty(T, dtype=torch.float32,
                                                                                    device="cuda")))
    stream = torch.cuda.Stream()

    def pass_(variant):
        for x, g, d, xn, xq, am in bufs:
            if variant == "rmsnorm_act_quant":
                sbl.sbl_rmsnorm_act_quant(x, g, 1e-6, T, d, xn, xq, am, stream)
            elif variant == "rmsnorm_act_quant_no_xn":
                sbl.sbl_rmsnorm_act_quant(x, g, 1e-6, T, d, None, xq, am, stream)
            else:
                sbl.sbl_act_quant(x, T, d, xq, am, stream)

    pk = peaks()
    out = {}
    for fused in ("rmsnorm_act_quant", "rmsnorm_act_quant_no_xn", "act_quant"):
        with torch.cuda.stream(stream):
            for _ in range(args.warmup):
                pass_(fused)
        stream.synchronize()
        reps = max(args.steps, 5)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        with torch.cuda.stream(stream):
            for _ in range(reps):
                pass_(fused)
        e1.record(stream)
        stream.synchronize()
        sbl.sbl_check()
        ms = e0.elapsed_time(e1) / reps
        elems = sum(T * d for (_, _, d, _, _, _) in bufs)
        nbytes = elems * (5 if fused == "rmsnorm_act_quant" else 3) + 4 * T * len(bufs)
        out[fused] = {
            "ms_per_pass": ms, "bytes": nbytes, "gbs": nbytes / (ms / 1e3) / 1e9,
            "frac_hbm": nbytes / (ms / 1e3) / 1e9 / pk["hbm"]}
    print(json.dumps({"metric": "Q_a(RMSNorm(x)) fused, HBM bytes/s", "unit": "GB/s", "tokens": T,
                      "workload": "the four distinct inputs of the qwen2.5-3b layer set", "peak_hbm_gbs": pk["hbm"],
                      "results": out}))


def run_optimizer(args):
    """The optimizer step over the 3B layer set (7 projections, 77 M weights):
    sbl_grad_sqnorm over every dW (the global clip norm), then one
    sbl_adamw_step per projection on three side streams (AdamW on the bf16
    master weight, clip at max_norm 1, the next step's exact gamma pass, the
    mask flip count, then the ternary pass).  Also the same with an fp32 master copy.  Inputs:
    trimodal bf16 weights, synthetic fp32 gradients and moments (synth),
    1.3 GB or more resident, far larger than L2.  CUDA events on the
    launching stream."""
    import semi_structured_sparsity_step_b200 as sbl
    torch.cuda.set_device(0)
    ls = synth.layer_set("qwen2.5-3b")
    N, M = N_KEEP, M_GROUP
    projs = []
    for i, p in enumerate(ls.projections):
        w = make_weight(ls, i, p).cuda()
        dw, m, v = synth.optimizer_state(p.d_out, p.d_in, seed=0, tensor_id=400 + i)
        ws_bytes = sbl.sbl_mask_quant_workspace_bytes(p.d_out, p.d_in)
        projs.append(dict(
            p=p, W=w, W32=w.float(), dW=dw.cuda(), m=m.cuda(), v=v.cuda(),
            weff=torch.empty(p.d_out, p.d_in, dtype=torch.int8, device="cuda"),
            weff16=torch.empty(p.d_out, p.d_in, dtype=torch.bfloat16, device="cuda"),
            bits=torch.empty(p.d_out, p.d_in // 8, dtype=torch.uint8, device="cuda"),
            gamma=torch.empty(1, dtype=torch.float32, device="cuda"),
            ws=torch.empty(ws_bytes, dtype=torch.uint8, device="cuda"), ws_bytes=ws_bytes))
    stream = torch.cuda.Stream()
    sumsq = torch.zeros(1, dtype=torch.float64, device="cuda")
    flips = torch.zeros(1, dtype=torch.int64, device="cuda")
    with torch.cuda.stream(stream):
        for q in projs:
            p = q["p"]
            sbl.sbl_mask_quant(q["W"], p.d_out, p.d_in, N, M, q["weff"], q["weff16"], q["bits"], q["gamma"],
                               q["ws"], q["ws_bytes"], stream)
    n_w = sum(q["p"].d_out * q["p"].d_in for q in projs)
    state = {"t": 1000}

    def sqnorm():
        sumsq.zero_()
        for q in projs:
            sbl.sbl_grad_sqnorm(q["dW"], q["dW"].numel(), sumsq, q["ws"], q["ws_bytes"], stream)

    # The projections' steps are independent once the global norm is known
    # (each has its own workspace; the flip counter is added atomically), so
    # they run on three side streams, largest first, as the training step runs
    # its weight steps; sbl_grad_sqnorm adds into one sum and stays in order on
    # the main stream.
    side = [torch.cuda.Stream() for _ in range(3)]
    by_size = sorted(projs, key=lambda q: -q["p"].d_out * q["p"].d_in)

    def adamw(master32):
        state["t"] += 1
        fork = torch.cuda.Event()
        fork.record(stream)
        for sd in side:
            sd.wait_event(fork)
        for i, q in enumerate(by_size):
            p = q["p"]
            sbl.sbl_adamw_step(q["W"], q["W32"] if master32 else None, q["dW"], q["m"], q["v"], p.d_out, p.d_in,
                               N, M, 1e-5, 0.9, 0.95, 1e-5, 0.1, state["t"], sumsq, 1.0, q["weff"], q["weff16"],
                               q["bits"], q["gamma"], flips, q["ws"], q["ws_bytes"], side[i % len(side)])
        for sd in side:
            join = torch.cuda.Event()
            join.record(sd)
            stream.wait_event(join)

    # algorithmic bytes per weight: adamw launch (W 2+2 or W32 4+4 and the bf16 W write, dW 4, m 4+4,
    # v 4+4, old mask 1/8) + ternary pass (W 2, W_eff 1, W_eff bf16 2, mask 1/8)
    bpw = {"grad_sqnorm": 4.0, "adamw_step_bf16_master": 24.125 + 5.125,
           "adamw_step_fp32_master": 30.125 + 5.125}
    fns = {"grad_sqnorm": sqnorm, "adamw_step_bf16_master": lambda: adamw(False),
           "adamw_step_fp32_master": lambda: adamw(True)}
    pk = peaks()
    out = {}
    with torch.cuda.stream(stream):
        sqnorm()
    for name, fn in fns.items():
        with torch.cuda.stream(stream):
            for _ in range(args.warmup):
                fn()
        stream.synchronize()
        reps = max(args.steps, 5)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        with torch.cuda.stream(stream):
            for _ in range(reps):
                fn()
        e1.record(stream)
        stream.synchronize()
        sbl.sbl_check()
        ms = e0.elapsed_time(e1) / reps
        gbs = bpw[name] * n_w / (ms / 1e3) / 1e9
        out[name] = {"ms_per_pass": ms, "bytes_per_weight": bpw[name], "gbs": gbs, "frac_hbm": gbs / pk["hbm"]}
    flip_rate = None
    with torch.cuda.stream(stream):
        flips.zero_()
        adamw(False)
    stream.synchronize()
    flip_rate = int(flips.item()) / n_w
    print(json.dumps({"metric": "optimizer step (AdamW + next weight step), HBM bytes/s", "unit": "GB/s",
                      "weights": n_w, "nm": args.nm, "lr": 1e-5,
                      "workload": "the seven projections of the qwen2.5-3b layer set",
                      "peak_hbm_gbs": pk["hbm"], "mask_flip_rate_one_step": flip_rate, "results": out}))


# ----------------------------------------------------------------- ranks
def rank_env():
    """(rank, world_size, local_rank) from the torchrun environment (1 process: 0, 1, 0)."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def max_over_ranks(value, dist=None, device="cpu"):
    """The largest `value` over all ranks (the job's time is its slowest rank's)."""
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.item()


def job_throughput(world, tokens_per_rank, ms_per_step):
    """Whole-job tokens/s: every rank runs its own batch (weak scaling) and the
    step time is the maximum over ranks."""
    return world * tokens_per_rank / (ms_per_step / 1e3)


# ----------------------------------------------------------------- main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=40)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["sbl", "reference"], default="sbl")
    ap.add_argument("--e2e-steps", type=int, default=6)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="qwen2.5-3b")
    ap.add_argument("--tokens", type=int, default=0, help="tokens per step (0: the workload's default)")
    ap.add_argument("--mode", choices=["train", "decode", "prefill", "normquant", "optimizer"], default="train")
    ap.add_argument("--layers", type=int, default=36, help="decode mode: distinct layer sets in the stack")
    ap.add_argument("--gemv-variant", type=int, default=0,
                    help="decode kernel: 0 per-warp streaming (default), 1 block-wide TMA ring")
    ap.add_argument("--nm", default="6:8", help="N:M of the mask (the sweep: 8:8, 6:8, 4:8, 2:8, 2:4)")
    ap.add_argument("--sparse24", action="store_true", help="2:4: forward on the sparse tensor core")
    args = ap.parse_args()
    global N_KEEP, M_GROUP, SPARSE24
    N_KEEP, M_GROUP = (int(v) for v in args.nm.split(":"))
    SPARSE24 = args.sparse24
    if args.mode == "decode":
        run_decode(args)
        return
    if args.mode == "prefill":
        run_prefill(args)
        return
    if args.mode == "normquant":
        run_normquant(args)
        return
    if args.mode == "optimizer":
        run_optimizer(args)
        return

    rank, world, local_rank = rank_env()
    ls = synth.layer_set(args.workload)
    T = args.tokens or WORKLOADS[args.workload][0]
    dist_name, outl, ties = WORKLOADS[args.workload][1:]
    shapes = ", ".join(f"{p.name} {p.d_out}x{p.d_in}" for p in ls.projections)
    config = {"workload": f"{args.workload} ({shapes}), {T} tokens, N:M {N_KEEP}:{M_GROUP}, {dist_name} bf16 "
                          f"master W" + (f" with {ties:.0%} boundary-tie groups" if ties else "") +
                          f", X ~ N(0,1)" + (f" with {outl:.1%} outlier channels x10" if outl else "") +
                          ", dY ~ N(0,1)",
              "tokens_per_step": T, "params": ls.params, "nm": f"{N_KEEP}:{M_GROUP}",
              "l2": "per-step working set larger than L2, no flush", "parallelism": f"dp{args.gpus} replicas",
              "forward_kernel": ("2:4 compress + sparse int8 MMA (tcgen05.mma.sp)"
                                 if SPARSE24 and (N_KEEP, M_GROUP) == (2, 4)
                                 else "dense int8 MMA (tcgen05.mma kind::i8)")}

    if args.impl == "reference":
        if rank != 0:
            return
        step_s, cores, sample, spent = oracle_sample(ls, T)
        v = T / step_s
        print(json.dumps({
            "impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_s * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "i8/bf16 (oracle: fp32/fp64/int64 on CPU)",
            "data": "synthetic", "config": config,
            "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": sample,
                             "cpu_seconds_spent": spent},
            "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        }))
        return

    torch.cuda.set_device(local_rank)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    import semi_structured_sparsity_step_b200 as sbl
    sbl.load()

    stream = torch.cuda.Stream()
    Wp, Xp, dYp = make_inputs(ls, T, seed=rank, device="pinned")
    with torch.cuda.stream(stream):
        W = {k: v.to("cuda", non_blocking=True) for k, v in Wp.items()}
        X = {k: v.to("cuda", non_blocking=True) for k, v in Xp.items()}
        dY = {k: v.to("cuda", non_blocking=True) for k, v in dYp.items()}
        step = Step(ls, T, W, X, dY)
    stream.synchronize()

    for _ in range(args.warmup):
        step.run(stream)
    sbl.sbl_check(stream)

    def barrier():
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()

    # ---- device-timed steps (inputs resident in HBM)
    ev = {}
    barrier()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    with ClockSampler(local_rank) as clk:
        start.record(stream)
        for _ in range(args.steps):
            step.run(stream, ev)
        end.record(stream)
        stream.synchronize()
    barrier()
    sbl.sbl_check(stream)
    elapsed_ms = max_over_ranks(start.elapsed_time(end), dist, "cuda")
    ms_per_step = elapsed_ms / args.steps
    value = job_throughput(world, T, ms_per_step)

    per_call = {k: sum(a.elapsed_time(b) for a, b in v) / args.steps for k, v in ev.items()}
    launches = {k: len(v) // args.steps for k, v in ev.items()}

    # ---- end to end through host buffers (pinned), copies inside the timed region.
    # Every step copies its inputs (W, X, dY) host -> device and its results
    # (y, dX, dW) device -> host.  Steps are pipelined on three streams over
    # two device buffer sets: the upload of step i+1 and the download of
    # step i-1 run while step i computes (PCIe is full duplex).
    h2d = sum(t.numel() * t.element_size() for d in (Wp, Xp, dYp) for t in d.values())
    sets = [(W, X, dY, step)]
    if args.e2e_steps > 1:
        with torch.cuda.stream(stream):
            W2 = {k: torch.empty_like(v) for k, v in W.items()}
            X2 = {k: torch.empty_like(v) for k, v in X.items()}
            dY2 = {k: torch.empty_like(v) for k, v in dY.items()}
            sets.append((W2, X2, dY2, Step(ls, T, W2, X2, dY2)))
    outs_of = lambda st: [*st.Y.values(), *st.dX.values(), *st.dW.values()]  # noqa: E731
    host_out = [[torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in outs_of(st)] for (_, _, _, st) in sets]
    d2h = sum(t.numel() * t.element_size() for t in outs_of(step))
    s_up, s_down = torch.cuda.Stream(), torch.cuda.Stream()
    barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(s_up)
    done_down = [None] * len(sets)
    for i in range(args.e2e_steps):
        b = i % len(sets)
        Wd, Xd, dYd, st = sets[b]
        if done_down[b] is not None:
            s_up.wait_event(done_down[b])  # set b's previous step is computed and downloaded
        with torch.cuda.stream(s_up):
            for src, dst in ((Wp, Wd), (Xp, Xd), (dYp, dYd)):
                for k in src:
                    dst[k].copy_(src[k], non_blocking=True)
        up = torch.cuda.Event()
        up.record(s_up)
        stream.wait_event(up)
        st.run(stream)
        comp = torch.cuda.Event()
        comp.record(stream)
        s_down.wait_event(comp)
        with torch.cuda.stream(s_down):
            for h, d in zip(host_out[b], outs_of(st)):
                h.copy_(d, non_blocking=True)
        done_down[b] = torch.cuda.Event()
        done_down[b].record(s_down)
    s_down.wait_stream(stream)
    s_down.wait_stream(s_up)
    e1.record(s_down)
    e1.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / max(1, args.e2e_steps), dist, "cuda")
    e2e_value = job_throughput(world, T, e2e_ms)
    sbl.sbl_check(stream)

    # ---- roofline of the dominant call family and of the whole step
    pk = peaks()
    fwd_ops, dx_flops, dw_flops = algorithmic_work(ls, T)
    work = {"forward_i8": (fwd_ops, pk["bf16_sust"] * NOMINAL_I8_OVER_BF16),
            "backward_dx_bf16": (dx_flops, pk["bf16_sust"]),
            "backward_dw_bf16": (dw_flops, pk["bf16_sust"])}
    dom = max(work, key=lambda k: per_call.get(k, 0.0))
    flops, peak_tf = work[dom]
    n_launch = launches[dom]
    achieved_tf = (flops / n_launch) / ((per_call[dom] / n_launch) / 1e3) / 1e12
    roofline = {"bound": "tensor", "kernel": dom, "achieved": achieved_tf, "peak": peak_tf, "unit": "TFLOP/s",
                "frac": achieved_tf / peak_tf, "traffic": traffic_for(dom),
                "peak_source": f"{pk['src']} bf16 sustained" + (" x2 nominal int8/bf16" if dom == "forward_i8"
                                                                 else ""),
                "per_launch_work": flops / n_launch, "launches_per_step": n_launch,
                "note": "achieved = dense-equivalent algorithmic ops of the 7 projections / summed CUDA-event "
                        "time of those launches in the timed region"}
    t_roof = fwd_ops / (pk["bf16_sust"] * NOMINAL_I8_OVER_BF16 * 1e12) + (dx_flops + dw_flops) / (
        pk["bf16_sust"] * 1e12)
    step_roofline = {"roofline_ms": t_roof * 1e3, "measured_ms": ms_per_step, "frac": t_roof * 1e3 / ms_per_step,
                     "basis": "dense-equivalent int8 fwd + bf16 dX, dW on measured sustained peaks"}

    cpu = None
    if rank == 0 and not args.no_cpu_baseline:
        step_s, cores, sample, spent = oracle_sample(ls, T)
        cpu = {"value": T / step_s, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": sample,
               "cpu_seconds_spent": spent}

    if rank == 0:
        print(json.dumps({
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "i8 fwd / bf16 bwd (fp32 accumulate)", "data": "synthetic",
            "config": config, "roofline": roofline, "step_roofline": step_roofline, "cpu_baseline": cpu,
            "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "ms_per_step": e2e_ms, "steps": args.e2e_steps,
                    "note": "pinned host buffers; uploads, steps and downloads pipelined on three streams"},
            "gpu_launches": step.kernels_per_step * args.steps,
            "per_call_ms_per_step": per_call, "clocks": clk.summary(),
        }))
    if dist is not None:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
