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
SPARSE24 = True  # 2:4 layers use the sparse tensor core (--dense24: the dense int8 product)
METRIC = "Sparse-BitLinear fwd+bwd tokens/s (3B-shape, 6:8)"

NOMINAL_I8_OVER_BF16 = 2.0  # dense int8 / dense bf16 tensor throughput (4.5 / 2.25 PFLOP/s)


def peaks():
    """Roofline denominators: HBM copy GB/s and bf16 TFLOP/s, burst (a kernel
    timed alone, at about the maximum SM clock) and sustained (a seconds-long
    loop under the power cap), with the SM clock each was measured at."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        cl = d.get("clocks_under_load", {})
        return dict(hbm=d["hbm_gbs"], bf16=d["bf16_tflops"],
                    bf16_sust=d.get("bf16_tflops_sustained", d["bf16_tflops"]),
                    burst_mhz=d.get("sm_max_mhz", 1965.0), sust_mhz=cl.get("sm_mhz_median", 1305.0),
                    src="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sust=1400.0, burst_mhz=1965.0, sust_mhz=1300.0, src="fallback")


def measure_int8_peak(reps=10, n=8192):
    """Dense int8 tensor-core reference rate on this GPU: a library int8 GEMM
    (torch._int_mm, int32 output) at n^3, best of `reps`, CUDA events.  None
    if the call is unavailable."""
    try:
        g = torch.Generator(device="cuda")
        g.manual_seed(5)
        a = torch.randint(-127, 128, (n, n), dtype=torch.int8, device="cuda", generator=g)
        b = torch.randint(-127, 128, (n, n), dtype=torch.int8, device="cuda", generator=g)
        for _ in range(3):
            torch._int_mm(a, b)
        torch.cuda.synchronize()
        best = float("inf")
        for _ in range(reps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            torch._int_mm(a, b)
            e1.record()
            e1.synchronize()
            best = min(best, e0.elapsed_time(e1))
        del a, b
        torch.cuda.empty_cache()
        return 2.0 * n ** 3 / (best / 1e3) / 1e12
    except Exception:  # pragma: no cover - library path missing
        return None


def pick_peak(pk, sm_mhz):
    """'burst' or 'sustained': the measured peak whose SM clock is nearest the
    clock the timed region ran at."""
    if sm_mhz is None:
        return "sustained"
    return "burst" if abs(sm_mhz - pk["burst_mhz"]) <= abs(sm_mhz - pk["sust_mhz"]) else "sustained"


# ----------------------------------------------------------------- inputs
def make_weight(ls, i, p, N=None, M=None):
    N = N_KEEP if N is None else N
    M = M_GROUP if M is None else M
    _, dist, _, ties = WORKLOADS[ls.name]
    if dist == "trimodal":
        w = synth.trimodal_weight(p.d_out, p.d_in, seed=0, tensor_id=i)
    else:
        w = synth.normal_weight(p.d_out, p.d_in, seed=0, tensor_id=i)
    if ties > 0 and N < M:
        w = synth.with_boundary_ties(w, N, M, seed=0, tensor_id=300 + i, frac=ties)
    return w


def make_inputs(ls, T, seed, device, with_weights=True):
    """Seeded synthetic tensors for one step, on `device` (CPU pinned or cuda)."""
    W, X, dY = {}, {}, {}
    outl = WORKLOADS[ls.name][2]
    for i, p in enumerate(ls.projections if with_weights else []):
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

    def __init__(self, ls, T, W, X, dY, N=None, M=None, sparse24=None):
        import semi_structured_sparsity_step_b200 as sbl
        from semi_structured_sparsity_step_b200.layer import SparseBitLinearLayer
        N = N_KEEP if N is None else N
        M = M_GROUP if M is None else M
        sparse24 = SPARSE24 if sparse24 is None else sparse24
        self.sbl, self.ls, self.T = sbl, ls, T
        self.W, self.X, self.dY = W, X, dY
        dev = "cuda"
        self.layers = {p.name: SparseBitLinearLayer(W[p.name], N, M, sparse24=sparse24)
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
        self.sparse24 = sparse24 and (N, M) == (2, 4)  # compress + sparse tensor-core forward
        self.kernels_per_step = 2 * n_p + n_x + 3 * n_p + (n_p if self.sparse24 else 0)
        self.train = False
        self.pipelined = False

    def enable_pipelined_weights(self):
        """Compute the weight side (mask, gamma, ternary) of the next step
        during this step's backward products, on the side streams, into a
        second set of W_eff buffers; the step then starts with act_quant
        alone.  The weight side is HBM-bound and the products are bound by
        the tensor cores, so the two overlap.  Valid because W changes only
        in an optimizer step, which the fwd + bwd step does not take (with
        one, sbl_adamw_step computes the next weight side itself)."""
        from semi_structured_sparsity_step_b200.layer import SparseBitLinearLayer
        L0 = next(iter(self.layers.values()))
        self.layers_next = {p.name: SparseBitLinearLayer(self.W[p.name], L0.N, L0.M, sparse24=self.sparse24)
                            for p in self.ls.projections}
        self.pipelined = True
        self.primed = False

    def enable_training(self, lr=1e-5, betas=(0.9, 0.95), eps=1e-5, weight_decay=0.1, max_norm=1.0):
        """Make every step a full data-parallel training step: the dW of the
        projections live in one GradBucket, each is summed over the ranks as
        soon as it is written (NCCL, overlapping the remaining products), and
        the step ends with the global clip norm (sbl_grad_sqnorm) and one
        sbl_adamw_step per projection, which also computes the next step's
        gamma, mask and W_eff.  From the second step on, the weight side at
        the start of the step is therefore skipped (Algorithm 1 steps (2)-(8),
        with (8) fused with the next step's (2), (4), (5))."""
        from semi_structured_sparsity_step_b200.data_parallel import GradBucket, GradExchange
        from semi_structured_sparsity_step_b200.layer import SparseBitLinearLayer
        ls = self.ls
        self.grads = GradBucket({p.name: (p.d_out, p.d_in) for p in ls.projections}, "cuda")
        self.dW = dict(self.grads.views)
        self.exchange = GradExchange(self.grads)
        for p in ls.projections:     # the optimizer reads and updates the old mask (flip count)
            L = self.layers[p.name]
            if L.mask_bits is None:
                L.mask_bits = torch.empty(p.d_out, p.d_in // 8, dtype=torch.uint8, device="cuda")
        self.m = {p.name: torch.zeros(p.d_out, p.d_in, dtype=torch.float32, device="cuda") for p in ls.projections}
        self.v = {p.name: torch.zeros(p.d_out, p.d_in, dtype=torch.float32, device="cuda") for p in ls.projections}
        self.sumsq = torch.zeros(1, dtype=torch.float64, device="cuda")
        self.flips = torch.zeros(1, dtype=torch.int64, device="cuda")
        self.hp = dict(lr=lr, betas=betas, eps=eps, weight_decay=weight_decay, max_norm=max_norm)
        self.t = 0
        self.weights_ready = False
        self.train = True
        n_p = len(ls.projections)
        self.kernels_per_step = len(ls.inputs) + 3 * n_p + n_p + 2 * n_p  # act quant, products, sqnorm, adamw

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
            if not (self.train and self.weights_ready):
                for i, p in enumerate(ls.projections):
                    self.layers[p.name].weight_step(self.side[i % len(self.side)])
            for n, d in ls.inputs.items():
                sbl.sbl_act_quant(self.X[n], T, d, self.Xq[n], self.amax[n], stream)
            for sd in self.side:
                join = torch.cuda.Event()
                join.record(sd)
                stream.wait_event(join)

        def act_quant_only():
            for n, d in ls.inputs.items():
                sbl.sbl_act_quant(self.X[n], T, d, self.Xq[n], self.amax[n], stream)

        if self.pipelined:
            if not self.primed:  # the first step computes its own weight side
                weight_and_act_quant()
                self.primed = True
            else:
                timed("act_quant", act_quant_only)
        else:
            timed("weight_and_act_quant", weight_and_act_quant)
        for p in ls.projections:
            L = self.layers[p.name]
            timed("forward_i8", lambda p=p, L=L: L.forward(self.Xq[p.input_name], self.amax[p.input_name],
                                                           self.Y[p.name], stream=stream))
        if self.pipelined:
            # the next step's weight side, overlapped with the backward products
            fork = torch.cuda.Event()
            fork.record(stream)
            for sd in self.side:
                sd.wait_event(fork)
            by_size = sorted(ls.projections, key=lambda p: -p.d_out * p.d_in)
            for i, p in enumerate(by_size):
                self.layers_next[p.name].weight_step(self.side[i % len(self.side)])
        for p in ls.projections:
            L = self.layers[p.name]
            timed("backward_dx_bf16", lambda p=p, L=L: L.backward(self.dY[p.name], self.X[p.input_name],
                                                                  self.dX[p.name], None, stream=stream))
            timed("backward_dw_bf16", lambda p=p, L=L: L.backward(self.dY[p.name], self.X[p.input_name],
                                                                  None, self.dW[p.name], stream=stream))
            if self.train:
                with torch.cuda.stream(stream):
                    self.exchange.launch(p.name)
        if self.train:
            timed("optimizer", lambda: self._optimizer(stream))
        if self.pipelined:
            for sd in self.side:
                join = torch.cuda.Event()
                join.record(sd)
                stream.wait_event(join)
            self.layers, self.layers_next = self.layers_next, self.layers

    def _optimizer(self, stream):
        """Wait for the dW exchange, then the global clip norm and AdamW with
        the next step's weight side, per projection on the side streams
        (largest first)."""
        sbl, ls, hp = self.sbl, self.ls, self.hp
        with torch.cuda.stream(stream):
            self.exchange.wait()
            self.sumsq.zero_()
        for p in ls.projections:
            L = self.layers[p.name]
            sbl.sbl_grad_sqnorm(self.dW[p.name], p.d_out * p.d_in, self.sumsq, L.ws, L.ws_bytes, stream)
        self.t += 1
        fork = torch.cuda.Event()
        fork.record(stream)
        for sd in self.side:
            sd.wait_event(fork)
        by_size = sorted(ls.projections, key=lambda p: -p.d_out * p.d_in)
        for i, p in enumerate(by_size):
            L = self.layers[p.name]
            sbl.sbl_adamw_step(L.W, None, self.dW[p.name], self.m[p.name], self.v[p.name], p.d_out, p.d_in, L.N,
                               L.M, hp["lr"], hp["betas"][0], hp["betas"][1], hp["eps"], hp["weight_decay"], self.t,
                               self.sumsq, hp["max_norm"], L.W_eff, L.W_eff_bf16, L.mask_bits, L.gamma, self.flips,
                               L.ws, L.ws_bytes, self.side[i % len(self.side)])
        for sd in self.side:
            join = torch.cuda.Event()
            join.record(sd)
            stream.wait_event(join)
        self.weights_ready = True


def algorithmic_work(ls, T):
    P = ls.params
    fwd_ops = 2.0 * T * P          # dense-equivalent int8 ops
    dx_flops = 2.0 * T * P
    dw_flops = 2.0 * T * P
    return fwd_ops, dx_flops, dw_flops


# ----------------------------------------------------------------- clocks
class ClockSampler:
    """SM clock and clock-event reasons of one GPU, sampled every `period_s`
    while the context is open: NVML (read-only queries) from a thread, or
    `nvidia-smi -lms` when NVML is not importable.  The GPU is found by its
    PCI address, so the sample is the CUDA device's even under
    CUDA_VISIBLE_DEVICES."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40), ("sw_thermal_slowdown", 0x20),
               ("sw_power_cap", 0x4))

    def __init__(self, cuda_index, period_s=0.02):
        self.cuda_index = cuda_index
        self.period = period_s
        self.samples = []          # (sm_mhz, reason bits)
        self.sm_max = None
        self.proc = None
        self.thread = None
        self.stop = threading.Event()
        self.how = None

    def _nvml_handle(self):
        import pynvml
        pynvml.nvmlInit()
        try:
            pr = torch.cuda.get_device_properties(self.cuda_index)
            bus = f"{pr.pci_domain_id:08x}:{pr.pci_bus_id:02x}:{pr.pci_device_id:02x}.0"
            return pynvml, pynvml.nvmlDeviceGetHandleByPciBusId(bus)
        except Exception:
            return pynvml, pynvml.nvmlDeviceGetHandleByIndex(self.cuda_index)

    def __enter__(self):
        try:
            nv, h = self._nvml_handle()
            self.sm_max = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
            get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons",
                                  getattr(nv, "nvmlDeviceGetCurrentClocksThrottleReasons", None))

            def loop():
                while not self.stop.is_set():
                    try:
                        self.samples.append((float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)),
                                             int(get_reasons(h))))
                    except Exception:
                        pass
                    self.stop.wait(self.period)
            self.how = f"nvml every {self.period * 1e3:.0f} ms"
            self.thread = threading.Thread(target=loop, daemon=True)
            self.thread.start()
            return self
        except Exception:
            pass
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.cuda_index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", str(max(20, int(self.period * 1e3)))],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read_smi, daemon=True)
            self.thread.start()
            self.how = "nvidia-smi -lms"
        except (OSError, ValueError):
            self.proc = None
        return self

    def _read_smi(self):
        for ln in self.proc.stdout:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm = float(f[1])
                self.sm_max = float(f[2])
            except ValueError:
                continue
            bits = 0
            for (nm, bit), v in zip(self.REASONS, f[5:9]):
                if v.lower().startswith("active"):
                    bits |= bit
            self.samples.append((sm, bits))

    def __exit__(self, *exc):
        self.stop.set()
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        if self.thread is not None:
            self.thread.join(timeout=5)

    def summary(self):
        sm = [a for a, _ in self.samples]
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": self.sm_max, "reasons": [], "samples": 0, "how": self.how}
        reasons = sorted({nm for _, bits in self.samples for nm, bit in self.REASONS if bits & bit})
        return {"sm_mhz": statistics.median(sm), "sm_min_mhz": min(sm), "sm_max_mhz": self.sm_max,
                "reasons": reasons, "samples": len(sm), "how": self.how}


# ----------------------------------------------------------------- CPU oracle timing
def oracle_steps(ls, T_full, steps, warmup, tokens=4, N=None, M=None):
    """Time the oracle as it stands, on the host, over `warmup` + `steps`
    bounded sample steps of the workload.  One sample step is the whole path
    for `tokens` tokens with the full step's mix of work per token:

      weight side  mask, gamma and ternary (oracle.effective_weight) on a row
                   slice of the q projection holding the step's share of the
                   weights, params * tokens / T_full;
      token side   act quant of every input, then for every projection the
                   int32 product and output scaling, dX and dW, on `tokens`
                   fresh tokens.

    W_eff of every full projection (needed by the token side) is computed
    once before the steps and not timed.  Returns (seconds per step, tokens
    per step, threads, description)."""
    import oracle
    N = N_KEEP if N is None else N
    M = M_GROUP if M is None else M
    weffs = {}
    for i, p in enumerate(ls.projections):
        weffs[p.name] = oracle.effective_weight(synth.bits(make_weight(ls, i, p, N, M)), N, M)
    q = ls.projections[0]
    wq = synth.bits(make_weight(ls, 0, q, N, M))
    rows = max(1, min(q.d_out, round(ls.params * tokens / T_full / q.d_in)))
    outl = WORKLOADS[ls.name][2]
    times = []
    for s in range(warmup + steps):
        xs = {n: synth.bits(synth.activations(tokens, d, seed=1000 + s, tensor_id=100 + j, outlier_frac=outl))
              for j, (n, d) in enumerate(ls.inputs.items())}
        dys = {p.name: synth.bits(synth.grad_output(tokens, p.d_out, seed=1000 + s, tensor_id=200 + i))
               for i, p in enumerate(ls.projections)}
        r0 = (s * rows) % max(1, q.d_out - rows + 1)
        t0 = time.perf_counter()
        oracle.effective_weight(wq[r0:r0 + rows], N, M)
        q8 = {n: oracle.act_quant(xs[n]) for n in ls.inputs}
        for p in ls.projections:
            weff, gamma, _ = weffs[p.name]
            xq, amax = q8[p.input_name]
            oracle.forward_out(oracle.forward_acc(xq, weff), gamma, amax)
            oracle.backward_dx(dys[p.name], weff, gamma)
            oracle.backward_dw(dys[p.name], xs[p.input_name])
        dt = time.perf_counter() - t0
        if s >= warmup:
            times.append(dt)
    try:
        from threadpoolctl import threadpool_info
        blas = max([1] + [d.get("num_threads", 1) for d in threadpool_info()])
    except Exception:  # pragma: no cover
        blas = 1
    sample = (f"{steps} timed sample steps after {warmup} untimed; each: all {len(ls.projections)} projections "
              f"on {tokens} fresh tokens (act quant, int32 product + scaling, dX, dW) + the weight side on "
              f"{rows} rows of {q.name} ({rows * q.d_in} weights = the step's share, params x {tokens}/{T_full}); "
              f"W_eff of the full projections computed once beforehand, untimed")
    return statistics.mean(times), tokens, blas, sample


def cpu_threads_note(blas):
    return {"blas_threads": blas, "nproc": os.cpu_count(),
            "note": "fp64 products on BLAS threads; the int64 products, mask and quantisers run single-threaded "
                    "numpy"}


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
    del packs, dense
    torch.cuda.empty_cache()
    return {"metric": "Sparse-BitLinear packed decode GEMV, HBM bytes/s", "unit": "GB/s",
            "workload": f"{layers} distinct qwen2.5-3b layer sets, packed {N_KEEP}:{M_GROUP} "
                        f"({'2.5 bit/weight' if (N_KEEP, M_GROUP) == (6, 8) else 'packed'}), "
                        f"batch 1/8/16, one grouped GEMV launch per layer (7 projections), CUDA graph per pass",
            "gemv_kernel": ["dense layout: per-warp TMA rings filled before the dependency wait, activations staged in shared memory; "
                            "N:M format: per-warp TMA rings in persistent blocks", "block-wide TMA ring",
                            "per-warp TMA rings in persistent blocks"][args.gemv_variant],
            "peak_hbm_gbs": pkk["hbm"], "peak_source": pkk["src"], "results": results,
            "dense2": {"layout": "dense 2-bit codes of the same weights (2.0 bit/weight, no index plane)",
                       "results": results_d2}}


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
    # burst: each pass is timed on its own
    if getattr(args, "int8_peak", None):
        i8_peak, i8_src = args.int8_peak, "measured here: library int8 GEMM 8192^3, best of 10 (burst)"
    else:
        i8_peak = pk_peak["bf16"] * NOMINAL_I8_OVER_BF16
        i8_src = f"{pk_peak['src']} bf16 burst x2 nominal int8/bf16"
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
    del layers, unpacked
    torch.cuda.empty_cache()
    return {"metric": "Sparse-BitLinear prefill forward on the packed 6:8 format (3B layer set)",
            "unit": "tokens/s", "peak_int8_tops": i8_peak, "peak_source": i8_src,
            "workload": "qwen2.5-3b layer set, 6:8 packed (2.5 bit/weight), T = 512 / 8192 / 32768, "
                        "Xq from absmax-quantised N(0,1), fp32 outputs",
            "results": results}


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


# ----------------------------------------------------------------- other configurations
def step_roofline_ms(ls, T, pk, which, i8_peak):
    """Dense roofline time (ms) of one training step: int8 forward + bf16 dX
    and dW at the chosen peak ('burst' or 'sustained')."""
    fwd, dx, dw = algorithmic_work(ls, T)
    bf = pk["bf16"] if which == "burst" else pk["bf16_sust"]
    i8 = i8_peak * (1.0 if which == "burst" else pk["bf16_sust"] / pk["bf16"])
    return (fwd / (i8 * 1e12) + (dx + dw) / (bf * 1e12)) * 1e3


def train_point(ls, T, N, M, sparse24, steps, warmup, X=None, dY=None, pk=None, i8_peak=None):
    """One training-step configuration, inputs resident: `warmup` untimed
    steps, then `steps` steps timed with CUDA events on the launching stream,
    SM clocks sampled meanwhile.  Returns ms per step, tokens/s, per-family
    ms and the step's roofline fraction."""
    W = {p.name: make_weight(ls, i, p, N, M).cuda() for i, p in enumerate(ls.projections)}
    if X is None:
        _, X, dY = make_inputs(ls, T, seed=0, device="cuda", with_weights=False)
    stream = torch.cuda.Stream()
    st = Step(ls, T, W, X, dY, N, M, sparse24)
    st.enable_pipelined_weights()
    for _ in range(warmup):
        st.run(stream)
    stream.synchronize()
    ev = {}
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(torch.cuda.current_device()) as clk:
        e0.record(stream)
        for _ in range(steps):
            st.run(stream, ev)
        e1.record(stream)
        stream.synchronize()
    st.sbl.sbl_check(stream)
    ms = e0.elapsed_time(e1) / steps
    cl = clk.summary()
    out = {"N:M": f"{N}:{M}", "sparse24_forward": bool(st.sparse24), "tokens": T, "ms_per_step": ms,
           "tokens_per_s": T / (ms / 1e3),
           "per_call_ms_per_step": {k: sum(a.elapsed_time(b) for a, b in v) / steps for k, v in ev.items()},
           "clocks": cl}
    if pk is not None and i8_peak:
        which = pick_peak(pk, cl["sm_mhz"])
        out["step_roofline"] = {"peak": which, "roofline_ms": step_roofline_ms(ls, T, pk, which, i8_peak),
                                "frac": step_roofline_ms(ls, T, pk, which, i8_peak) / ms}
    del st, W
    return out


def run_extras(pk, i8_peak, steps=10, warmup=3):
    """The other configurations of the benchmark, each timed on its own with
    CUDA events and its own clock record: decode GEMV on the packed 3B stack,
    prefill on the packed 3B set, the N:M sweep on the 3B up projection at
    8192 tokens, and the 0.5B layer set at 4096 tokens."""
    import types
    extras = {}
    t_all = time.perf_counter()
    ns = types.SimpleNamespace(steps=steps, warmup=warmup, layers=36, gemv_variant=0, int8_peak=i8_peak)

    def guarded(name, fn):
        t0 = time.perf_counter()
        try:
            with ClockSampler(torch.cuda.current_device()) as clk:
                r = fn()
            if isinstance(r, dict) and "clocks" not in r:
                r["clocks"] = clk.summary()
        except Exception as e:  # pragma: no cover - reported, the headline stands
            r = {"error": f"{type(e).__name__}: {e}"}
        r["wall_s"] = time.perf_counter() - t0
        extras[name] = r
        torch.cuda.empty_cache()

    guarded("decode", lambda: run_decode(ns))
    guarded("prefill", lambda: run_prefill(ns))

    def sweep():
        ls = synth.layer_set("qwen2.5-3b-up")
        T = WORKLOADS["qwen2.5-3b-up"][0]
        _, X, dY = make_inputs(ls, T, seed=0, device="cuda", with_weights=False)
        pts = [train_point(ls, T, n, m, sp, steps, warmup, X, dY, pk, i8_peak)
               for n, m, sp in ((8, 8, False), (6, 8, False), (4, 8, False), (2, 8, False), (2, 4, False),
                                (2, 4, True))]
        return {"workload": "qwen2.5-3b up projection 11008x2048, 8192 tokens, trimodal W with 1% boundary-tie "
                            "groups, X ~ N(0,1) with 0.1% outlier channels x10, fwd+bwd",
                "points": pts}

    guarded("nm_sweep", sweep)

    def q05():
        ls = synth.layer_set("qwen2.5-0.5b")
        r = train_point(ls, 4096, 6, 8, False, steps, warmup, pk=pk, i8_peak=i8_peak)
        r["workload"] = "qwen2.5-0.5b layer set, 4096 tokens (8 x 512), 6:8, W ~ N(0, 0.02), fwd+bwd"
        return r

    guarded("qwen05b", q05)
    extras["wall_s_total"] = time.perf_counter() - t_all
    return extras


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
                    help="decode kernel: 0 default, 1 block-wide TMA ring, 2 per-warp TMA rings in persistent blocks")
    ap.add_argument("--nm", default="6:8", help="N:M of the mask (the sweep: 8:8, 6:8, 4:8, 2:8, 2:4)")
    ap.add_argument("--sparse24", action="store_true",
                    help="2:4: forward on the sparse tensor core (the default; kept for explicit commands)")
    ap.add_argument("--dense24", action="store_true", help="2:4: forward through the dense int8 product instead")
    ap.add_argument("--settle-s", type=float, default=2.0,
                    help="untimed steps after the warm-up until this many seconds have passed")
    ap.add_argument("--serial-weights", action="store_true",
                    help="run each step's weight side before its forward instead of during the previous backward")
    ap.add_argument("--dp-train", action="store_true",
                    help="full data-parallel training step: dW summed over ranks (NCCL), clip norm, AdamW")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the decode / prefill / N:M sweep / 0.5B keys of the default line")
    args = ap.parse_args()
    global N_KEEP, M_GROUP, SPARSE24
    N_KEEP, M_GROUP = (int(v) for v in args.nm.split(":"))
    SPARSE24 = not args.dense24
    if args.mode == "decode":
        print(json.dumps(run_decode(args)))
        return
    if args.mode == "prefill":
        args.int8_peak = measure_int8_peak()
        print(json.dumps(run_prefill(args)))
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
              "weight_side": "computed during the previous step's backward (pipelined)",
              "forward_kernel": ("2:4 compress + sparse int8 MMA (tcgen05.mma.sp)"
                                 if SPARSE24 and (N_KEEP, M_GROUP) == (2, 4)
                                 else "dense int8 MMA (tcgen05.mma kind::i8)")}

    if args.serial_weights:
        config["weight_side"] = "before the step's forward (overlapped with act_quant)"
    if args.dp_train:
        config["weight_side"] = "fused into the optimizer step (sbl_adamw_step) of the previous step"
        config["parallelism"] = f"dp{args.gpus}: dW summed over ranks (NCCL all-reduce), then clip norm and AdamW"
        config["step"] = ("act quant, int8 forward, bf16 dX and dW, dW all-reduce per projection overlapping the "
                          "remaining products, sbl_grad_sqnorm, sbl_adamw_step with the next step's weight side")
    metric = METRIC if not args.dp_train else \
        "Sparse-BitLinear data-parallel training step tokens/s (fwd+bwd+dW all-reduce+AdamW, 3B-shape, 6:8)"

    if args.impl == "reference":
        if rank != 0:
            return
        step_s, tok, blas, sample = oracle_steps(ls, T, args.steps, args.warmup)
        v = tok / step_s
        print(json.dumps({
            "impl": "reference", "metric": metric, "value": v, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_s * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "i8/bf16 (oracle: fp32/fp64/int64 on CPU)",
            "data": "synthetic", "config": config, "extrapolated": False, "sample_tokens_per_step": tok,
            "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": blas, "kind": "oracle", "sample": sample,
                             **cpu_threads_note(blas)},
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
    pk = peaks()
    i8_peak = measure_int8_peak() if world == 1 else None
    i8_src = ("measured here: library int8 GEMM 8192^3, best of 10 (burst)" if i8_peak else
              f"{pk['src']} bf16 burst x2 nominal int8/bf16")
    if not i8_peak:
        i8_peak = pk["bf16"] * NOMINAL_I8_OVER_BF16

    stream = torch.cuda.Stream()
    Wp, Xp, dYp = make_inputs(ls, T, seed=rank, device="pinned")
    with torch.cuda.stream(stream):
        W = {k: v.to("cuda", non_blocking=True) for k, v in Wp.items()}
        X = {k: v.to("cuda", non_blocking=True) for k, v in Xp.items()}
        dY = {k: v.to("cuda", non_blocking=True) for k, v in dYp.items()}
        step = Step(ls, T, W, X, dY)
        if args.dp_train:
            step.enable_training()
        elif not args.serial_weights:
            step.enable_pipelined_weights()
    stream.synchronize()

    def barrier():
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()

    # W warm-up steps, then more untimed steps until `settle_s` seconds have
    # passed, so the SM clock has settled under the power cap before timing.
    # Every rank takes the same number of steps (rank 0 decides).
    t_w = time.perf_counter()
    for _ in range(args.warmup):
        step.run(stream)
    stream.synchronize()
    t_p = time.perf_counter()
    for _ in range(2):               # the per-step time once warm (the first steps carry one-time set-up)
        step.run(stream)
    stream.synchronize()
    per = (time.perf_counter() - t_p) / 2
    extra = max(0, int((args.settle_s - (time.perf_counter() - t_w)) / max(per, 1e-4)) + 1) \
        if args.settle_s > 0 else 0
    if dist is not None:
        t = torch.tensor([extra], dtype=torch.int64, device="cuda")
        dist.broadcast(t, 0)
        extra = int(t.item())
    for _ in range(extra):
        step.run(stream)
    sbl.sbl_check(stream)
    settle_s = time.perf_counter() - t_w

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
    clocks = clk.summary()

    per_call = {k: sum(a.elapsed_time(b) for a, b in v) / args.steps for k, v in ev.items()}
    launches = {k: len(v) // args.steps for k, v in ev.items()}
    kernels_per_step = step.kernels_per_step

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
            st2 = Step(ls, T, W2, X2, dY2)
            if args.dp_train:
                st2.enable_training()
            elif not args.serial_weights:
                st2.enable_pipelined_weights()
            sets.append((W2, X2, dY2, st2))
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

    # ---- roofline of the dominant call family and of the whole step, against
    # the burst and the sustained measured peaks; the headline takes the one
    # measured at the SM clock nearest the timed region's median clock.
    which = pick_peak(pk, clocks["sm_mhz"])
    fwd_ops, dx_flops, dw_flops = algorithmic_work(ls, T)
    i8_sust = i8_peak * pk["bf16_sust"] / pk["bf16"]
    work = {"forward_i8": (fwd_ops, i8_peak, i8_sust),
            "backward_dx_bf16": (dx_flops, pk["bf16"], pk["bf16_sust"]),
            "backward_dw_bf16": (dw_flops, pk["bf16"], pk["bf16_sust"])}
    dom = max(work, key=lambda k: per_call.get(k, 0.0))
    fams = {}
    for k, (flops, pb, ps) in work.items():
        if k not in per_call:
            continue
        n_l = launches[k]
        ach = (flops / n_l) / ((per_call[k] / n_l) / 1e3) / 1e12
        fams[k] = {"achieved": ach, "frac_burst": ach / pb, "frac_sustained": ach / ps, "launches": n_l,
                   "ms_per_step": per_call[k]}
    flops, p_burst, p_sust = work[dom]
    peak_tf = p_burst if which == "burst" else p_sust
    achieved_tf = fams[dom]["achieved"]
    roofline = {"bound": "tensor", "kernel": dom, "achieved": achieved_tf, "peak": peak_tf, "unit": "TFLOP/s",
                "frac": achieved_tf / peak_tf, "frac_burst": achieved_tf / p_burst,
                "frac_sustained": achieved_tf / p_sust, "peak_used": which,
                "traffic": traffic_for(dom),
                "peak_source": (f"{pk['src']} bf16 {which} (burst {pk['bf16']} at {pk['burst_mhz']:.0f} MHz, "
                                f"sustained {pk['bf16_sust']} at {pk['sust_mhz']:.0f} MHz); chosen by the nearest "
                                f"SM clock to the timed region's median {clocks['sm_mhz']} MHz"),
                "int8_peak_measured": i8_peak, "int8_peak_source": i8_src,
                "per_launch_work": flops / launches[dom], "launches_per_step": launches[dom],
                "families": fams,
                "note": "achieved = dense-equivalent algorithmic ops of the 7 projections / summed CUDA-event "
                        "time of those launches in the timed region; int8 sustained = int8 burst x bf16 "
                        "sustained/burst"}
    t_b = step_roofline_ms(ls, T, pk, "burst", i8_peak)
    t_s = step_roofline_ms(ls, T, pk, "sustained", i8_peak)
    step_roofline = {"roofline_ms": t_b if which == "burst" else t_s, "measured_ms": ms_per_step,
                     "frac": (t_b if which == "burst" else t_s) / ms_per_step, "peak_used": which,
                     "frac_burst": t_b / ms_per_step, "frac_sustained": t_s / ms_per_step,
                     "roofline_ms_burst": t_b, "roofline_ms_sustained": t_s,
                     "basis": "dense-equivalent int8 fwd (measured int8 peak) + bf16 dX, dW (measured bf16 peaks)"}

    cpu = None
    if rank == 0 and not args.no_cpu_baseline:
        step_s, tok, blas, sample = oracle_steps(ls, T, 3, 1)
        cpu = {"value": tok / step_s, "unit": "tokens/s", "cores": blas, "kind": "oracle", "sample": sample,
               **cpu_threads_note(blas)}

    extras = None
    if rank == 0 and world == 1 and not args.no_extras and not args.dp_train and args.workload == "qwen2.5-3b":
        del sets, host_out, step, W, X, dY
        torch.cuda.empty_cache()
        extras = run_extras(pk, i8_peak)

    if rank == 0:
        line = {
            "metric": metric, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "i8 fwd / bf16 bwd (fp32 accumulate)", "data": "synthetic",
            "config": dict(config, settle_s=settle_s, settle_steps=args.warmup + 2 + extra),
            "roofline": roofline, "step_roofline": step_roofline, "cpu_baseline": cpu,
            "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "ms_per_step": e2e_ms, "steps": args.e2e_steps,
                    "note": "pinned host buffers; uploads, steps and downloads pipelined on three streams"},
            "gpu_launches": kernels_per_step * args.steps,
            "per_call_ms_per_step": per_call, "clocks": clocks,
        }
        if extras is not None:
            line["extra_keys"] = sorted(k for k in extras if k != "wall_s_total")
            line.update(extras)
        print(json.dumps(line))
    if dist is not None:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
