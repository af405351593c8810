"""GPU parity of the optimizer step (sbl_adamw_step, sbl_grad_sqnorm) against
the oracle, through the C ABI.

Sparse-BitNet summary, Algorithm 1 step (8) (AdamW on the master weight,
grad clip 1.0) followed by the next step's (2), (4), (5), and the mask flip
rate of Fig. 3b.  Every element is updated with the same IEEE fp32
operations in the same order on both sides, so the new W (bf16 bits), the
fp32 master copy and both moments must be bit-equal; the next step's W_eff,
gamma and mask are bit-exact functions of the new W; the flip count is an
exact integer.  The squared gradient norm is an fp64 sum in another order
than the oracle's correctly rounded one: relative 1e-12.  The clip factor is
rounded to fp32 from it on both sides (and the tests check it came out the
same).
"""
import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu

HP = dict(beta1=0.9, beta2=0.95, eps=1e-5, weight_decay=0.1)


def _unpack_mask(bits: np.ndarray) -> np.ndarray:
    return np.unpackbits(bits, axis=1, bitorder="little").astype(bool)


def _u32(t: torch.Tensor) -> np.ndarray:
    return t.cpu().numpy().view(np.uint32)


class Opt:
    """Device buffers of one weight with its optimizer state."""

    def __init__(self, lib, w_bf16, N, M, master32=False):
        self.lib, self.N, self.M = lib, N, M
        self.d_out, self.d_in = w_bf16.shape
        self.W = w_bf16.cuda()
        self.W32 = w_bf16.float().cuda() if master32 else None
        self.m = torch.zeros(self.d_out, self.d_in, dtype=torch.float32, device="cuda")
        self.v = torch.zeros_like(self.m)
        self.weff = torch.empty(self.d_out, self.d_in, dtype=torch.int8, device="cuda")
        self.weff16 = torch.empty(self.d_out, self.d_in, dtype=torch.bfloat16, device="cuda")
        self.bits = torch.empty(self.d_out, self.d_in // 8, dtype=torch.uint8, device="cuda")
        self.gamma = torch.empty(1, dtype=torch.float32, device="cuda")
        self.flips = torch.zeros(1, dtype=torch.int64, device="cuda")
        self.ws_bytes = lib.sbl_mask_quant_workspace_bytes(self.d_out, self.d_in)
        self.ws = torch.empty(self.ws_bytes, dtype=torch.uint8, device="cuda")
        lib.sbl_mask_quant(self.W, self.d_out, self.d_in, N, M, self.weff, self.weff16, self.bits, self.gamma,
                           self.ws, self.ws_bytes)

    def step(self, dW, lr, t, sumsq=None, max_norm=1.0, count_flips=True):
        self.lib.sbl_adamw_step(self.W, self.W32, dW, self.m, self.v, self.d_out, self.d_in, self.N, self.M, lr,
                                HP["beta1"], HP["beta2"], HP["eps"], HP["weight_decay"], t, sumsq, max_norm,
                                self.weff, self.weff16, self.bits, self.gamma,
                                self.flips if count_flips else None, self.ws, self.ws_bytes)
        self.lib.sbl_check()


def _check_against(o: Opt, ref: dict, flips_before: int = 0):
    assert np.array_equal(synth.bits(o.W.cpu()), ref["w_bits"]), "new W"
    if ref["w32"] is not None:
        assert np.array_equal(_u32(o.W32), ref["w32"].view(np.uint32)), "fp32 master"
    assert np.array_equal(_u32(o.m), ref["m"].view(np.uint32)), "first moment"
    assert np.array_equal(_u32(o.v), ref["v"].view(np.uint32)), "second moment"
    assert o.gamma.item() == float(ref["gamma"])
    assert np.array_equal(o.weff.cpu().numpy(), ref["weff"])
    assert np.array_equal(synth.bits(o.weff16.cpu()), oracle.f32_to_bf16(ref["weff"].astype(np.float32)))
    assert np.array_equal(_unpack_mask(o.bits.cpu().numpy()), ref["keep"])
    assert int(o.flips.item()) - flips_before == ref["flips"]


@pytest.mark.parametrize("master32", [False, True])
@pytest.mark.parametrize("N,M", [(6, 8), (2, 4)])
@pytest.mark.parametrize("clip", [False, True])
def test_adamw_step_matches_oracle(lib, master32, N, M, clip):
    """Three consecutive steps (t = 1, 2, 3) on a ragged shape (8400 groups of
    8 weights: 33 blocks, the last partly filled), with and without clipping,
    bf16 or fp32 master; each step's mask is the next step's old mask."""
    d_out, d_in = 200, 336
    w = synth.trimodal_weight(d_out, d_in, seed=61)
    o = Opt(lib, w, N, M, master32)
    wb = synth.bits(w)
    w32 = w.float().numpy() if master32 else None
    m = np.zeros((d_out, d_in), np.float32)
    v = np.zeros_like(m)
    lr = 1e-3
    sumsq = torch.zeros(1, dtype=torch.float64, device="cuda")
    for t in (1, 2, 3):
        dw = synth.optimizer_state(d_out, d_in, seed=70 + t)[0]
        dW = dw.cuda()
        c = np.float32(1.0)
        if clip:
            sumsq.zero_()
            lib.sbl_grad_sqnorm(dW, dW.numel(), sumsq, o.ws, o.ws_bytes)
            S = oracle.grad_sqnorm(dw.numpy())
            assert sumsq.item() == pytest.approx(S, rel=1e-12)
            c = oracle.grad_clip_scale(S, 0.1)
            assert c < 1.0
            assert oracle.grad_clip_scale(sumsq.item(), 0.1) == c
        before = int(o.flips.item())
        o.step(dW, lr, t, sumsq if clip else None, 0.1)
        ref = oracle.adamw_weight_step(wb, dw.numpy(), m, v, N, M,
                                       oracle.adamw_scalars(lr, step=t, **HP), c, w32)
        _check_against(o, ref, before)
        assert ref["flips"] > 0
        wb, m, v, w32 = ref["w_bits"], ref["m"], ref["v"], ref["w32"]


@pytest.mark.parametrize("t", [1, 1000])
def test_adamw_step_from_state(lib, t):
    """From non-zero moments (the synthetic optimizer state) at an early and a
    late step, on a shape of 2M weights (the grid-stride loop runs several
    times per thread)."""
    d_out, d_in = 1024, 2048
    w = synth.normal_weight(d_out, d_in, seed=62)
    dw, m0, v0 = synth.optimizer_state(d_out, d_in, seed=62)
    o = Opt(lib, w, 6, 8)
    o.m.copy_(m0)
    o.v.copy_(v0)
    o.step(dw.cuda(), 2e-3, t)
    ref = oracle.adamw_weight_step(synth.bits(w), dw.numpy(), m0.numpy(), v0.numpy(), 6, 8,
                                   oracle.adamw_scalars(2e-3, step=t, **HP))
    _check_against(o, ref)


def test_adamw_zero_lr_is_identity(lib):
    """lr = 0 leaves W bit for bit and flips nothing; the moments still move."""
    d_out, d_in = 64, 128
    w = synth.normal_weight(d_out, d_in, seed=63)
    o = Opt(lib, w, 6, 8)
    bits0 = o.bits.clone()
    o.step(synth.optimizer_state(d_out, d_in, seed=63)[0].cuda(), 0.0, 5)
    assert torch.equal(o.W, w.cuda())
    assert torch.equal(o.bits, bits0)
    assert int(o.flips.item()) == 0
    assert o.m.abs().max().item() > 0


def test_adamw_without_flip_counter(lib):
    """flips = NULL skips the count and changes nothing else."""
    d_out, d_in = 64, 256
    w = synth.trimodal_weight(d_out, d_in, seed=64)
    dw = synth.optimizer_state(d_out, d_in, seed=64)[0]
    a, b = Opt(lib, w, 6, 8), Opt(lib, w, 6, 8)
    a.step(dw.cuda(), 1e-3, 1, count_flips=True)
    b.step(dw.cuda(), 1e-3, 1, count_flips=False)
    assert torch.equal(a.W, b.W) and torch.equal(a.bits, b.bits) and torch.equal(a.weff, b.weff)
    assert int(b.flips.item()) == 0 and int(a.flips.item()) > 0


def test_grad_sqnorm_ragged_and_deterministic(lib):
    """Several gradients into one accumulator, one with n % 4 != 0 (the tail
    path) and one empty; two runs are bitwise equal."""
    ws_bytes = lib.sbl_mask_quant_workspace_bytes(8, 16)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    grads = [synth.optimizer_state(1, 1000003 + 5, seed=65)[0].reshape(-1)[:1000003],
             synth.optimizer_state(256, 1024, seed=66)[0].reshape(-1),
             torch.zeros(0, dtype=torch.float32)]
    dev = []
    for g in grads:
        buf = torch.zeros(max(g.numel(), 4) + 4, dtype=torch.float32, device="cuda")  # 16-byte aligned start
        buf[: g.numel()] = g.cuda()
        dev.append((buf, g.numel()))
    out = []
    for _ in range(2):
        s = torch.zeros(1, dtype=torch.float64, device="cuda")
        for buf, n in dev:
            lib.sbl_grad_sqnorm(buf, n, s, ws, ws_bytes)
        lib.sbl_check()
        out.append(s.item())
    assert out[0] == out[1]
    assert out[0] == pytest.approx(oracle.grad_sqnorm(*[g.numpy() for g in grads]), rel=1e-12)


def test_adamw_full_size_projection(lib):
    """The 3B up projection (11008 x 2048, 22.5 M weights, 6:8) at step 1000
    with clipping at the pages' max_norm = 1 against the whole oracle."""
    d_out, d_in = 11008, 2048
    w = synth.trimodal_weight(d_out, d_in, seed=67)
    dw, m0, v0 = synth.optimizer_state(d_out, d_in, seed=67, g_std=1e-3)
    o = Opt(lib, w, 6, 8)
    o.m.copy_(m0)
    o.v.copy_(v0)
    sumsq = torch.zeros(1, dtype=torch.float64, device="cuda")
    dW = dw.cuda()
    lib.sbl_grad_sqnorm(dW, dW.numel(), sumsq, o.ws, o.ws_bytes)
    o.step(dW, 1e-3, 1000, sumsq, 1.0)
    S = oracle.grad_sqnorm(dw.numpy())
    assert sumsq.item() == pytest.approx(S, rel=1e-12)
    c = oracle.grad_clip_scale(S, 1.0)
    assert c < 1.0  # norm about 4.7 at this size
    ref = oracle.adamw_weight_step(synth.bits(w), dw.numpy(), m0.numpy(), v0.numpy(), 6, 8,
                                   oracle.adamw_scalars(1e-3, step=1000, **HP), c)
    _check_against(o, ref)
