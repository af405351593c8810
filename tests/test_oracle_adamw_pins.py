"""Pins for the oracle's optimizer step: AdamW on the master weight, the
gradient-norm clip and the mask flip count.

Sparse-BitNet summary, Algorithm 1 step (8) (AdamW with beta = (0.9, 0.95),
eps = 1e-5, weight decay 0.1, grad clip 1.0, BF16 master weight) and the
weaknesses section (the mask flip rate of Fig. 3b).  The pins check the
oracle against closed forms of the first step, against torch.optim.AdamW and
torch.nn.utils.clip_grad_norm_ (independent library implementations of the
textbook algorithms), and against a brute-force flip count.  A dropped bias
correction, a swapped moment, a coupled (L2) decay, a wrong sign or an
off-by-one step fails at least one of them.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import synth

HP = dict(beta1=0.9, beta2=0.95, eps=1e-5, weight_decay=0.1)


def _state(shape, seed):
    dw, m, v = synth.optimizer_state(*shape, seed=seed)
    return dw.numpy(), m.numpy(), v.numpy()


def test_first_step_closed_form():
    """t = 1 from zero moments: m' = (1 - b1) g, v' = (1 - b2) g^2, and the
    bias-corrected step is g / (|g| + eps), so
    w' = w (1 - lr wd) - lr g / (|g| + eps)."""
    lr = 1e-3
    rng = np.random.default_rng(5)
    w = rng.normal(0, 0.02, 4096).astype(np.float32)
    g = (rng.normal(0, 1e-3, 4096) * rng.choice([1e-3, 1.0, 1e3], 4096)).astype(np.float32)
    z = np.zeros_like(w)
    sc = oracle.adamw_scalars(lr, step=1, **HP)
    w1, m1, v1 = oracle.adamw_update(w, g, z, z, sc)
    g64, w64 = g.astype(np.float64), w.astype(np.float64)
    np.testing.assert_allclose(m1, 0.1 * g64, rtol=2e-7)
    np.testing.assert_allclose(v1, 0.05 * g64 * g64, rtol=4e-7)
    want = w64 * (1 - lr * 0.1) - lr * g64 / (np.abs(g64) + 1e-5)
    np.testing.assert_allclose(w1, want, rtol=0, atol=4 * np.spacing(np.float32(0.1)))
    # the sign: a positive gradient lowers the weight by about lr
    big = np.abs(g64) > 1e-3
    assert np.all(np.sign(w64 * (1 - lr * 0.1) - w1)[big] == np.sign(g64[big]))


def test_weight_decay_alone():
    """No gradient and zero moments: the update term is 0 / eps = 0 and only
    the decoupled decay acts, w' = fl32(w * fl32(1 - lr wd))."""
    lr = 3e-4
    w = np.float32([0.5, -0.25, 1e-3, 0.0, -7.0])
    z = np.zeros_like(w)
    sc = oracle.adamw_scalars(lr, step=7, **HP)
    w1, m1, v1 = oracle.adamw_update(w, z, z, z, sc)
    assert np.array_equal(w1, w * np.float32(1 - lr * 0.1))
    assert not m1.any() and not v1.any()


def test_zero_lr_keeps_weight_and_mask():
    """lr = 0: decay = 1 and alpha = 0, so every weight comes back bit for
    bit and no mask entry flips."""
    shape = (8, 64)
    wb = synth.bits(synth.normal_weight(*shape, seed=3))
    dw, m, v = _state(shape, 3)
    sc = oracle.adamw_scalars(0.0, step=3, **HP)
    out = oracle.adamw_weight_step(wb, dw, m, v, 6, 8, sc)
    assert np.array_equal(out["w_bits"], wb)
    assert out["flips"] == 0


@pytest.mark.parametrize("start", [0, 999])
def test_matches_torch_adamw(start):
    """Six steps against torch.optim.AdamW on an fp32 parameter.  The library
    orders some fp32 operations differently (it forms m' as a lerp, which
    cancels where m and g differ in sign), so the moments agree to a few
    ulps of their own scale rather than of each element."""
    shape = (16, 128)
    lr = 2e-3
    w0 = synth.normal_weight(*shape, seed=11).float().numpy()
    _, m0, v0 = _state(shape, 11)
    p = torch.nn.Parameter(torch.from_numpy(w0.copy()))
    opt = torch.optim.AdamW([p], lr=lr, betas=(HP["beta1"], HP["beta2"]), eps=HP["eps"],
                            weight_decay=HP["weight_decay"], foreach=False, fused=False)
    opt.state[p] = {"step": torch.tensor(float(start)), "exp_avg": torch.from_numpy(m0.copy()),
                    "exp_avg_sq": torch.from_numpy(v0.copy())}
    w, m, v = w0.copy(), m0.copy(), v0.copy()
    for k in range(6):
        g = synth.optimizer_state(*shape, seed=100 + k)[0].numpy()
        p.grad = torch.from_numpy(g.copy())
        opt.step()
        w, m, v = oracle.adamw_update(w, g, m, v, oracle.adamw_scalars(lr, step=start + k + 1, **HP))
    st = opt.state[p]
    tm, tv = st["exp_avg"].numpy(), st["exp_avg_sq"].numpy()
    np.testing.assert_allclose(m, tm, rtol=1e-6, atol=2e-6 * np.abs(tm).max())
    np.testing.assert_allclose(v, tv, rtol=1e-6, atol=2e-6 * np.abs(tv).max())
    np.testing.assert_allclose(w, p.detach().numpy(), rtol=0, atol=8 * np.spacing(np.float32(0.1)))
    # and the update is not lost in that tolerance
    assert np.abs(w - w0).max() > 100 * np.spacing(np.float32(0.1))


@pytest.mark.parametrize("max_norm", [0.01, 1.0])
def test_clip_matches_torch(max_norm):
    """The clip factor of several gradients against clip_grad_norm_ (fp64
    gradients, so its norm is the fp64 one).  The gradients' norm is about
    0.04, so max_norm = 0.01 clips and max_norm = 1 (the pages' value) gives
    exactly 1."""
    grads = [synth.optimizer_state(8, 32 * (k + 1), seed=20 + k)[0].numpy() for k in range(3)]
    S = oracle.grad_sqnorm(*grads)
    ps = [torch.nn.Parameter(torch.zeros(g.shape, dtype=torch.float64)) for g in grads]
    for p, g in zip(ps, grads):
        p.grad = torch.from_numpy(g.astype(np.float64))
    total = float(torch.nn.utils.clip_grad_norm_(ps, max_norm))
    assert math.sqrt(S) == pytest.approx(total, rel=1e-14)
    c = oracle.grad_clip_scale(S, max_norm)
    want = min(1.0, max_norm / (total + 1e-6))
    assert c == pytest.approx(want, rel=6e-8)
    if max_norm >= 1.0:
        assert c == np.float32(1.0)
    else:
        assert c < 1.0
        # clip_grad_norm_ scaled the gradients by the same factor
        np.testing.assert_allclose(ps[0].grad.numpy(), grads[0].astype(np.float64) * want, rtol=1e-12)


def test_clip_scales_gradient_before_moments():
    """With clipping, the first step from zero moments is the unclipped one
    for a scale-invariant part (g / |g|) but the moments shrink by c."""
    g = np.float32([4e-3, -2e-3, 1e-3])
    z = np.zeros_like(g)
    sc = oracle.adamw_scalars(1e-3, step=1, **HP)
    c = np.float32(0.25)
    _, m1, v1 = oracle.adamw_update(z, g, z, z, sc, clip=c)
    np.testing.assert_allclose(m1, 0.1 * 0.25 * g.astype(np.float64), rtol=2e-7)
    np.testing.assert_allclose(v1, 0.05 * (0.25 * g.astype(np.float64)) ** 2, rtol=4e-7)


def _brute_keep(w, N, M):
    keep = np.zeros(w.shape, bool)
    for r in range(w.shape[0]):
        for g0 in range(0, w.shape[1], M):
            order = sorted(range(M), key=lambda j: (-abs(float(w[r, g0 + j])), j))
            for j in order[:N]:
                keep[r, g0 + j] = True
    return keep


def test_flip_count_brute_force():
    """Flips between the masks of two weights, counted position by position
    with a sort per group; within a group the count is even (N kept before
    and after)."""
    a = synth.normal_weight(6, 32, seed=41)
    b = (a.float() + synth.normal_weight(6, 32, seed=42).float() * 0.5).to(torch.bfloat16)
    ab, bb = synth.bits(a), synth.bits(b)
    ka, kb = _brute_keep(a.float().numpy(), 6, 8), _brute_keep(b.float().numpy(), 6, 8)
    count = sum(int(ka[r, c] != kb[r, c]) for r in range(6) for c in range(32))
    assert count > 0
    assert oracle.mask_flips(oracle.nm_mask(ab, 6, 8), oracle.nm_mask(bb, 6, 8)) == count
    per_group = (ka != kb).reshape(6, 4, 8).sum(axis=2)
    assert np.all(per_group % 2 == 0)


def test_bf16_master_rounds_once():
    """The pages' bf16 master: the new W is bf16_rn of the fp32 result, so an
    update below half a bf16 ulp is lost, while an fp32 master keeps it."""
    wb = synth.bits(torch.tensor([[1.0] * 8], dtype=torch.bfloat16))
    dw = np.full((1, 8), 1e-3, np.float32)
    z = np.zeros((1, 8), np.float32)
    sc = oracle.adamw_scalars(1e-5, step=1, **HP)
    out16 = oracle.adamw_weight_step(wb, dw, z, z, 8, 8, sc)
    assert np.array_equal(out16["w_bits"], wb)            # 1 - 1e-5 rounds back to 1.0
    out32 = oracle.adamw_weight_step(wb, dw, z, z, 8, 8, sc, w32=np.ones((1, 8), np.float32))
    assert np.all(out32["w32"] < 1.0) and np.all(out32["w32"] > 1.0 - 2e-5)
    assert np.array_equal(out32["w_bits"], wb)


def test_weight_step_feeds_next_mask():
    """The step's mask, gamma and W_eff are those of the new bf16 weight, and
    its flip count compares the masks of the old and new weights."""
    shape = (8, 64)
    wb = synth.bits(synth.trimodal_weight(*shape, seed=9))
    dw, m, v = _state(shape, 9)
    dw *= 30.0   # large enough steps that some masks change
    sc = oracle.adamw_scalars(5e-3, step=2, **HP)
    out = oracle.adamw_weight_step(wb, dw, m, v, 6, 8, sc)
    weff, gamma, keep = oracle.effective_weight(out["w_bits"], 6, 8)
    assert np.array_equal(weff, out["weff"]) and gamma == out["gamma"]
    assert np.array_equal(keep, out["keep"])
    assert out["flips"] == int((oracle.nm_mask(wb, 6, 8) != keep).sum()) > 0
