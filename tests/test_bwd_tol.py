"""The backward tolerance itself (CPU): an fp32-accumulated product passes
it, and the mistakes it exists to catch (a dropped block of the reduction, a
wrong split-K partial, a transposed operand) fail it."""
import numpy as np
import pytest
import torch

import oracle
import synth
from bwd_tol import abs_dw, abs_dx, check_bwd


def _inputs(T=1024, d_out=96, d_in=160, seed=31):
    x = synth.bits(synth.activations(T, d_in, seed=seed, tensor_id=1))
    dy = synth.bits(synth.grad_output(T, d_out, seed=seed, tensor_id=2))
    w = synth.bits(synth.trimodal_weight(d_out, d_in, seed=seed, tensor_id=3))
    weff, gamma, _ = oracle.effective_weight(w, 6, 8)
    return x, dy, weff, gamma


def _f32(bits):
    return torch.from_numpy(oracle.bf16_to_f32(bits))


def test_fp32_accumulated_products_pass():
    x, dy, weff, gamma = _inputs()
    dw32 = (_f32(dy).T @ _f32(x)).numpy()                      # fp32 accumulation
    med = check_bwd(dw32, oracle.backward_dw(dy, x), abs_dw(dy, x), "dW fp32")
    assert med < 1e-5
    dx32 = (float(gamma) * (_f32(dy) @ torch.from_numpy(weff.astype(np.float32)))).numpy()
    check_bwd(dx32, oracle.backward_dx(dy, weff, gamma), abs_dx(dy, weff, gamma), "dX fp32")
    # sequential fp32 sums over 128-token blocks, the order a K-blocked kernel takes
    acc = np.zeros((dy.shape[1], x.shape[1]), np.float32)
    for s in range(0, x.shape[0], 128):
        acc = (acc + (_f32(dy[s:s + 128]).T @ _f32(x[s:s + 128])).numpy()).astype(np.float32)
    check_bwd(acc, oracle.backward_dw(dy, x), abs_dw(dy, x), "dW blocked")


def test_dropped_block_fails():
    x, dy, weff, gamma = _inputs()
    ref = oracle.backward_dw(dy, x)
    bad = (_f32(dy[128:]).T @ _f32(x[128:])).numpy()           # first 128 tokens lost
    with pytest.raises(AssertionError):
        check_bwd(bad, ref, abs_dw(dy, x), "dW dropped block")


def test_one_wrong_tile_fails():
    """A split-K partial of 64 tokens added twice on one 32 x 32 tile."""
    x, dy, weff, gamma = _inputs()
    ref = oracle.backward_dw(dy, x)
    part = (_f32(dy[:64]).T @ _f32(x[:64])).numpy()
    bad = ref.astype(np.float32).copy()
    bad[:32, :32] += part[:32, :32]
    with pytest.raises(AssertionError):
        check_bwd(bad, ref, abs_dw(dy, x), "dW tile")


def test_transposed_weight_fails():
    x, dy, weff, gamma = _inputs(d_out=160, d_in=160)
    ref = oracle.backward_dx(dy, weff, gamma)
    bad = oracle.backward_dx(dy, np.ascontiguousarray(weff.T), gamma)
    with pytest.raises(AssertionError):
        check_bwd(bad, ref, abs_dx(dy, weff, gamma), "dX transposed")
