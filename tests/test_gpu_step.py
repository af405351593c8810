"""The training step as bench.py runs it, on the GPU, against the oracle.

* Pipelined weight side: each step's mask, gamma and W_eff are computed during
  the previous step's backward, on side streams, into the other of two buffer
  sets.  Three consecutive steps must each give the oracle's W_eff, gamma and
  int32-exact y, and dX and dW within the backward tolerance; a race between
  the side streams and the products would show here.
* Data-parallel training step (one rank: the dW exchange is a no-op): after
  one step, the bf16 master W, the moments, the next W_eff, gamma and mask
  must equal the oracle's AdamW step applied to the step's own dW with the
  step's global norm, bit for bit.
"""
import numpy as np
import pytest
import torch

import bench
import oracle
import synth
from bwd_tol import abs_dw, abs_dx, check_bwd

pytestmark = pytest.mark.gpu

T = 256


def _inputs(ls):
    W, X, dY = bench.make_inputs(ls, T, seed=3, device="cpu")
    return W, X, dY


def test_pipelined_weight_side_matches_oracle_every_step(lib):
    ls = synth.layer_set("qwen2.5-0.5b")
    W, X, dY = _inputs(ls)
    Wg = {k: v.cuda() for k, v in W.items()}
    Xg = {k: v.cuda() for k, v in X.items()}
    dYg = {k: v.cuda() for k, v in dY.items()}
    st = bench.Step(ls, T, Wg, Xg, dYg, 6, 8, False)
    st.enable_pipelined_weights()
    stream = torch.cuda.Stream()
    ref = {}
    for i, p in enumerate(ls.projections):
        wb = synth.bits(W[p.name])
        weff, gamma, _ = oracle.effective_weight(wb, 6, 8)
        xb = synth.bits(X[p.input_name])
        xq, amax = oracle.act_quant(xb)
        dyb = synth.bits(dY[p.name])
        ref[p.name] = dict(weff=weff, gamma=gamma, y=oracle.forward_out(oracle.forward_acc(xq, weff), gamma, amax),
                           dx=oracle.backward_dx(dyb, weff, gamma), dw=oracle.backward_dw(dyb, xb),
                           adx=abs_dx(dyb, weff, gamma), adw=abs_dw(dyb, xb))
    used = []
    for step in range(3):
        layers = st.layers  # the buffer set this step multiplies with
        used.append(id(layers))
        st.run(stream)
        stream.synchronize()
        lib.sbl_check()
        for p in ls.projections:
            r = ref[p.name]
            L = layers[p.name]
            assert np.array_equal(L.W_eff.cpu().numpy(), r["weff"]), (step, p.name)
            assert L.gamma.item() == float(r["gamma"]), (step, p.name)
            np.testing.assert_allclose(st.Y[p.name].cpu().numpy(), r["y"], rtol=1e-3)
            check_bwd(st.dX[p.name].cpu().numpy(), r["dx"], r["adx"], f"step {step} {p.name} dX")
            check_bwd(st.dW[p.name].cpu().numpy(), r["dw"], r["adw"], f"step {step} {p.name} dW")
    assert used[0] == used[2] != used[1]  # the two buffer sets alternate


def test_data_parallel_training_step_matches_oracle_adamw(lib):
    ls = synth.layer_set("qwen2.5-0.5b")
    W, X, dY = _inputs(ls)
    Wg = {k: v.cuda() for k, v in W.items()}
    st = bench.Step(ls, T, Wg, {k: v.cuda() for k, v in X.items()}, {k: v.cuda() for k, v in dY.items()}, 6, 8,
                    False)
    st.enable_training(lr=1e-3)
    stream = torch.cuda.Stream()
    st.run(stream)
    stream.synchronize()
    lib.sbl_check()
    dws = {p.name: st.dW[p.name].cpu().numpy().copy() for p in ls.projections}
    S = float(st.sumsq.item())
    assert S == pytest.approx(oracle.grad_sqnorm(*dws.values()), rel=1e-12)
    clip = oracle.grad_clip_scale(S, st.hp["max_norm"])
    sc = oracle.adamw_scalars(st.hp["lr"], st.hp["betas"][0], st.hp["betas"][1], st.hp["eps"],
                              st.hp["weight_decay"], step=1)
    flips = 0
    for p in ls.projections:
        z = np.zeros((p.d_out, p.d_in), np.float32)
        r = oracle.adamw_weight_step(synth.bits(W[p.name]), dws[p.name], z, z, 6, 8, sc, clip)
        L = st.layers[p.name]
        assert np.array_equal(synth.bits(L.W.cpu()), r["w_bits"]), p.name
        assert np.array_equal(st.m[p.name].cpu().numpy(), r["m"]), p.name
        assert np.array_equal(st.v[p.name].cpu().numpy(), r["v"]), p.name
        assert np.array_equal(L.W_eff.cpu().numpy(), r["weff"]), p.name
        assert L.gamma.item() == float(r["gamma"]), p.name
        keep = np.unpackbits(L.mask_bits.cpu().numpy(), axis=1, bitorder="little").astype(bool)
        assert np.array_equal(keep, r["keep"]), p.name
        flips += r["flips"]
    assert int(st.flips.item()) == flips
