"""GPU parity at the benchmark's full sizes, in the launch configuration
bench.py times (same C-ABI calls, same shapes, same inputs).

The oracle computes gamma and W_eff for every full weight tensor itself;
outputs whose oracle cost grows with T x params are compared on a seeded
sample: 64 tokens (activation codes, int32 accumulators, y, dX) and 64 output
rows of W (dW).  Tolerances as in test_gpu_parity.py (``bwd_tol`` for dX
and dW).
"""
import numpy as np
import pytest
import torch

import bench
import oracle
import synth
from bwd_tol import abs_dx, check_bwd

pytestmark = pytest.mark.gpu

def _dw_rows(dy_bits, x_bits, rows, chunk=4096):
    """Oracle dW restricted to output rows `rows`, summed over token chunks
    (fp64 throughout; bounds host memory for the 32768-token inputs), and
    the sum of absolute products behind each of those outputs."""
    out = np.zeros((len(rows), x_bits.shape[1]), np.float64)
    absb = np.zeros_like(out)
    for s in range(0, dy_bits.shape[0], chunk):
        out += oracle.backward_dw(dy_bits[s:s + chunk][:, rows], x_bits[s:s + chunk]).astype(np.float64)
        dy = np.abs(oracle.bf16_to_f32(dy_bits[s:s + chunk][:, rows]).astype(np.float64))
        absb += dy.T @ np.abs(oracle.bf16_to_f32(x_bits[s:s + chunk]).astype(np.float64))
    return out, absb


def _run_layer_set(name, T, N=6, M=8, sample=64, seed=0, sparse24=False):
    import semi_structured_sparsity_step_b200 as sbl
    from semi_structured_sparsity_step_b200.layer import SparseBitLinearLayer
    ls = synth.layer_set(name)
    W, X, dY = bench.make_inputs(ls, T, seed=seed, device="cpu")
    rng = np.random.default_rng(1234)
    toks = np.sort(rng.choice(T, size=min(sample, T), replace=False))
    Xg = {k: v.cuda() for k, v in X.items()}
    xq = {n: torch.empty(T, d, dtype=torch.int8, device="cuda") for n, d in ls.inputs.items()}
    amax = {n: torch.empty(T, dtype=torch.float32, device="cuda") for n in ls.inputs}
    for n, d in ls.inputs.items():
        sbl.sbl_act_quant(Xg[n], T, d, xq[n], amax[n])
    # activation codes on the sampled tokens
    xb = {n: synth.bits(X[n]) for n in ls.inputs}
    for n in ls.inputs:
        rq, ra = oracle.act_quant(xb[n][toks])
        assert np.array_equal(xq[n][toks].cpu().numpy(), rq), n
        assert np.array_equal(amax[n][toks].cpu().numpy(), ra), n
    for i, p in enumerate(ls.projections):
        L = SparseBitLinearLayer(W[p.name].cuda(), N, M, sparse24=sparse24)
        L.weight_step()
        wb = synth.bits(W[p.name])
        weff, gamma, _ = oracle.effective_weight(wb, N, M)
        assert L.gamma.item() == float(gamma), p.name
        assert np.array_equal(L.W_eff.cpu().numpy(), weff), p.name
        Y = torch.empty(T, p.d_out, dtype=torch.float32, device="cuda")
        acc = torch.empty(T, p.d_out, dtype=torch.int32, device="cuda")
        L.forward(xq[p.input_name], amax[p.input_name], Y, acc=acc)
        rq, ra = oracle.act_quant(xb[p.input_name][toks])
        racc = oracle.forward_acc(rq, weff)
        assert np.array_equal(acc[toks].cpu().numpy(), racc), p.name
        np.testing.assert_allclose(Y[toks].cpu().numpy(), oracle.forward_out(racc, gamma, ra), rtol=1e-3)
        dYg = dY[p.name].cuda()
        dX = torch.empty(T, p.d_in, dtype=torch.float32, device="cuda")
        dW = torch.empty(p.d_out, p.d_in, dtype=torch.float32, device="cuda")
        L.backward(dYg, Xg[p.input_name], dX, None)
        L.backward(dYg, Xg[p.input_name], None, dW)
        sbl.sbl_check()
        dyb = synth.bits(dY[p.name])
        check_bwd(dX[toks].cpu().numpy(), oracle.backward_dx(dyb[toks], weff, gamma),
                  abs_dx(dyb[toks], weff, gamma), f"{p.name} dX")
        rows = np.sort(rng.choice(p.d_out, size=min(sample, p.d_out), replace=False))
        rdw, adw = _dw_rows(dyb, xb[p.input_name], rows)
        check_bwd(dW[rows].cpu().numpy(), rdw, adw, f"{p.name} dW")
        del L, Y, acc, dX, dW, dYg
        torch.cuda.empty_cache()


def test_qwen05b_layer_set_4096_tokens():
    """0.5B-shaped layer set, 4096 tokens (8 x 512), 6:8, W ~ N(0, 0.02)."""
    _run_layer_set("qwen2.5-0.5b", 4096)


def test_qwen3b_layer_set_32768_tokens():
    """3B-shaped layer set, 32768 tokens (16 x 2048), 6:8, trimodal W,
    0.1% outlier channels: the benchmark's workload."""
    _run_layer_set("qwen2.5-3b", 32768)


@pytest.mark.parametrize("N,M", [(8, 8), (6, 8), (4, 8), (2, 8), (2, 4)])
def test_nm_sweep_up_proj_8192_tokens(N, M, monkeypatch):
    """3B up projection 11008 x 2048, 8192 tokens, trimodal W with exact |W|
    ties in 1% of groups, for every N:M of the sweep."""
    monkeypatch.setattr(bench, "N_KEEP", N)
    monkeypatch.setattr(bench, "M_GROUP", M)
    _run_layer_set("qwen2.5-3b-up", 8192, N=N, M=M)


def test_2of4_sparse_tensor_core_up_proj_8192_tokens(monkeypatch):
    """The 2:4 sweep point with the forward on the sparse tensor core
    (sbl_compress24 + sbl_forward_sparse24), at the benchmark's size."""
    monkeypatch.setattr(bench, "N_KEEP", 2)
    monkeypatch.setattr(bench, "M_GROUP", 4)
    _run_layer_set("qwen2.5-3b-up", 8192, N=2, M=4, sparse24=True)


@pytest.mark.parametrize("batch", [1, 8, 16])
def test_decode_gemv_on_packed_3b_layers(batch):
    """Decode on the packed 6:8 format of every 3B projection (batch 1, 8,
    16): packed bytes on sampled rows and the full GEMV output against the
    oracle."""
    import semi_structured_sparsity_step_b200 as sbl
    ls = synth.layer_set("qwen2.5-3b")
    rng = np.random.default_rng(99)
    for i, p in enumerate(ls.projections):
        w = bench.make_weight(ls, i, p)
        weff, gamma, _ = oracle.effective_weight(synth.bits(w), 6, 8)
        nbytes = sbl.sbl_packed_bytes(p.d_out, p.d_in, 6, 8)
        packed = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
        sbl.sbl_pack(torch.from_numpy(weff).cuda(), p.d_out, p.d_in, 6, 8, packed, nbytes)
        crow, irow, _ = oracle.packed_layout(p.d_out, p.d_in, 6, 8)
        rows = np.sort(rng.choice(p.d_out, size=16, replace=False))
        got = packed.cpu().numpy()
        for r in rows:
            ref = oracle.pack(weff[r:r + 1], 6, 8)
            assert np.array_equal(got[r * crow:(r + 1) * crow], ref[:crow]), (p.name, r)
            base = p.d_out * crow
            assert np.array_equal(got[base + r * irow: base + (r + 1) * irow], ref[crow:]), (p.name, r)
        x = synth.activations(batch, p.d_in, seed=5, tensor_id=100 + i)
        xq, amax = oracle.act_quant(synth.bits(x))
        Y = torch.empty(batch, p.d_out, dtype=torch.float32, device="cuda")
        g = torch.tensor([float(gamma)], dtype=torch.float32, device="cuda")
        sbl.sbl_gemv_packed(torch.from_numpy(xq).cuda(), torch.from_numpy(amax).cuda(), batch, packed, g, p.d_in,
                            p.d_out, 6, 8, Y)
        sbl.sbl_check()
        ref = oracle.forward_out(oracle.forward_acc(xq, weff), gamma, amax)
        assert np.array_equal(Y.cpu().numpy(), ref), p.name
