"""GPU parity: the CUDA path through the C ABI against the CPU oracle.

Bit-exact: keep masks, ternary codes (int8 and bf16 copies), gamma, int8
activations, amax, int32 accumulators, packed bytes.  Float outputs: the
forward output within a relative 1e-3 (it is computed with the same fp32
operation order, so it is normally bit-equal); dX and dW (bf16 tensor-core
products with fp32 accumulation against an fp64 oracle) within
max|gpu - ref| <= 2e-2 * max|ref| per tensor and, element by element, within
the fp32 accumulation bound of ``bwd_tol``.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from bwd_tol import abs_dw, abs_dx, check_bwd

pytestmark = pytest.mark.gpu

REL_Y = 1e-3


def _dev(t):
    return t.to("cuda")


def _unpack_mask(bits: np.ndarray) -> np.ndarray:
    return np.unpackbits(bits, axis=1, bitorder="little").astype(bool)


def _check_y(gpu: np.ndarray, ref: np.ndarray):
    np.testing.assert_allclose(gpu, ref, rtol=REL_Y, atol=REL_Y * np.abs(ref).max() * 1e-3)


class Layer:
    """Runs the whole path for one layer on the GPU and keeps host copies."""

    def __init__(self, lib, w, x, dy, N, M, accumulate=None):
        from semi_structured_sparsity_step_b200.layer import SparseBitLinearLayer, act_quant
        d_out, d_in = w.shape
        T = x.shape[0]
        self.L = SparseBitLinearLayer(_dev(w), N, M, keep_mask=True)
        self.L.weight_step()
        X = _dev(x)
        self.Xq = torch.empty(T, d_in, dtype=torch.int8, device="cuda")
        self.amax = torch.empty(max(T, 1), dtype=torch.float32, device="cuda")
        act_quant(X, self.Xq, self.amax)
        self.Y = torch.empty(T, d_out, dtype=torch.float32, device="cuda")
        self.acc = torch.empty(T, d_out, dtype=torch.int32, device="cuda")
        self.L.forward(self.Xq, self.amax, self.Y, acc=self.acc)
        dY = _dev(dy)
        self.dX = torch.empty(T, d_in, dtype=torch.float32, device="cuda")
        self.dW = torch.empty(d_out, d_in, dtype=torch.float32, device="cuda") if accumulate is None \
            else _dev(accumulate.clone())
        self.L.backward(dY, X, self.dX, self.dW, accumulate_dW=accumulate is not None)
        lib.sbl_check()
        torch.cuda.synchronize()


def _full_parity(lib, w, x, dy, N, M):
    g = Layer(lib, w, x, dy, N, M)
    wb, xb, dyb = synth.bits(w), synth.bits(x), synth.bits(dy)
    ref = oracle.forward(xb, wb, N, M)
    assert np.array_equal(_unpack_mask(g.L.mask_bits.cpu().numpy()), ref["keep"])
    assert g.L.gamma.item() == float(ref["gamma"])
    assert np.array_equal(g.L.W_eff.cpu().numpy(), ref["weff"])
    assert np.array_equal(oracle.bf16_to_f32(synth.bits(g.L.W_eff_bf16.cpu())), ref["weff"].astype(np.float32))
    assert np.array_equal(g.Xq.cpu().numpy(), ref["xq"])
    assert np.array_equal(g.amax.cpu().numpy()[: x.shape[0]], ref["amax"])
    assert np.array_equal(g.acc.cpu().numpy(), ref["acc"])
    _check_y(g.Y.cpu().numpy(), ref["y"])
    check_bwd(g.dX.cpu().numpy(), oracle.backward_dx(dyb, ref["weff"], ref["gamma"]),
              abs_dx(dyb, ref["weff"], ref["gamma"]), "dX")
    check_bwd(g.dW.cpu().numpy(), oracle.backward_dw(dyb, xb), abs_dw(dyb, xb), "dW")
    return g, ref


@pytest.fixture(params=[0, 1], ids=["pair", "single"])
def variant(lib, request):
    """Runs a test with each tensor-core kernel variant (CTA pairs, one CTA)."""
    lib.sbl_set_gemm_variant(request.param)
    yield request.param
    lib.sbl_set_gemm_variant(0)


def test_library_loads_on_gpu(lib):
    assert lib.sbl_version() >= 100
    lib.sbl_check()


def test_single_layer_256_6of8_full_parity(lib, variant):
    """One 256 x 256 layer, 64 tokens, 6:8, W ~ N(0, 0.02), X, dY ~ N(0, 1)."""
    w = synth.normal_weight(256, 256, seed=0, tensor_id=0)
    x = synth.activations(64, 256, seed=0, tensor_id=100)
    dy = synth.grad_output(64, 256, seed=0, tensor_id=200)
    g, ref = _full_parity(lib, w, x, dy, 6, 8)
    assert np.array_equal(g.Y.cpu().numpy(), ref["y"])  # same fp32 op order: bit-equal


@pytest.mark.parametrize("T,d_out,d_in,N,M", [
    (1, 8, 16, 6, 8), (7, 136, 48, 2, 4), (129, 264, 272, 6, 8), (200, 392, 400, 4, 8),
    (130, 256, 1040, 3, 4), (333, 520, 144, 8, 8), (64, 8, 2064, 1, 8),
])
def test_ragged_shapes(lib, variant, T, d_out, d_in, N, M):
    """Sizes that are not tile multiples (tiles are 128 x 256 x 128 bytes)."""
    w = synth.trimodal_weight(d_out, d_in, seed=3, tensor_id=T)
    x = synth.activations(T, d_in, seed=3, tensor_id=100 + T, outlier_frac=0.01)
    dy = synth.grad_output(T, d_out, seed=3, tensor_id=200 + T)
    _full_parity(lib, w, x, dy, N, M)


@pytest.mark.parametrize("N,M", [(8, 8), (6, 8), (4, 8), (2, 8), (2, 4), (1, 4), (3, 4)])
def test_mask_quant_sweep_with_ties(lib, N, M):
    """Exact |W| ties straddling the top-N boundary keep the lower index."""
    w = synth.trimodal_weight(384, 512, seed=4, tensor_id=N * 10 + M)
    if N < M:
        w = synth.with_boundary_ties(w, N, M, seed=4, frac=0.05, all_equal_groups=16)
    from semi_structured_sparsity_step_b200.layer import SparseBitLinearLayer
    L = SparseBitLinearLayer(_dev(w), N, M, keep_mask=True)
    L.weight_step()
    lib.sbl_check()
    weff, gamma, keep = oracle.effective_weight(synth.bits(w), N, M)
    assert np.array_equal(_unpack_mask(L.mask_bits.cpu().numpy()), keep)
    assert L.gamma.item() == float(gamma)
    assert np.array_equal(L.W_eff.cpu().numpy(), weff)


def test_gamma_exact_on_extreme_magnitudes(lib):
    """Magnitudes outside the fast window (subnormal, tiny, >= 2) and a
    sum that naive fp32/fp64 accumulation would round differently."""
    vals = torch.full((64, 64), 0.0)
    vals[0, :8] = torch.tensor([1.0, 2.0 ** -53, 2.0 ** -53, 3.0e-39, 1.0e-36, 300.0, -4096.0, 2.0 ** -40])
    vals[1:] = torch.randn(63, 64) * 0.02
    w = vals.to(torch.bfloat16)
    from semi_structured_sparsity_step_b200.layer import SparseBitLinearLayer
    L = SparseBitLinearLayer(_dev(w), 6, 8)
    L.weight_step()
    lib.sbl_check()
    weff, gamma, _ = oracle.effective_weight(synth.bits(w), 6, 8)
    assert L.gamma.item() == float(gamma)
    assert np.array_equal(L.W_eff.cpu().numpy(), weff)


@pytest.mark.parametrize("kind", ["zero", "constant_magnitude"])
def test_degenerate_weights(lib, kind):
    """An all-zero weight (gamma = 0: every weight is divided by eps alone and
    rounds to 0) and a weight of one magnitude with random signs (every group
    is a full tie, so the lowest N positions are kept, and every kept weight
    is +-1).  The whole path matches the oracle."""
    d_out, d_in, T, N, M = 136, 400, 70, 6, 8
    if kind == "zero":
        w = torch.zeros(d_out, d_in, dtype=torch.bfloat16)
    else:
        g = torch.Generator().manual_seed(11)
        sign = torch.randint(0, 2, (d_out, d_in), generator=g) * 2 - 1
        w = (sign.float() * 0.375).to(torch.bfloat16)
    x = synth.activations(T, d_in, seed=6, tensor_id=1)
    dy = synth.grad_output(T, d_out, seed=6, tensor_id=2)
    gl, ref = _full_parity(lib, w, x, dy, N, M)
    if kind == "zero":
        assert gl.L.gamma.item() == 0.0
        assert not gl.Y.cpu().numpy().any()
    else:
        keep = _unpack_mask(gl.L.mask_bits.cpu().numpy()).reshape(d_out, d_in // M, M)
        assert keep[:, :, :N].all() and not keep[:, :, N:].any()
        assert np.array_equal(np.abs(gl.L.W_eff.cpu().numpy()).reshape(d_out, d_in // M, M)[:, :, :N],
                              np.ones((d_out, d_in // M, N), np.int8))


@pytest.mark.parametrize("accumulate", [False, True])
def test_empty_token_batch(lib, variant, accumulate):
    """T = 0, an empty batch: the weight side still runs; quantisation, the
    forward product and dX have no rows to write; dW is the empty sum (all
    zeros, written over whatever the buffer held) or, when accumulating, the
    incoming gradient unchanged."""
    from semi_structured_sparsity_step_b200.layer import SparseBitLinearLayer, act_quant
    d_out, d_in, N, M = 264, 400, 6, 8
    w = synth.trimodal_weight(d_out, d_in, seed=5, tensor_id=0)
    x = synth.activations(0, d_in, seed=5, tensor_id=1)
    dy = synth.grad_output(0, d_out, seed=5, tensor_id=2)
    L = SparseBitLinearLayer(_dev(w), N, M, keep_mask=True)
    L.weight_step()
    X = _dev(x)
    Xq = torch.empty(0, d_in, dtype=torch.int8, device="cuda")
    amax = torch.full((1,), -1.0, dtype=torch.float32, device="cuda")
    act_quant(X, Xq, amax)
    Y = torch.empty(0, d_out, dtype=torch.float32, device="cuda")
    L.forward(Xq, amax, Y)
    dX = torch.empty(0, d_in, dtype=torch.float32, device="cuda")
    before = 0.25 if accumulate else float("nan")
    dW = torch.full((d_out, d_in), before, dtype=torch.float32, device="cuda")
    L.backward(_dev(dy), X, dX, dW, accumulate_dW=accumulate)
    lib.sbl_check()
    torch.cuda.synchronize()
    weff, gamma, _ = oracle.effective_weight(synth.bits(w), N, M)
    assert np.array_equal(L.W_eff.cpu().numpy(), weff)
    assert L.gamma.item() == float(gamma)
    assert amax.item() == -1.0  # nothing written for an empty batch
    assert torch.all(dW == (0.25 if accumulate else 0.0)).item()


def test_dw_split_k_and_accumulate(lib, variant):
    """Small d_out (k/v-like) takes the split-K path with atomics; the
    accumulate flag adds into an existing gradient."""
    T, d_out, d_in = 1000, 128, 512
    w = synth.normal_weight(d_out, d_in, seed=5)
    x = synth.activations(T, d_in, seed=5)
    dy = synth.grad_output(T, d_out, seed=5)
    prior = torch.randn(d_out, d_in, generator=torch.Generator().manual_seed(5))
    g = Layer(lib, w, x, dy, 6, 8, accumulate=prior)
    ref = oracle.backward_dw(synth.bits(dy), synth.bits(x)) + prior.numpy()
    check_bwd(g.dW.cpu().numpy(), ref, abs_dw(synth.bits(dy), synth.bits(x)) + np.abs(prior.numpy()),
              "dW accumulate")


def test_zero_activation_row(lib):
    """An all-zero token quantises to zeros with amax = 1e-5 and gives y = 0."""
    w = synth.normal_weight(64, 128, seed=6)
    x = synth.activations(5, 128, seed=6).to(torch.float32)
    x[2] = 0.0
    x = x.to(torch.bfloat16)
    dy = synth.grad_output(5, 64, seed=6)
    g, ref = _full_parity(lib, w, x, dy, 6, 8)
    assert (g.Xq[2] == 0).all() and g.amax[2].item() == np.float32(1e-5) and (g.Y[2] == 0).all()


def test_argument_errors_return_status(lib):
    import semi_structured_sparsity_step_b200._binding as B
    ll = B.load()
    W = torch.zeros(8, 16, dtype=torch.bfloat16, device="cuda")
    out = torch.zeros(8, 16, dtype=torch.int8, device="cuda")
    g = torch.zeros(1, device="cuda")
    ws = torch.zeros(1 << 16, dtype=torch.uint8, device="cuda")
    s = torch.cuda.current_stream().cuda_stream
    assert ll.sbl_mask_quant(W.data_ptr(), 8, 16, 7, 6, out.data_ptr(), None, None, g.data_ptr(), ws.data_ptr(),
                             ws.numel(), s) == 1  # M not in {4, 8}
    assert ll.sbl_mask_quant(W.data_ptr(), 8, 12, 6, 8, out.data_ptr(), None, None, g.data_ptr(), ws.data_ptr(),
                             ws.numel(), s) == 2  # d_in % 16
    assert ll.sbl_mask_quant(W.data_ptr() + 2, 8, 16, 6, 8, out.data_ptr(), None, None, g.data_ptr(),
                             ws.data_ptr(), ws.numel(), s) == 3  # misaligned
    assert ll.sbl_mask_quant(W.data_ptr(), 8, 16, 6, 8, out.data_ptr(), None, None, g.data_ptr(), ws.data_ptr(),
                             16, s) == 5  # workspace too small
    lib.sbl_check()


# ------------------------------------------------------------------ pack / GEMV
@pytest.mark.parametrize("N,M", [(6, 8), (2, 4), (8, 8), (4, 8), (1, 8), (3, 4)])
def test_pack_bytes_bit_exact(lib, N, M):
    d_out, d_in = 24, 272
    w = synth.trimodal_weight(d_out, d_in, seed=7, tensor_id=N * 10 + M)
    weff, _, _ = oracle.effective_weight(synth.bits(w), N, M)
    nbytes = lib.sbl_packed_bytes(d_out, d_in, N, M)
    assert nbytes == oracle.packed_layout(d_out, d_in, N, M)[2]
    packed = torch.full((nbytes,), 0xAB, dtype=torch.uint8, device="cuda")
    lib.sbl_pack(torch.from_numpy(weff).cuda(), d_out, d_in, N, M, packed, nbytes)
    lib.sbl_check()
    assert np.array_equal(packed.cpu().numpy(), oracle.pack(weff, N, M))


def test_pack_rejects_too_many_nonzeros(lib):
    weff = torch.ones(8, 16, dtype=torch.int8, device="cuda")
    nbytes = lib.sbl_packed_bytes(8, 16, 6, 8)
    packed = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    lib.sbl_pack(weff, 8, 16, 6, 8, packed, nbytes)
    with pytest.raises(lib.SblError) as e:
        lib.sbl_check()
    assert e.value.status == 8
    lib.sbl_check()  # the latched error was cleared


@pytest.fixture(params=[0, 1, 2], ids=["stream", "ring", "direct"])
def gemv_variant(request, lib):
    """Runs a GEMV test with each decode kernel (sbl_set_gemv_variant)."""
    lib.sbl_set_gemv_variant(request.param)
    yield request.param
    lib.sbl_set_gemv_variant(0)


@pytest.mark.parametrize("batch", [1, 3, 8, 16])
@pytest.mark.parametrize("N,M", [(6, 8), (2, 4), (8, 8)])
def test_gemv_packed_parity(lib, gemv_variant, batch, N, M):
    d_out, d_in = 520, 2064
    w = synth.trimodal_weight(d_out, d_in, seed=8, tensor_id=batch)
    weff, gamma, _ = oracle.effective_weight(synth.bits(w), N, M)
    x = synth.activations(batch, d_in, seed=8, tensor_id=100 + batch)
    xq, amax = oracle.act_quant(synth.bits(x))
    nbytes = lib.sbl_packed_bytes(d_out, d_in, N, M)
    packed = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    lib.sbl_pack(torch.from_numpy(weff).cuda(), d_out, d_in, N, M, packed, nbytes)
    Y = torch.empty(batch, d_out, dtype=torch.float32, device="cuda")
    g = torch.tensor([float(gamma)], dtype=torch.float32, device="cuda")
    lib.sbl_gemv_packed(torch.from_numpy(xq).cuda(), torch.from_numpy(amax).cuda(), batch, packed, g, d_in, d_out,
                        N, M, Y)
    lib.sbl_check()
    ref = oracle.forward_out(oracle.forward_acc(xq, weff), gamma, amax)
    assert np.array_equal(Y.cpu().numpy(), ref)


def test_gamma_exact_on_log_uniform_magnitudes(lib):
    """Magnitudes spread log-uniformly over 2^-133 .. 2^12 fill many exponent
    buckets as well as the register window; gamma and the codes stay exact."""
    g = torch.Generator().manual_seed(11)
    e = torch.rand(512, 1024, generator=g) * 145.0 - 133.0
    sign = torch.where(torch.rand(512, 1024, generator=g) < 0.5, -1.0, 1.0)
    w = (sign * torch.exp2(e)).to(torch.bfloat16)
    from semi_structured_sparsity_step_b200.layer import SparseBitLinearLayer
    for N, M in [(6, 8), (2, 4)]:
        L = SparseBitLinearLayer(_dev(w), N, M)
        L.weight_step()
        lib.sbl_check()
        weff, gamma, _ = oracle.effective_weight(synth.bits(w), N, M)
        assert L.gamma.item() == float(gamma)
        assert np.array_equal(L.W_eff.cpu().numpy(), weff)


@pytest.mark.parametrize("batch", [5, 16])
def test_gemv_group_matches_single_calls(lib, gemv_variant, batch):
    """One grouped launch over projections of different shapes equals the
    oracle.  The long-K problems run as 8-row units, the shortest as 16-row
    units, so both unit shapes are covered, with one and two token tiles."""
    shapes = [(264, 2048), (8, 896), (520, 11008), (136, 4864)]
    probs, refs = [], []
    for i, (d_out, d_in) in enumerate(shapes):
        w = synth.trimodal_weight(d_out, d_in, seed=30, tensor_id=i)
        weff, gamma, _ = oracle.effective_weight(synth.bits(w), 6, 8)
        x = synth.activations(batch, d_in, seed=30, tensor_id=100 + i)
        xq, amax = oracle.act_quant(synth.bits(x))
        nbytes = lib.sbl_packed_bytes(d_out, d_in, 6, 8)
        packed = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
        lib.sbl_pack(torch.from_numpy(weff).cuda(), d_out, d_in, 6, 8, packed, nbytes)
        Y = torch.empty(batch, d_out, dtype=torch.float32, device="cuda")
        g = torch.tensor([float(gamma)], dtype=torch.float32, device="cuda")
        probs.append((packed, torch.from_numpy(xq).cuda(), torch.from_numpy(amax).cuda(), g, Y, d_in, d_out))
        refs.append(oracle.forward_out(oracle.forward_acc(xq, weff), gamma, amax))
    lib.sbl_gemv_packed_group(probs, batch, 6, 8)
    lib.sbl_check()
    for (_, _, _, _, Y, _, _), ref in zip(probs, refs):
        assert np.array_equal(Y.cpu().numpy(), ref)


@pytest.mark.parametrize("variant", [0, 1])
def test_forward_group_matches_single_calls(lib, variant):
    """One grouped launch over products of different shapes (ragged tokens,
    rows and d_in; a long-K product; an empty product and a zero-token one)
    gives each product's exact int32 sums and outputs."""
    T = 300
    shapes = [(264, 2048), (8, 896), (520, 11008), (136, 4368), (2048, 256), (40, 0), (16, 64)]
    toks = [T, T, T, 129, T, T, 0]
    probs, refs = [], []
    for i, ((d_out, d_in), t) in enumerate(zip(shapes, toks)):
        w = synth.trimodal_weight(d_out, max(d_in, 16), seed=47, tensor_id=i)[:, :d_in].contiguous()
        x = synth.activations(t, max(d_in, 16), seed=47, tensor_id=100 + i)[:, :d_in].contiguous()
        weff, gamma, _ = oracle.effective_weight(synth.bits(w), 6, 8) if d_in else (
            np.zeros((d_out, 0), np.int8), np.float32(0.0), None)
        xq, amax = oracle.act_quant(synth.bits(x)) if d_in else (np.zeros((t, 0), np.int8), np.ones(t, np.float32))
        Y = torch.full((t, d_out), float("nan"), dtype=torch.float32, device="cuda")
        acc = torch.full((t, d_out), 7, dtype=torch.int32, device="cuda")
        g = torch.tensor([float(gamma)], dtype=torch.float32, device="cuda")
        xq_d = torch.from_numpy(xq).cuda() if d_in else torch.empty((max(t, 1), 16), dtype=torch.int8, device="cuda")
        w_d = torch.from_numpy(weff).cuda() if d_in else torch.empty((d_out, 16), dtype=torch.int8, device="cuda")
        probs.append((xq_d, torch.from_numpy(amax).cuda() if t else torch.ones(1, device="cuda"), w_d, g, t, d_in,
                      d_out, Y, acc))
        racc = oracle.forward_acc(xq, weff) if d_in else np.zeros((t, d_out), np.int32)
        refs.append((racc, oracle.forward_out(racc, gamma, amax) if t else np.zeros((0, d_out), np.float32)))
    lib.sbl_set_gemm_variant(variant)
    try:
        lib.sbl_forward_group(probs)
        lib.sbl_check()
    finally:
        lib.sbl_set_gemm_variant(0)
    for (_, _, _, _, t, d_in, d_out, Y, acc), (racc, ry) in zip(probs, refs):
        assert np.array_equal(acc.cpu().numpy(), racc), (t, d_in, d_out)
        if d_in:
            assert np.array_equal(Y.cpu().numpy(), ry), (t, d_in, d_out)
        else:
            assert not Y.cpu().numpy().any()


@pytest.mark.parametrize("T,d_out,d_in", [(64, 512, 11008), (300, 264, 4368), (512, 2048, 2048), (17, 8, 16384)])
@pytest.mark.parametrize("variant", [0, 1])
def test_forward_split_k_exact(lib, T, d_out, d_in, variant):
    """Short token batches with long rows: the CTA-pair forward splits K
    (fewer output tiles than CTA pairs) and its splits add exact integer
    sums that a finalize pass scales; y and the int32 accumulators must equal
    the oracle's exactly, as for the unsplit one-CTA kernel."""
    w = synth.trimodal_weight(d_out, d_in, seed=46, tensor_id=d_in)
    x = synth.activations(T, d_in, seed=46, tensor_id=100 + T, outlier_frac=0.01)
    weff, gamma, _ = oracle.effective_weight(synth.bits(w), 6, 8)
    xq, amax = oracle.act_quant(synth.bits(x))
    Y = torch.full((T, d_out), float("nan"), dtype=torch.float32, device="cuda")
    acc = torch.empty(T, d_out, dtype=torch.int32, device="cuda")
    g = torch.tensor([float(gamma)], dtype=torch.float32, device="cuda")
    lib.sbl_set_gemm_variant(variant)
    try:
        lib.sbl_forward(torch.from_numpy(xq).cuda(), torch.from_numpy(amax).cuda(), torch.from_numpy(weff).cuda(),
                        g, T, d_in, d_out, Y, acc)
        lib.sbl_check()
    finally:
        lib.sbl_set_gemm_variant(0)
    racc = oracle.forward_acc(xq, weff)
    assert np.array_equal(acc.cpu().numpy(), racc)
    assert np.array_equal(Y.cpu().numpy(), oracle.forward_out(racc, gamma, amax))


@pytest.mark.parametrize("T,d_out,d_in,N,M", [
    (64, 256, 256, 6, 8), (300, 264, 2064, 6, 8), (129, 520, 1040, 2, 4), (257, 136, 400, 4, 8),
    (100, 392, 2048, 8, 8), (33, 8, 4864, 1, 8), (77, 128, 272, 3, 4),
])
def test_forward_from_packed_matches_oracle(lib, T, d_out, d_in, N, M):
    """The forward that expands the packed weight in shared memory gives the
    oracle's int32 accumulators and outputs (and so sbl_forward's)."""
    w = synth.trimodal_weight(d_out, d_in, seed=40, tensor_id=T)
    x = synth.activations(T, d_in, seed=40, tensor_id=100 + T, outlier_frac=0.01)
    weff, gamma, _ = oracle.effective_weight(synth.bits(w), N, M)
    xq, amax = oracle.act_quant(synth.bits(x))
    nbytes = lib.sbl_packed_bytes(d_out, d_in, N, M)
    packed = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    lib.sbl_pack(torch.from_numpy(weff).cuda(), d_out, d_in, N, M, packed, nbytes)
    Y = torch.empty(T, d_out, dtype=torch.float32, device="cuda")
    acc = torch.empty(T, d_out, dtype=torch.int32, device="cuda")
    g = torch.tensor([float(gamma)], dtype=torch.float32, device="cuda")
    lib.sbl_forward_packed(torch.from_numpy(xq).cuda(), torch.from_numpy(amax).cuda(), packed, g, T, d_in, d_out, N,
                           M, Y, acc)
    lib.sbl_check()
    racc = oracle.forward_acc(xq, weff)
    assert np.array_equal(acc.cpu().numpy(), racc)
    assert np.array_equal(Y.cpu().numpy(), oracle.forward_out(racc, gamma, amax))


@pytest.mark.parametrize("d_out,d_in,N,M", [
    (8, 16, 6, 8), (264, 2064, 6, 8), (136, 400, 2, 4), (520, 1040, 8, 8), (72, 4864, 4, 8), (40, 272, 3, 8),
    (16, 112, 1, 4), (24, 208, 3, 4),
])
def test_unpack_restores_weff(lib, d_out, d_in, N, M):
    """sbl_unpack of sbl_pack gives back W_eff bit for bit (and the oracle's
    unpack of the same bytes), including runs cut short by d_in % 64."""
    w = synth.trimodal_weight(d_out, d_in, seed=70, tensor_id=d_in)
    weff, _, _ = oracle.effective_weight(synth.bits(w), N, M)
    nbytes = lib.sbl_packed_bytes(d_out, d_in, N, M)
    packed = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    lib.sbl_pack(torch.from_numpy(weff).cuda(), d_out, d_in, N, M, packed, nbytes)
    out = torch.full((d_out, d_in), 77, dtype=torch.int8, device="cuda")
    lib.sbl_unpack(packed, d_out, d_in, N, M, out)
    lib.sbl_check()
    assert np.array_equal(out.cpu().numpy(), weff)
    assert np.array_equal(oracle.unpack(packed.cpu().numpy(), d_out, d_in, N, M), weff)


@pytest.mark.parametrize("d_out,d_in,N,M", [(8, 16, 6, 8), (264, 2064, 6, 8), (136, 400, 2, 4), (40, 272, 8, 8)])
def test_pack_dense2_bit_exact(lib, d_out, d_in, N, M):
    w = synth.trimodal_weight(d_out, d_in, seed=80, tensor_id=d_in)
    weff, _, _ = oracle.effective_weight(synth.bits(w), N, M)
    nbytes = lib.sbl_dense2_bytes(d_out, d_in)
    out = torch.full((nbytes,), 0xAB, dtype=torch.uint8, device="cuda")
    lib.sbl_pack_dense2(torch.from_numpy(weff).cuda(), d_out, d_in, out, nbytes)
    lib.sbl_check()
    assert np.array_equal(out.cpu().numpy(), oracle.pack_dense2(weff))


@pytest.mark.parametrize("batch", [1, 5, 16])
def test_gemv_dense2_group_matches_oracle(lib, gemv_variant, batch):
    """Decode GEMV on the dense 2-bit layout: one grouped launch over shapes
    that give 16- and 8-row units and a ragged last K tile."""
    shapes = [(264, 2048), (8, 896), (520, 11008), (136, 4864)]
    probs, refs = [], []
    for i, (d_out, d_in) in enumerate(shapes):
        w = synth.trimodal_weight(d_out, d_in, seed=81, tensor_id=i)
        weff, gamma, _ = oracle.effective_weight(synth.bits(w), 6, 8)
        x = synth.activations(batch, d_in, seed=81, tensor_id=100 + i)
        xq, amax = oracle.act_quant(synth.bits(x))
        nbytes = lib.sbl_dense2_bytes(d_out, d_in)
        d2 = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
        lib.sbl_pack_dense2(torch.from_numpy(weff).cuda(), d_out, d_in, d2, nbytes)
        Y = torch.full((batch, d_out), float("nan"), dtype=torch.float32, device="cuda")
        g = torch.tensor([float(gamma)], dtype=torch.float32, device="cuda")
        probs.append((d2, torch.from_numpy(xq).cuda(), torch.from_numpy(amax).cuda(), g, Y, d_in, d_out))
        refs.append(oracle.forward_out(oracle.forward_acc(xq, weff), gamma, amax))
    lib.sbl_gemv_dense2_group(probs, batch)
    lib.sbl_check()
    for (_, _, _, _, Y, _, _), ref in zip(probs, refs):
        assert np.array_equal(Y.cpu().numpy(), ref)


@pytest.mark.parametrize("batch", [1, 2, 8])
def test_gemv_dense2_group_shared_activations(lib, batch):
    """Projections that read the same activations (as q, k and v do) in one
    grouped launch: the kernel stages each activation tensor in shared memory
    once per block when it fits and shares it between those problems, and
    reads the rest (here the 11008-wide input at batch > 1) from global
    memory; every output must still be the oracle's, bit for bit."""
    inputs = {"a": 2048, "b": 11008, "c": 4864}
    shapes = [("a", 264), ("a", 40), ("a", 1040), ("b", 136), ("c", 520), ("c", 8)]
    xs = {}
    for j, (name, d_in) in enumerate(inputs.items()):
        x = synth.activations(batch, d_in, seed=84, tensor_id=100 + j)
        xq, amax = oracle.act_quant(synth.bits(x))
        xs[name] = (xq, amax, torch.from_numpy(xq).cuda(), torch.from_numpy(amax).cuda())
    probs, refs = [], []
    for i, (name, d_out) in enumerate(shapes):
        d_in = inputs[name]
        w = synth.trimodal_weight(d_out, d_in, seed=84, tensor_id=i)
        weff, gamma, _ = oracle.effective_weight(synth.bits(w), 6, 8)
        nbytes = lib.sbl_dense2_bytes(d_out, d_in)
        d2 = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
        lib.sbl_pack_dense2(torch.from_numpy(weff).cuda(), d_out, d_in, d2, nbytes)
        Y = torch.full((batch, d_out), float("nan"), dtype=torch.float32, device="cuda")
        g = torch.tensor([float(gamma)], dtype=torch.float32, device="cuda")
        xq, amax, xq_d, amax_d = xs[name]
        probs.append((d2, xq_d, amax_d, g, Y, d_in, d_out))
        refs.append(oracle.forward_out(oracle.forward_acc(xq, weff), gamma, amax))
    lib.sbl_gemv_dense2_group(probs, batch)
    lib.sbl_check()
    for (_, _, _, _, Y, _, _), ref in zip(probs, refs):
        assert np.array_equal(Y.cpu().numpy(), ref)


@pytest.mark.parametrize("N,M", [(1, 8), (3, 8), (5, 8), (7, 8), (1, 4), (3, 4), (4, 8)])
@pytest.mark.parametrize("d_out,d_in", [(8, 16), (24, 48), (40, 2320), (136, 4368)])
def test_gemv_every_k_and_ragged_rows(lib, gemv_variant, N, M, d_out, d_in):
    """Every slot count K = 8N/M, rows that do not fill a 16-row block, k
    ranges shorter than one 256-weight step or not a multiple of 64 weights,
    and rows cut into several k slices (d_in > 2048)."""
    if d_in % M:
        pytest.skip("d_in must be a multiple of M")
    batch = 3
    w = synth.trimodal_weight(d_out, d_in, seed=82, tensor_id=d_in + N)
    weff, gamma, _ = oracle.effective_weight(synth.bits(w), N, M)
    x = synth.activations(batch, d_in, seed=82, tensor_id=100 + d_in)
    xq, amax = oracle.act_quant(synth.bits(x))
    nbytes = lib.sbl_packed_bytes(d_out, d_in, N, M)
    packed = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    lib.sbl_pack(torch.from_numpy(weff).cuda(), d_out, d_in, N, M, packed, nbytes)
    Y = torch.full((batch, d_out), float("nan"), dtype=torch.float32, device="cuda")
    g = torch.tensor([float(gamma)], dtype=torch.float32, device="cuda")
    lib.sbl_gemv_packed(torch.from_numpy(xq).cuda(), torch.from_numpy(amax).cuda(), batch, packed, g, d_in, d_out,
                        N, M, Y)
    lib.sbl_check()
    ref = oracle.forward_out(oracle.forward_acc(xq, weff), gamma, amax)
    assert np.array_equal(Y.cpu().numpy(), ref)


@pytest.mark.parametrize("batch", [2, 11])
def test_gemv_many_split_rows_reuse_slots(lib, batch):
    """Rows of 4352 weights are cut into three k slices whose partial sums
    meet in shared-memory slots; 28416 rows give every block about a dozen
    such row blocks, more than its eight slots, so the slots are reused."""
    d_out, d_in = 28416, 4352
    w = synth.normal_weight(d_out, d_in, seed=83)
    weff, gamma, _ = oracle.effective_weight(synth.bits(w), 6, 8)
    x = synth.activations(batch, d_in, seed=83, tensor_id=100)
    xq, amax = oracle.act_quant(synth.bits(x))
    nbytes = lib.sbl_packed_bytes(d_out, d_in, 6, 8)
    packed = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    lib.sbl_pack(torch.from_numpy(weff).cuda(), d_out, d_in, 6, 8, packed, nbytes)
    Y = torch.full((batch, d_out), float("nan"), dtype=torch.float32, device="cuda")
    g = torch.tensor([float(gamma)], dtype=torch.float32, device="cuda")
    lib.sbl_gemv_packed(torch.from_numpy(xq).cuda(), torch.from_numpy(amax).cuda(), batch, packed, g, d_in, d_out,
                        6, 8, Y)
    lib.sbl_check()
    ref = oracle.forward_out(oracle.forward_acc(xq, weff), gamma, amax)
    assert np.array_equal(Y.cpu().numpy(), ref)


@pytest.mark.parametrize("T,d_in", [(1, 16), (64, 896), (333, 2048), (40, 4864), (17, 11008), (9, 17408)])
@pytest.mark.parametrize("with_xn", [True, False])
def test_rmsnorm_act_quant_matches_oracle(lib, T, d_in, with_xn):
    """Q_a(RMSNorm(x)) in one kernel: the normalised bf16 row, the int8
    codes and amax bit for bit against the oracle; d_in = 17408 exercises
    the rows longer than the register-resident part."""
    x = synth.activations(T, d_in, seed=90, tensor_id=d_in, outlier_frac=0.01)
    if T > 2:
        x[1] = 0.0  # an all-zero token
    g = (torch.rand(d_in, generator=torch.Generator().manual_seed(d_in)) + 0.5).to(torch.bfloat16)
    eps = 1e-6
    Xn = torch.empty(T, d_in, dtype=torch.bfloat16, device="cuda") if with_xn else None
    Xq = torch.empty(T, d_in, dtype=torch.int8, device="cuda")
    amax = torch.empty(T, dtype=torch.float32, device="cuda")
    lib.sbl_rmsnorm_act_quant(x.cuda(), g.cuda(), eps, T, d_in, Xn, Xq, amax)
    lib.sbl_check()
    rxn, rxq, ramax = oracle.rms_norm_act_quant(synth.bits(x), synth.bits(g), eps)
    if with_xn:
        assert np.array_equal(synth.bits(Xn.cpu()), rxn)
    assert np.array_equal(Xq.cpu().numpy(), rxq)
    assert np.array_equal(amax.cpu().numpy(), ramax)


@pytest.mark.parametrize("d_out,d_in,N,M", [(256, 256, 6, 8), (264, 2064, 2, 4), (40, 400, 4, 8), (8, 16, 3, 4)])
def test_mask_from_quantised_matches_oracle(lib, d_out, d_in, N, M):
    """Ablation: the mask from |W_q| (flags = SBL_MASK_FROM_QUANTISED) gives
    the oracle's mask, gamma and W_eff bit for bit; flags = 0 is the default."""
    w = synth.trimodal_weight(d_out, d_in, seed=95, tensor_id=d_in)
    wb = synth.bits(w)
    W = w.cuda()
    ws_bytes = lib.sbl_mask_quant_workspace_bytes(d_out, d_in)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    for flags, ref_fn in ((lib.SBL_MASK_FROM_QUANTISED, oracle.effective_weight_mask_from_quantised),
                          (0, oracle.effective_weight)):
        we = torch.empty(d_out, d_in, dtype=torch.int8, device="cuda")
        bits = torch.empty(d_out, d_in // 8, dtype=torch.uint8, device="cuda")
        g = torch.empty(1, dtype=torch.float32, device="cuda")
        lib.sbl_mask_quant_ex(W, d_out, d_in, N, M, flags, we, None, bits, g, ws, ws_bytes)
        lib.sbl_check()
        rweff, rgamma, rkeep = ref_fn(wb, N, M)
        assert g.item() == float(rgamma)
        assert np.array_equal(we.cpu().numpy(), rweff)
        assert np.array_equal(_unpack_mask(bits.cpu().numpy()), rkeep)


def test_mask_grad_zeroes_masked_positions(lib):
    """Ablation without the Dual-STE: dW (.) M after sbl_backward, exact
    against the unmasked GPU dW and within the backward tolerance of the
    oracle's masked gradient."""
    T, d_out, d_in = 96, 264, 400
    w = synth.trimodal_weight(d_out, d_in, seed=96)
    x = synth.activations(T, d_in, seed=96, tensor_id=1)
    dy = synth.grad_output(T, d_out, seed=96, tensor_id=2)
    g = Layer(lib, w, x, dy, 6, 8)
    dw = g.dW.clone()
    lib.sbl_mask_grad(g.dW, g.L.mask_bits, d_out, d_in)
    lib.sbl_check()
    keep = _unpack_mask(g.L.mask_bits.cpu().numpy())
    assert np.array_equal(g.dW.cpu().numpy(), np.where(keep, dw.cpu().numpy(), 0.0))
    ref = oracle.masked_grad(oracle.backward_dw(synth.bits(dy), synth.bits(x)), keep)
    check_bwd(g.dW.cpu().numpy(), ref, abs_dw(synth.bits(dy), synth.bits(x)) * keep, "dW (.) M")
