"""GPU parity of the 2:4 sparse tensor-core path through the C ABI.

sbl_compress24 must give the oracle's compressed bytes bit for bit, and
sbl_forward_sparse24 the oracle's int32 accumulators and fp32 outputs bit for
bit (the same integers as the dense product, the same fp32 epilogue).
Shapes cover several 256 x 224 tiles with ragged edges in every dimension
(tokens, weight rows, d_in not a multiple of 256), single tokens, groups with
fewer than two nonzeros, all-zero rows, and a group with too many nonzeros.
"""
import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu

SHAPES = [
    (64, 256, 256), (300, 264, 2064), (129, 520, 1040), (1, 8, 16), (225, 136, 400),
    (448, 512, 512), (97, 1032, 272), (513, 256, 4864),
]


def _weff24(d_out, d_in, seed):
    w = synth.trimodal_weight(d_out, d_in, seed=seed, tensor_id=d_out + d_in)
    weff, gamma, _ = oracle.effective_weight(synth.bits(w), 2, 4)
    return weff, gamma


def _compress(lib, weff):
    d_out, d_in = weff.shape
    nbytes = lib.sbl_compress24_bytes(d_out, d_in)
    out = torch.full((nbytes,), 0xAB, dtype=torch.uint8, device="cuda")
    lib.sbl_compress24(torch.from_numpy(weff).cuda(), d_out, d_in, out, nbytes)
    return out, nbytes


@pytest.mark.parametrize("T,d_out,d_in", SHAPES)
def test_compress24_bytes_bit_exact(lib, T, d_out, d_in):
    weff, _ = _weff24(d_out, d_in, seed=60)
    out, nbytes = _compress(lib, weff)
    lib.sbl_check()
    ref = oracle.compress24(weff)
    assert nbytes == ref.size
    assert np.array_equal(out.cpu().numpy(), ref)


@pytest.mark.parametrize("T,d_out,d_in", SHAPES)
def test_forward_sparse24_matches_oracle(lib, T, d_out, d_in):
    weff, gamma = _weff24(d_out, d_in, seed=61)
    if d_out >= 16:
        weff[3] = 0                                  # an all-zero weight row
        weff[5, : d_in // 2] = 0                     # groups with no nonzero
    x = synth.activations(T, d_in, seed=61, tensor_id=100 + T, outlier_frac=0.01)
    xq, amax = oracle.act_quant(synth.bits(x))
    w24, _ = _compress(lib, weff)
    Y = torch.full((T, d_out), float("nan"), dtype=torch.float32, device="cuda")
    acc = torch.full((T, d_out), -7, dtype=torch.int32, device="cuda")
    g = torch.tensor([float(gamma)], dtype=torch.float32, device="cuda")
    lib.sbl_forward_sparse24(torch.from_numpy(xq).cuda(), torch.from_numpy(amax).cuda(), w24, g, T, d_in, d_out, Y,
                             acc)
    lib.sbl_check()
    racc = oracle.forward_acc(xq, weff)
    assert np.array_equal(acc.cpu().numpy(), racc)
    assert np.array_equal(Y.cpu().numpy(), oracle.forward_out(racc, gamma, amax))
    # the oracle's own sparse product from the compressed bytes agrees too
    assert np.array_equal(oracle.forward_acc_sparse24(xq, oracle.compress24(weff), d_out, d_in), racc)


def test_forward_sparse24_equals_dense_forward(lib):
    """Same inputs through sbl_forward (dense int8 MMA) and
    sbl_forward_sparse24: identical accumulators and outputs."""
    T, d_out, d_in = 1000, 768, 1536
    weff, gamma = _weff24(d_out, d_in, seed=62)
    x = synth.activations(T, d_in, seed=62, tensor_id=7)
    xq, amax = oracle.act_quant(synth.bits(x))
    Xq, A = torch.from_numpy(xq).cuda(), torch.from_numpy(amax).cuda()
    g = torch.tensor([float(gamma)], dtype=torch.float32, device="cuda")
    w24, _ = _compress(lib, weff)
    Yd = torch.empty(T, d_out, dtype=torch.float32, device="cuda")
    Ys = torch.empty_like(Yd)
    ad = torch.empty(T, d_out, dtype=torch.int32, device="cuda")
    asp = torch.empty_like(ad)
    lib.sbl_forward(Xq, A, torch.from_numpy(weff).cuda(), g, T, d_in, d_out, Yd, ad)
    lib.sbl_forward_sparse24(Xq, A, w24, g, T, d_in, d_out, Ys, asp)
    lib.sbl_check()
    assert torch.equal(ad, asp)
    assert torch.equal(Yd, Ys)


def test_compress24_rejects_three_nonzeros(lib):
    weff = np.zeros((8, 16), dtype=np.int8)
    weff[2, 4:7] = 1                                  # three nonzeros in one group
    out, nbytes = _compress(lib, weff)
    with pytest.raises(lib.SblError) as e:
        lib.sbl_check()
    assert e.value.status == 8
    lib.sbl_check()  # the latched error was cleared


def test_sparse24_argument_errors(lib):
    z = torch.zeros(64, dtype=torch.int8, device="cuda")
    with pytest.raises(lib.SblError) as e:
        lib.sbl_compress24(z, 8, 12, z, 1 << 20)      # d_in % 16 != 0
    assert e.value.status == 2
    with pytest.raises(lib.SblError) as e:
        lib.sbl_compress24(z, 8, 16, z, 16)           # buffer too small
    assert e.value.status == 5
    assert lib.sbl_compress24_bytes(8, 12) == 0
