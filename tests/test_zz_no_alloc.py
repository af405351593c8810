"""sbl_mask_quant_noalloc: the weight step for callers that cannot allocate
device memory when it runs (processes that reserve their whole device-memory
budget at start-up, or plugin hosts that pass only inputs and outputs).

It must give exactly what sbl_mask_quant gives with a caller-supplied
workspace, on consecutive calls that reuse the one static scratch array.
This file is collected last so that a failure here leaves every other test
already run; it also passes when run alone in a fresh process.
"""
import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu


def _outputs(d_out, d_in):
    return (torch.empty(d_out, d_in, dtype=torch.int8, device="cuda"),
            torch.empty(d_out, d_in, dtype=torch.bfloat16, device="cuda"),
            torch.empty(d_out, d_in // 8, dtype=torch.uint8, device="cuda"),
            torch.empty(1, dtype=torch.float32, device="cuda"))


def test_noalloc_matches_workspace_call_on_two_calls_in_a_row(lib):
    assert lib.sbl_mask_quant_noalloc_scratch_bytes() == 7040
    # Two different weights (and shapes) back to back: the second call must not
    # see anything the first left in the shared scratch.
    # The third weight has d_out * d_in / 8 = 530,448 eight-weight vectors:
    # not a multiple of 256, and far more than the gamma pass's grid of at most
    # 592 blocks of 256 threads covers in one sweep.  Its magnitudes (and so
    # its ternary threshold) differ from the call before it.
    cases = [(synth.trimodal_weight(1024, 2048, seed=21, tensor_id=0), 6, 8),
             (synth.with_boundary_ties(synth.normal_weight(264, 528, seed=22, tensor_id=1), 2, 4, seed=22), 2, 4),
             (synth.normal_weight(2056, 2064, seed=23, tensor_id=2) * 3, 6, 8)]
    for k, (w_cpu, N, M) in enumerate(cases):
        W = w_cpu.cuda()
        d_out, d_in = W.shape
        ref = _outputs(d_out, d_in)
        ws_bytes = lib.sbl_mask_quant_workspace_bytes(d_out, d_in)
        ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
        lib.sbl_mask_quant(W, d_out, d_in, N, M, ref[0], ref[1], ref[2], ref[3], ws, ws_bytes)
        got = _outputs(d_out, d_in)
        lib.sbl_mask_quant_noalloc(W, d_out, d_in, N, M, got[0], got[1], got[2], got[3])
        lib.sbl_check()
        for a, b in zip(ref, got):
            assert torch.equal(a, b)
        assert got[3].item() > 0.0
        if k == 2:
            weff, gamma, keep = oracle.effective_weight(synth.bits(w_cpu), N, M)
            assert got[3].item() == float(gamma)
            assert np.array_equal(got[0].cpu().numpy(), weff)
            bits = np.unpackbits(got[2].cpu().numpy(), axis=1, bitorder="little").astype(bool)
            assert np.array_equal(bits, keep)


def test_noalloc_rejects_oversized_weight(lib):
    """W with 2^32 or more elements is refused before anything is launched."""
    import semi_structured_sparsity_step_b200._binding as B
    cl = B.load()
    buf = torch.empty(64, dtype=torch.uint8, device="cuda")
    p = buf.data_ptr()
    assert cl.sbl_mask_quant_noalloc(p, 65536, 65536, 6, 8, p, None, None, p, None) == 2
    lib.sbl_check()
