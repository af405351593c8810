"""CPU-side checks of the C-ABI library: it loads, exports every entry point
that include/sbl.h declares, and rejects bad arguments on the host before
touching CUDA (no GPU is needed for any of this)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sbl.h")


@pytest.fixture(scope="module")
def cl():
    from semi_structured_sparsity_step_b200 import build
    build.build()
    from semi_structured_sparsity_step_b200 import _binding
    return _binding.load()


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(sbl_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_core_entry_points():
    names = _declared()
    for n in ["sbl_mask_quant", "sbl_act_quant", "sbl_forward", "sbl_backward", "sbl_pack", "sbl_gemv_packed",
              "sbl_check", "sbl_status_string", "sbl_packed_bytes"]:
        assert n in names


def test_every_declared_symbol_is_exported(cl):
    from semi_structured_sparsity_step_b200._binding import SIGNATURES
    for n in _declared():
        assert hasattr(cl, n), n
        assert n in SIGNATURES, n


def test_status_strings(cl):
    from semi_structured_sparsity_step_b200 import _binding as B
    for code, name in B.STATUS.items():
        assert B.sbl_status_string(code) == name
    assert B.sbl_status_string(99) == "SBL_ERR_UNKNOWN"


def test_host_validation_without_gpu(cl):
    al = 1 << 12  # fake, 16-byte aligned addresses: never dereferenced on these paths
    # bad N:M
    assert cl.sbl_mask_quant(al, 8, 16, 0, 8, al, None, None, al, al * 4, 1 << 20, None) == 1
    assert cl.sbl_mask_quant(al, 8, 16, 5, 6, al, None, None, al, al * 4, 1 << 20, None) == 1
    assert cl.sbl_mask_quant(al, 8, 16, 9, 8, al, None, None, al, al * 4, 1 << 20, None) == 1
    # shapes
    assert cl.sbl_mask_quant(al, 8, 24, 6, 8, al, None, None, al, al * 4, 1 << 20, None) == 2
    assert cl.sbl_mask_quant(al, 12, 16, 6, 8, al, None, None, al, al * 4, 1 << 20, None) == 2
    assert cl.sbl_act_quant(al, -1, 16, al, al, None) == 2
    assert cl.sbl_forward(al, al, al, al, 4, 20, 8, al, None, None) == 2
    assert cl.sbl_gemv_packed(al, al, 17, al, al, 16, 8, 6, 8, al, None) == 2
    # null and misaligned pointers
    assert cl.sbl_mask_quant(None, 8, 16, 6, 8, al, None, None, al, al * 4, 1 << 20, None) == 1
    assert cl.sbl_act_quant(al + 8, 4, 16, al, al, None) == 3
    assert cl.sbl_forward(al, al, al + 4, al, 4, 16, 8, al, None, None) == 3
    assert cl.sbl_mask_quant(al, 8, 16, 6, 8, al, None, None, al, al + 16, 1 << 20, None) == 3
    # workspace and packed buffer too small
    assert cl.sbl_mask_quant(al, 8, 16, 6, 8, al, None, None, al, al * 4, 8, None) == 5
    assert cl.sbl_pack(al, 8, 16, 6, 8, al, 4, None) == 5
    # optimizer step: bad hyperparameters, flips without a mask, misalignment
    def adamw(step=1, lr=1e-3, b1=0.9, b2=0.95, eps=1e-5, wd=0.1, sq=None, mn=1.0, bits=al, flips=None, W32=None,
              d_in=16, ws=1 << 20):
        return cl.sbl_adamw_step(al, W32, al, al, al, 8, d_in, 6, 8, lr, b1, b2, eps, wd, step, sq, mn, al, None,
                                 bits, al, flips, al * 4, ws, None)
    assert adamw(step=0) == 1
    assert adamw(lr=-1.0) == 1
    assert adamw(lr=float("nan")) == 1
    assert adamw(b1=1.0) == 1
    assert adamw(b2=-0.1) == 1
    assert adamw(eps=0.0) == 1
    assert adamw(wd=-0.5) == 1
    assert adamw(sq=al, mn=0.0) == 1
    assert adamw(bits=None, flips=al) == 1
    assert adamw(d_in=24) == 2
    assert adamw(W32=al + 8) == 3
    assert adamw(sq=al + 4) == 3
    assert adamw(ws=8) == 5
    assert cl.sbl_grad_sqnorm(al, 16, None, al * 4, 1 << 20, None) == 1
    assert cl.sbl_grad_sqnorm(al + 4, 16, al, al * 4, 1 << 20, None) == 3
    assert cl.sbl_grad_sqnorm(al, 16, al, al * 4, 8, None) == 5
    assert cl.sbl_grad_sqnorm(None, 0, al, al * 4, 1 << 20, None) == 0
    # empty work is a no-op that needs no device
    assert cl.sbl_act_quant(al, 0, 16, al, al, None) == 0
    assert cl.sbl_forward(al, al, al, al, 0, 16, 8, al, None, None) == 0


def test_group_and_variant_validation_without_gpu(cl):
    """Grouped calls check every descriptor on the host; the kernel-variant
    selectors accept only their documented values."""
    from semi_structured_sparsity_step_b200 import _binding as B
    al = 1 << 12
    assert cl.sbl_set_gemm_variant(2) == 1
    assert cl.sbl_set_gemm_variant(-1) == 1
    assert cl.sbl_set_gemv_variant(3) == 1
    assert cl.sbl_set_gemv_variant(-1) == 1
    assert cl.sbl_set_gemm_variant(0) == 0 and cl.sbl_set_gemv_variant(0) == 0

    def fwd(*problems):
        arr = (B.ForwardProblem * max(1, len(problems)))()
        for i, q in enumerate(problems):
            arr[i] = B.ForwardProblem(*q)
        return cl.sbl_forward_group(ctypes.cast(arr, ctypes.c_void_p), len(problems), None)

    good = (al, al, al, al, 4, 16, 8, al, None)
    assert cl.sbl_forward_group(None, -1, None) == 1
    assert cl.sbl_forward_group(None, 1, None) == 1
    assert cl.sbl_forward_group(None, 0, None) == 0
    assert fwd(good, (al, al, al, al, 4, 20, 8, al, None)) == 2   # d_in % 16 in the second problem
    assert fwd(good, (al, al, al, al, -1, 16, 8, al, None)) == 2  # negative T
    assert fwd(good, (al, None, al, al, 4, 16, 8, al, None)) == 1
    assert fwd(good, (al, al, al, al + 2, 4, 16, 8, al, None)) == 3  # gamma not 4-byte aligned
    assert fwd((al, al, al, al, 0, 16, 8, al, None)) == 0         # only empty work: no device needed

    def gemv(batch, *problems, N=6, M=8):
        arr = (B.GemvProblem * max(1, len(problems)))()
        for i, q in enumerate(problems):
            arr[i] = B.GemvProblem(*q)
        return cl.sbl_gemv_packed_group(arr, len(problems), batch, N, M, None)

    gp = (al, al, al, al, al, 16, 8)
    assert cl.sbl_gemv_dense2_group(None, 1, 17, None) == 2
    assert cl.sbl_gemv_dense2_group(None, 1, 1, None) == 1
    assert gemv(17, gp) == 2
    assert gemv(1, gp, N=5, M=6) == 1
    assert gemv(1, gp, (al, al, al, al, al, 24, 8)) == 2  # d_in % 16
    assert gemv(1, gp, (None, al, al, al, al, 16, 8)) == 1
    assert gemv(1, gp, (al + 8, al, al, al, al, 16, 8)) == 3
    assert gemv(0, gp) == 0


def test_packed_bytes_matches_format(cl):
    import oracle
    for (d_out, d_in, N, M) in [(8, 16, 6, 8), (24, 272, 2, 4), (2048, 11008, 6, 8), (16, 64, 8, 8)]:
        assert cl.sbl_packed_bytes(d_out, d_in, N, M) == oracle.packed_layout(d_out, d_in, N, M)[2]
    assert cl.sbl_packed_bytes(8, 24, 6, 8) == 0  # invalid shape


def test_remaining_entry_points_validate_on_the_host(cl):
    """Every other entry point rejects bad flags, N:M, shapes, null or
    misaligned pointers and short buffers before it needs a device, and
    treats empty work as done."""
    al = 1 << 12
    ws = 1 << 20
    # failure-detection self-test: the wait limit must be 1 us .. 1 s
    assert cl.sbl_selftest_wait_timeout(0, None) == 1
    assert cl.sbl_selftest_wait_timeout(2000000, None) == 1
    # mask from the quantised weight: unknown flag bits
    assert cl.sbl_mask_quant_ex(al, 8, 16, 6, 8, 2, al, None, None, al, al * 4, ws, None) == 1
    # dW (.) M
    assert cl.sbl_mask_grad(al, al, 8, 20, None) == 2
    assert cl.sbl_mask_grad(None, al, 8, 16, None) == 1
    assert cl.sbl_mask_grad(al + 4, al, 8, 16, None) == 3
    assert cl.sbl_mask_grad(al, al, 0, 16, None) == 0
    # forward from the packed format
    assert cl.sbl_forward_packed(al, al, al, al, 4, 16, 8, 5, 6, al, None, None) == 1
    assert cl.sbl_forward_packed(al, al, al, al, -1, 16, 8, 6, 8, al, None, None) == 2
    assert cl.sbl_forward_packed(al, al, None, al, 4, 16, 8, 6, 8, al, None, None) == 1
    assert cl.sbl_forward_packed(al, al, al, al, 0, 16, 8, 6, 8, al, None, None) == 0
    # unpack
    assert cl.sbl_unpack(al, 8, 16, 9, 8, al, None) == 1
    assert cl.sbl_unpack(al, 8, 16, 6, 8, None, None) == 1
    assert cl.sbl_unpack(al, 8, 16, 6, 8, al + 8, None) == 3
    # 2:4 compression and the sparse forward
    assert cl.sbl_compress24(al, 8, 16, None, 1 << 20, None) == 1
    assert cl.sbl_compress24(al, 8, 16, al, 16, None) == 5
    assert cl.sbl_forward_sparse24(al, al, al, al, -1, 16, 8, al, None, None) == 2
    assert cl.sbl_forward_sparse24(al, al, al, al + 2, 4, 16, 8, al, None, None) == 3
    assert cl.sbl_forward_sparse24(al, al, al, al, 0, 16, 8, al, None, None) == 0
    # dense 2-bit layout
    assert cl.sbl_pack_dense2(al, 8, 16, al, 4, None) == 5
    assert cl.sbl_pack_dense2(None, 8, 16, al, 1 << 20, None) == 1
    # fused norm + quantiser
    assert cl.sbl_rmsnorm_act_quant(al, al, 0.0, 4, 16, None, al, al, None) == 1
    assert cl.sbl_rmsnorm_act_quant(al, None, 1e-6, 4, 16, None, al, al, None) == 1
    assert cl.sbl_rmsnorm_act_quant(al, al, 1e-6, 4, 16, al + 8, al, al, None) == 3
    assert cl.sbl_rmsnorm_act_quant(al, al, 1e-6, 0, 16, None, al, al, None) == 0
    # backward
    assert cl.sbl_backward(al, al, al, al, -1, 16, 8, al, al, 0, None, 0, None) == 2
    assert cl.sbl_backward(al, al, None, al, 4, 16, 8, al, None, 0, None, 0, None) == 1
    assert cl.sbl_backward(al, al, al, al, 4, 16, 8, None, al + 4, 0, None, 0, None) == 3
    assert cl.sbl_backward(al, al, al, al, 4, 16, 8, None, None, 0, None, 0, None) == 0
