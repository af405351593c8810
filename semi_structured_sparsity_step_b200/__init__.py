"""B200-native Sparse-BitLinear: CUDA kernels for sm_100a behind a C ABI.

The library (``libsbl.so``, built by ``python -m
semi_structured_sparsity_step_b200.build``) exports the entry points declared
in ``include/sbl.h``; this package re-exports their ctypes binding under the
same names, plus :mod:`.layer`, a small helper that owns the device buffers of
one Sparse-BitLinear layer and runs its training step through the C ABI.
"""
from ._binding import (  # noqa: F401
    load, SBL_MASK_FROM_QUANTISED, SblError, sbl_act_quant, sbl_adamw_step, sbl_backward,
    sbl_backward_workspace_bytes, sbl_check, sbl_compress24, sbl_compress24_bytes, sbl_dense2_bytes,
    sbl_forward, sbl_forward_group, sbl_forward_packed, sbl_forward_sparse24, sbl_gemv_dense2_group,
    sbl_gemv_packed, sbl_gemv_packed_group, sbl_grad_sqnorm, sbl_mask_grad, sbl_mask_quant,
    sbl_mask_quant_ex, sbl_mask_quant_noalloc, sbl_mask_quant_noalloc_scratch_bytes,
    sbl_mask_quant_workspace_bytes, sbl_pack, sbl_pack_dense2, sbl_packed_bytes,
    sbl_rmsnorm_act_quant, sbl_selftest_wait_timeout, sbl_set_gemm_variant, sbl_set_gemv_variant,
    sbl_status_string, sbl_unpack, sbl_version,
)

__all__ = [
    "load", "sbl_act_quant", "sbl_adamw_step", "sbl_backward", "sbl_backward_workspace_bytes",
    "sbl_check", "sbl_compress24", "sbl_compress24_bytes", "sbl_dense2_bytes", "sbl_forward",
    "sbl_forward_group", "sbl_forward_packed", "sbl_forward_sparse24", "sbl_gemv_dense2_group",
    "sbl_gemv_packed", "sbl_gemv_packed_group", "sbl_grad_sqnorm", "SBL_MASK_FROM_QUANTISED",
    "sbl_mask_grad", "sbl_mask_quant", "sbl_mask_quant_ex", "sbl_mask_quant_noalloc",
    "sbl_mask_quant_noalloc_scratch_bytes", "sbl_mask_quant_workspace_bytes", "sbl_pack",
    "sbl_pack_dense2", "sbl_packed_bytes", "sbl_rmsnorm_act_quant", "sbl_selftest_wait_timeout",
    "sbl_set_gemm_variant", "sbl_set_gemv_variant", "sbl_status_string", "sbl_unpack",
    "sbl_version", "SblError",
]
