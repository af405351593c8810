"""ctypes binding of libsbl.so (the C ABI in include/sbl.h).

Argument marshalling only: each function takes torch tensors (or raw device
pointers as ints), passes their device pointers, sizes and the current CUDA
stream to the C entry point of the same name, and raises SblError on a
non-OK status.  Every computation runs in the library's CUDA kernels; there
is no fallback path.  Output tensors are allocated by the caller.
"""
from __future__ import annotations

import ctypes
import os

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libsbl.so")

_c_int = ctypes.c_int
_c_size = ctypes.c_size_t
_vp = ctypes.c_void_p

class ForwardProblem(ctypes.Structure):
    """sbl_forward_problem: one product of a grouped forward (device pointers)."""
    _fields_ = [("Xq", _vp), ("amax", _vp), ("W_eff", _vp), ("gamma", _vp), ("T", _c_int), ("d_in", _c_int),
                ("d_out", _c_int), ("Y", _vp), ("acc", _vp)]


class GemvProblem(ctypes.Structure):
    """sbl_gemv_problem: one decode GEMV of a group (device pointers)."""
    _fields_ = [("packed", _vp), ("Xq", _vp), ("amax", _vp), ("gamma", _vp), ("Y", _vp),
                ("d_in", _c_int), ("d_out", _c_int)]


# name -> (restype, argtypes)
SIGNATURES = {
    "sbl_status_string": (ctypes.c_char_p, [_c_int]),
    "sbl_version": (_c_int, []),
    "sbl_set_gemv_variant": (_c_int, [_c_int]),
    "sbl_check": (_c_int, [_vp]),
    "sbl_selftest_wait_timeout": (_c_int, [ctypes.c_uint, _vp]),
    "sbl_set_gemm_variant": (_c_int, [_c_int]),
    "sbl_mask_quant_workspace_bytes": (_c_size, [_c_int, _c_int]),
    "sbl_mask_quant": (_c_int, [_vp, _c_int, _c_int, _c_int, _c_int, _vp, _vp, _vp, _vp, _vp, _c_size, _vp]),
    "sbl_mask_quant_ex": (_c_int, [_vp, _c_int, _c_int, _c_int, _c_int, ctypes.c_uint, _vp, _vp, _vp, _vp, _vp, _c_size,
                                   _vp]),
    "sbl_mask_grad": (_c_int, [_vp, _vp, _c_int, _c_int, _vp]),
    "sbl_grad_sqnorm": (_c_int, [_vp, _c_size, _vp, _vp, _c_size, _vp]),
    "sbl_adamw_step": (_c_int, [_vp, _vp, _vp, _vp, _vp, _c_int, _c_int, _c_int, _c_int, ctypes.c_double,
                                ctypes.c_double, ctypes.c_double, ctypes.c_double, ctypes.c_double,
                                ctypes.c_longlong, _vp, ctypes.c_double, _vp, _vp, _vp, _vp, _vp, _vp, _c_size,
                                _vp]),
    "sbl_mask_quant_noalloc_scratch_bytes": (_c_size, []),
    "sbl_mask_quant_noalloc": (_c_int, [_vp, _c_int, _c_int, _c_int, _c_int, _vp, _vp, _vp, _vp, _vp]),
    "sbl_act_quant": (_c_int, [_vp, _c_int, _c_int, _vp, _vp, _vp]),
    "sbl_rmsnorm_act_quant": (_c_int, [_vp, _vp, ctypes.c_float, _c_int, _c_int, _vp, _vp, _vp, _vp]),
    "sbl_forward": (_c_int, [_vp, _vp, _vp, _vp, _c_int, _c_int, _c_int, _vp, _vp, _vp]),
    "sbl_forward_packed": (_c_int, [_vp, _vp, _vp, _vp, _c_int, _c_int, _c_int, _c_int, _c_int, _vp, _vp, _vp]),
    "sbl_forward_group": (_c_int, [_vp, _c_int, _vp]),
    "sbl_compress24_bytes": (_c_size, [_c_int, _c_int]),
    "sbl_compress24": (_c_int, [_vp, _c_int, _c_int, _vp, _c_size, _vp]),
    "sbl_forward_sparse24": (_c_int, [_vp, _vp, _vp, _vp, _c_int, _c_int, _c_int, _vp, _vp, _vp]),
    "sbl_backward_workspace_bytes": (_c_size, [_c_int, _c_int, _c_int]),
    "sbl_backward": (_c_int, [_vp, _vp, _vp, _vp, _c_int, _c_int, _c_int, _vp, _vp, _c_int, _vp, _c_size, _vp]),
    "sbl_packed_bytes": (_c_size, [_c_int, _c_int, _c_int, _c_int]),
    "sbl_pack": (_c_int, [_vp, _c_int, _c_int, _c_int, _c_int, _vp, _c_size, _vp]),
    "sbl_unpack": (_c_int, [_vp, _c_int, _c_int, _c_int, _c_int, _vp, _vp]),
    "sbl_gemv_packed": (_c_int, [_vp, _vp, _c_int, _vp, _vp, _c_int, _c_int, _c_int, _c_int, _vp, _vp]),
    "sbl_gemv_packed_group": (_c_int, [ctypes.POINTER(GemvProblem), _c_int, _c_int, _c_int, _c_int, _vp]),
    "sbl_dense2_bytes": (_c_size, [_c_int, _c_int]),
    "sbl_pack_dense2": (_c_int, [_vp, _c_int, _c_int, _vp, _c_size, _vp]),
    "sbl_gemv_dense2_group": (_c_int, [ctypes.POINTER(GemvProblem), _c_int, _c_int, _vp]),
}

STATUS = {
    0: "SBL_OK", 1: "SBL_ERR_INVALID_ARG", 2: "SBL_ERR_SHAPE", 3: "SBL_ERR_ALIGN",
    4: "SBL_ERR_UNSUPPORTED", 5: "SBL_ERR_WORKSPACE", 6: "SBL_ERR_TIMEOUT", 7: "SBL_ERR_CUDA",
    8: "SBL_ERR_DEVICE_CHECK",
}


class SblError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn} returned {STATUS.get(status, status)}")


_lib = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libsbl.so once; raises if it was not built (no fallback)."""
    global _lib
    if _lib is None:
        if not os.path.exists(path):
            raise ImportError(
                f"{path} is missing: build it with `python -m semi_structured_sparsity_step_b200.build`")
        lib = ctypes.CDLL(path)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _call(name, *args):
    st = getattr(load(), name)(*args)
    if st != 0:
        raise SblError(name, st)


def sbl_status_string(status: int) -> str:
    return load().sbl_status_string(status).decode()


def sbl_version() -> int:
    return load().sbl_version()


def sbl_set_gemm_variant(variant: int) -> None:
    _call("sbl_set_gemm_variant", int(variant))


def sbl_set_gemv_variant(variant: int) -> None:
    _call("sbl_set_gemv_variant", int(variant))


def sbl_check(stream=None) -> None:
    _call("sbl_check", _stream(stream))


def sbl_selftest_wait_timeout(limit_us: int, stream=None) -> None:
    _call("sbl_selftest_wait_timeout", int(limit_us), _stream(stream))


def sbl_mask_quant_workspace_bytes(d_out: int, d_in: int) -> int:
    return load().sbl_mask_quant_workspace_bytes(d_out, d_in)


def sbl_mask_quant(W, d_out, d_in, N, M, W_eff, W_eff_bf16, mask_bits, gamma, workspace, workspace_bytes,
                   stream=None) -> None:
    _call("sbl_mask_quant", _ptr(W), d_out, d_in, N, M, _ptr(W_eff), _ptr(W_eff_bf16), _ptr(mask_bits),
          _ptr(gamma), _ptr(workspace), workspace_bytes, _stream(stream))


SBL_MASK_FROM_QUANTISED = 1


def sbl_mask_quant_ex(W, d_out, d_in, N, M, flags, W_eff, W_eff_bf16, mask_bits, gamma, workspace, workspace_bytes,
                      stream=None) -> None:
    _call("sbl_mask_quant_ex", _ptr(W), d_out, d_in, N, M, int(flags), _ptr(W_eff), _ptr(W_eff_bf16), _ptr(mask_bits),
          _ptr(gamma), _ptr(workspace), workspace_bytes, _stream(stream))


def sbl_mask_grad(dW, mask_bits, d_out, d_in, stream=None) -> None:
    _call("sbl_mask_grad", _ptr(dW), _ptr(mask_bits), d_out, d_in, _stream(stream))


def sbl_grad_sqnorm(dW, n, sumsq, workspace, workspace_bytes, stream=None) -> None:
    _call("sbl_grad_sqnorm", _ptr(dW), int(n), _ptr(sumsq), _ptr(workspace), workspace_bytes, _stream(stream))


def sbl_adamw_step(W, W32, dW, m, v, d_out, d_in, N, M, lr, beta1, beta2, eps, weight_decay, step, grad_sqnorm,
                   max_norm, W_eff, W_eff_bf16, mask_bits, gamma, flips, workspace, workspace_bytes,
                   stream=None) -> None:
    _call("sbl_adamw_step", _ptr(W), _ptr(W32), _ptr(dW), _ptr(m), _ptr(v), d_out, d_in, N, M, float(lr),
          float(beta1), float(beta2), float(eps), float(weight_decay), int(step), _ptr(grad_sqnorm),
          float(max_norm), _ptr(W_eff), _ptr(W_eff_bf16), _ptr(mask_bits), _ptr(gamma), _ptr(flips),
          _ptr(workspace), workspace_bytes, _stream(stream))


def sbl_mask_quant_noalloc_scratch_bytes() -> int:
    return load().sbl_mask_quant_noalloc_scratch_bytes()


def sbl_mask_quant_noalloc(W, d_out, d_in, N, M, W_eff, W_eff_bf16, mask_bits, gamma, stream=None) -> None:
    """sbl_mask_quant for callers that cannot allocate device memory when
    the weight step runs: the scratch is a fixed array in the library's
    static device memory (see include/sbl.h for the size limit and for why
    calls must be ordered on one stream)."""
    _call("sbl_mask_quant_noalloc", _ptr(W), d_out, d_in, N, M, _ptr(W_eff), _ptr(W_eff_bf16), _ptr(mask_bits),
          _ptr(gamma), _stream(stream))


def sbl_act_quant(X, T, d_in, Xq, amax, stream=None) -> None:
    _call("sbl_act_quant", _ptr(X), T, d_in, _ptr(Xq), _ptr(amax), _stream(stream))


def sbl_rmsnorm_act_quant(X, g, eps, T, d_in, Xn, Xq, amax, stream=None) -> None:
    _call("sbl_rmsnorm_act_quant", _ptr(X), _ptr(g), float(eps), T, d_in, _ptr(Xn), _ptr(Xq), _ptr(amax),
          _stream(stream))


def sbl_forward(Xq, amax, W_eff, gamma, T, d_in, d_out, Y, acc=None, stream=None) -> None:
    _call("sbl_forward", _ptr(Xq), _ptr(amax), _ptr(W_eff), _ptr(gamma), T, d_in, d_out, _ptr(Y), _ptr(acc),
          _stream(stream))


def sbl_forward_group(problems, stream=None) -> None:
    """problems: list of (Xq, amax, W_eff, gamma, T, d_in, d_out, Y, acc_or_None)."""
    arr = (ForwardProblem * max(1, len(problems)))()
    for i, (xq, am, w, g, T, d_in, d_out, y, acc) in enumerate(problems):
        arr[i] = ForwardProblem(_ptr(xq), _ptr(am), _ptr(w), _ptr(g), T, d_in, d_out, _ptr(y), _ptr(acc))
    _call("sbl_forward_group", ctypes.cast(arr, _vp), len(problems), _stream(stream))


def sbl_forward_packed(Xq, amax, packed, gamma, T, d_in, d_out, N, M, Y, acc=None, stream=None) -> None:
    _call("sbl_forward_packed", _ptr(Xq), _ptr(amax), _ptr(packed), _ptr(gamma), T, d_in, d_out, N, M, _ptr(Y),
          _ptr(acc), _stream(stream))


def sbl_compress24_bytes(d_out, d_in) -> int:
    return load().sbl_compress24_bytes(d_out, d_in)


def sbl_compress24(W_eff, d_out, d_in, out, out_bytes, stream=None) -> None:
    _call("sbl_compress24", _ptr(W_eff), d_out, d_in, _ptr(out), out_bytes, _stream(stream))


def sbl_forward_sparse24(Xq, amax, w24, gamma, T, d_in, d_out, Y, acc=None, stream=None) -> None:
    _call("sbl_forward_sparse24", _ptr(Xq), _ptr(amax), _ptr(w24), _ptr(gamma), T, d_in, d_out, _ptr(Y), _ptr(acc),
          _stream(stream))


def sbl_backward_workspace_bytes(T, d_in, d_out) -> int:
    return load().sbl_backward_workspace_bytes(T, d_in, d_out)


def sbl_backward(dY, X, W_eff_bf16, gamma, T, d_in, d_out, dX, dW, accumulate_dW=0, workspace=None,
                 workspace_bytes=0, stream=None) -> None:
    _call("sbl_backward", _ptr(dY), _ptr(X), _ptr(W_eff_bf16), _ptr(gamma), T, d_in, d_out, _ptr(dX), _ptr(dW),
          int(accumulate_dW), _ptr(workspace), workspace_bytes, _stream(stream))


def sbl_packed_bytes(d_out, d_in, N, M) -> int:
    return load().sbl_packed_bytes(d_out, d_in, N, M)


def sbl_pack(W_eff, d_out, d_in, N, M, packed, packed_bytes, stream=None) -> None:
    _call("sbl_pack", _ptr(W_eff), d_out, d_in, N, M, _ptr(packed), packed_bytes, _stream(stream))


def sbl_unpack(packed, d_out, d_in, N, M, W_eff, stream=None) -> None:
    _call("sbl_unpack", _ptr(packed), d_out, d_in, N, M, _ptr(W_eff), _stream(stream))


def sbl_gemv_packed(Xq, amax, batch, packed, gamma, d_in, d_out, N, M, Y, stream=None) -> None:
    _call("sbl_gemv_packed", _ptr(Xq), _ptr(amax), batch, _ptr(packed), _ptr(gamma), d_in, d_out, N, M, _ptr(Y),
          _stream(stream))


def sbl_gemv_packed_group(problems, batch, N, M, stream=None) -> None:
    """problems: sequence of (packed, Xq, amax, gamma, Y, d_in, d_out)."""
    arr = (GemvProblem * len(problems))()
    for i, (pk, xq, am, gm, y, d_in, d_out) in enumerate(problems):
        arr[i] = GemvProblem(_ptr(pk), _ptr(xq), _ptr(am), _ptr(gm), _ptr(y), d_in, d_out)
    _call("sbl_gemv_packed_group", arr, len(problems), batch, N, M, _stream(stream))


def sbl_dense2_bytes(d_out, d_in) -> int:
    return load().sbl_dense2_bytes(d_out, d_in)


def sbl_pack_dense2(W_eff, d_out, d_in, out, out_bytes, stream=None) -> None:
    _call("sbl_pack_dense2", _ptr(W_eff), d_out, d_in, _ptr(out), out_bytes, _stream(stream))


def sbl_gemv_dense2_group(problems, batch, stream=None) -> None:
    """problems: sequence of (dense2 buffer, Xq, amax, gamma, Y, d_in, d_out)."""
    arr = (GemvProblem * len(problems))()
    for i, (pk, xq, am, gm, y, d_in, d_out) in enumerate(problems):
        arr[i] = GemvProblem(_ptr(pk), _ptr(xq), _ptr(am), _ptr(gm), _ptr(y), d_in, d_out)
    _call("sbl_gemv_dense2_group", arr, len(problems), batch, _stream(stream))
