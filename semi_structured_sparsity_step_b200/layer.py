"""Device buffers of one Sparse-BitLinear layer and its step through the C ABI.

PyTorch only provides device memory and the stream here; every step of the
operator runs in libsbl's kernels:

    weight_step()  -> sbl_mask_quant   (mask, gamma, ternary, quant-then-mask)
                      + sbl_compress24 for a 2:4 layer built with sparse24=True
    forward(X)     -> sbl_act_quant, sbl_forward (or sbl_forward_sparse24)
    backward(dY)   -> sbl_backward     (dX and the dense dW)
"""
from __future__ import annotations

import torch

from . import _binding as B


class SparseBitLinearLayer:
    def __init__(self, W: torch.Tensor, N: int, M: int, keep_mask: bool = False, sparse24: bool = True):
        assert W.is_cuda and W.dtype == torch.bfloat16 and W.is_contiguous()
        self.W = W
        self.d_out, self.d_in = W.shape
        self.N, self.M = N, M
        dev = W.device
        self.W_eff = torch.empty(self.d_out, self.d_in, dtype=torch.int8, device=dev)
        self.W_eff_bf16 = torch.empty(self.d_out, self.d_in, dtype=torch.bfloat16, device=dev)
        self.mask_bits = (torch.empty(self.d_out, self.d_in // 8, dtype=torch.uint8, device=dev)
                          if keep_mask else None)
        self.gamma = torch.empty(1, dtype=torch.float32, device=dev)
        self.ws_bytes = B.sbl_mask_quant_workspace_bytes(self.d_out, self.d_in)
        self.ws = torch.empty(self.ws_bytes, dtype=torch.uint8, device=dev)
        # 2:4 weights go to the sparse tensor core through the compressed
        # format (the same int32 sums as the dense product, bit for bit; on B200
        # about 1.2x faster than the dense int8 product at the measured shapes).
        # sparse24=False keeps the dense product for them.
        self.sparse24 = bool(sparse24) and (N, M) == (2, 4)
        self.w24_bytes = B.sbl_compress24_bytes(self.d_out, self.d_in) if self.sparse24 else 0
        self.w24 = torch.empty(self.w24_bytes, dtype=torch.uint8, device=dev) if self.sparse24 else None

    def weight_step(self, stream=None):
        B.sbl_mask_quant(self.W, self.d_out, self.d_in, self.N, self.M, self.W_eff, self.W_eff_bf16,
                         self.mask_bits, self.gamma, self.ws, self.ws_bytes, stream)
        if self.sparse24:
            B.sbl_compress24(self.W_eff, self.d_out, self.d_in, self.w24, self.w24_bytes, stream)

    def forward(self, Xq, amax, Y, T=None, acc=None, stream=None):
        T = Xq.shape[0] if T is None else T
        if self.sparse24:
            B.sbl_forward_sparse24(Xq, amax, self.w24, self.gamma, T, self.d_in, self.d_out, Y, acc, stream)
        else:
            B.sbl_forward(Xq, amax, self.W_eff, self.gamma, T, self.d_in, self.d_out, Y, acc, stream)

    def backward(self, dY, X, dX, dW, accumulate_dW=False, T=None, stream=None):
        T = dY.shape[0] if T is None else T
        B.sbl_backward(dY, X, self.W_eff_bf16, self.gamma, T, self.d_in, self.d_out, dX, dW,
                       int(accumulate_dW), None, 0, stream)


def act_quant(X: torch.Tensor, Xq: torch.Tensor, amax: torch.Tensor, stream=None):
    T, d_in = X.shape
    B.sbl_act_quant(X, T, d_in, Xq, amax, stream)
