"""The data-parallel exchange of the Sparse-BitLinear training step.

Every rank holds the same master weights W and runs the forward and the
Dual-STE backward on its own tokens.  gamma, the N:M mask and W_eff need no
exchange: each replica recomputes them from the same W, bit for bit.  The one
exchange is the gradient: the dense dW of every projection is summed over the
ranks before the optimizer step, so that every replica applies the same AdamW
update to the same W ("Sparse-BitNet：1.58-bit 大模型天然兼容半结构化稀疏",
方法步骤详情, Algorithm 1 steps (7) and (8)).  dW = dY^T X is a sum over
tokens, so the sum over ranks is dW of the concatenated batch.

The gradients of a layer set live in one flat fp32 buffer (`GradBucket`),
one view per projection, so the exchange can be issued per projection as
soon as its dW is written, overlapping the remaining backward products, and
waited for once before the clip norm.  The collective is torch.distributed's
all_reduce (NCCL on GPUs, gloo on the CPU); nothing here computes.
"""
from __future__ import annotations

from typing import Dict, Iterable, List, Tuple

import torch
import torch.distributed as dist


class GradBucket:
    """dW of every projection in one flat fp32 buffer.

    `shapes` maps a projection name to (d_out, d_in).  Views are laid out in
    the mapping's order, each starting at a multiple of 16 bytes (every
    d_out * d_in of this operator is a multiple of 8), so each view is a
    valid, aligned operand of the library's kernels."""

    def __init__(self, shapes: Dict[str, Tuple[int, int]], device, dtype=torch.float32):
        self.shapes = dict(shapes)
        self.offsets: Dict[str, Tuple[int, int]] = {}
        off = 0
        for name, (d_out, d_in) in self.shapes.items():
            n = d_out * d_in
            self.offsets[name] = (off, n)
            off += (n + 3) // 4 * 4
        self.numel = off
        self.flat = torch.zeros(off, dtype=dtype, device=device)
        self.views = {name: self.flat[o:o + n].view(self.shapes[name]) for name, (o, n) in self.offsets.items()}

    def __getitem__(self, name: str) -> torch.Tensor:
        return self.views[name]

    def nbytes(self) -> int:
        return self.flat.numel() * self.flat.element_size()


class GradExchange:
    """Sum of the bucket's views over all ranks of `group`.

    `launch(name)` starts the all-reduce of one projection's dW (call it
    after that dW has been enqueued on the current stream: the collective
    waits for the work already on that stream); `wait()` makes the current
    stream wait for every started exchange.  With one rank, or without an
    initialised process group, both do nothing: the local dW is already the
    sum."""

    def __init__(self, bucket: GradBucket, group=None):
        self.bucket = bucket
        self.group = group
        self.pending: List = []
        self.active = dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1

    def launch(self, name: str) -> None:
        if not self.active:
            return
        self.pending.append(dist.all_reduce(self.bucket[name], op=dist.ReduceOp.SUM, group=self.group,
                                            async_op=True))

    def launch_all(self, names: Iterable[str] | None = None) -> None:
        for name in (self.bucket.views if names is None else names):
            self.launch(name)

    def wait(self) -> None:
        for h in self.pending:
            h.wait()
        self.pending = []
