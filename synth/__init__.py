"""Seeded synthetic inputs for the Sparse-BitLinear operator.

This module is shared by the CPU oracle (``oracle/``) and the CUDA path
(``semi_structured_sparsity_step_b200``).  It only draws random numbers and
describes workload shapes; it holds none of the operator's arithmetic (no
mask, no quantiser, no scale, no product).  Every tensor comes out as a CPU
``torch.bfloat16`` tensor, drawn from a ``torch.Generator`` seeded with
``seed * 1000 + tensor_id`` so each tensor of a workload has its own stream.

Distributions follow the workloads the Sparse-BitNet pages describe:

* master weights ~ N(0, 0.02) (BitNet-style initialisation), or the trimodal
  "latent weight" mixture that mirrors the ternary state shares the
  Sparse-BitNet summary reports for a trained BitNet (Figure 1, 0 at about
  42%, +1 and -1 at about 29% each): 42% N(0, 0.3 s), 29% N(+1.3 s, 0.3 s),
  29% N(-1.3 s, 0.3 s) with s = 0.02;
* activations and upstream gradients ~ N(0, 1), optionally with a small
  fraction of outlier channels scaled by 10;
* groups with exact magnitude ties placed across the top-N boundary, built
  by construction (no ranking is computed here);
* optimizer state for the AdamW step: fp32 weight gradients ~ N(0, g_std),
  first moments ~ N(0, 0.3 g_std) and second moments = (g_std * |z|)^2 for
  z ~ N(0, 1) (non-negative, of the gradients' scale), g_std = 1e-3.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch

__all__ = [
    "gen",
    "normal_weight",
    "trimodal_weight",
    "activations",
    "grad_output",
    "with_boundary_ties",
    "optimizer_state",
    "bits",
    "from_bits",
    "Projection",
    "LayerSet",
    "layer_set",
]


def gen(seed: int, tensor_id: int) -> torch.Generator:
    """Return the CPU generator for tensor ``tensor_id`` of workload ``seed``."""
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed) * 1000 + int(tensor_id))
    return g


def normal_weight(d_out: int, d_in: int, seed: int = 0, tensor_id: int = 0,
                  std: float = 0.02) -> torch.Tensor:
    """Master weight W [d_out, d_in] ~ N(0, std), rounded to bf16."""
    g = gen(seed, tensor_id)
    w = torch.randn(d_out, d_in, generator=g, dtype=torch.float32) * std
    return w.to(torch.bfloat16)


def trimodal_weight(d_out: int, d_in: int, seed: int = 0, tensor_id: int = 0,
                    s: float = 0.02) -> torch.Tensor:
    """Master weight drawn from the trimodal latent mixture, rounded to bf16.

    Component 0 (p = 0.42): N(0, 0.3 s); component +1 (p = 0.29):
    N(+1.3 s, 0.3 s); component -1 (p = 0.29): N(-1.3 s, 0.3 s).
    """
    g = gen(seed, tensor_id)
    u = torch.rand(d_out, d_in, generator=g, dtype=torch.float32)
    z = torch.randn(d_out, d_in, generator=g, dtype=torch.float32)
    centre = torch.zeros_like(u)
    centre[u >= 0.42] = 1.3 * s
    centre[u >= 0.71] = -1.3 * s
    return (centre + 0.3 * s * z).to(torch.bfloat16)


def activations(T: int, d_in: int, seed: int = 0, tensor_id: int = 100,
                outlier_frac: float = 0.0, outlier_scale: float = 10.0) -> torch.Tensor:
    """Activations X [T, d_in] ~ N(0, 1) in bf16.

    With ``outlier_frac > 0``, max(1, round(outlier_frac * d_in)) channels
    chosen by the same generator are multiplied by ``outlier_scale``.
    """
    g = gen(seed, tensor_id)
    x = torch.randn(T, d_in, generator=g, dtype=torch.float32)
    if outlier_frac > 0.0:
        n_out = max(1, int(round(outlier_frac * d_in)))
        ch = torch.randperm(d_in, generator=g)[:n_out]
        x[:, ch] *= outlier_scale
    return x.to(torch.bfloat16)


def grad_output(T: int, d_out: int, seed: int = 0, tensor_id: int = 200) -> torch.Tensor:
    """Upstream gradient dY [T, d_out] ~ N(0, 1) in bf16."""
    g = gen(seed, tensor_id)
    return torch.randn(T, d_out, generator=g, dtype=torch.float32).to(torch.bfloat16)


def with_boundary_ties(w: torch.Tensor, N: int, M: int, seed: int = 0, tensor_id: int = 300,
                       frac: float = 0.01, all_equal_groups: int = 4,
                       s: float = 0.02) -> torch.Tensor:
    """Overwrite a fraction of the M-groups of ``w`` with tie-straddling groups.

    Each chosen group is rebuilt from scratch: N-1 "large" magnitudes in
    [2 s, 3 s), two copies of one tie magnitude 1.5 s, and M-N-1 "small"
    magnitudes in [0, s), at random positions with random signs.  The two
    equal magnitudes are therefore the N-th and (N+1)-th largest, so a top-N
    selection must break the tie.  ``all_equal_groups`` further groups get
    the same magnitude at all M positions.  Requires 1 <= N < M.
    """
    assert 1 <= N < M
    d_out, d_in = w.shape
    assert d_in % M == 0
    g = gen(seed, tensor_id)
    out = w.to(torch.float32).reshape(-1, M).clone()
    G = out.shape[0]
    n_tie = max(1, int(round(frac * G)))
    chosen = torch.randperm(G, generator=g)[: n_tie + all_equal_groups]
    tie_groups, eq_groups = chosen[:n_tie], chosen[n_tie:]
    large = (2.0 + torch.rand(n_tie, N - 1, generator=g)) * s
    small = torch.rand(n_tie, M - N - 1, generator=g) * s
    tie = torch.full((n_tie, 2), 1.5 * s)
    mags = torch.cat([large, tie, small], dim=1)
    perm = torch.argsort(torch.rand(n_tie, M, generator=g), dim=1)  # a random permutation per group
    sign = torch.where(torch.rand(n_tie, M, generator=g) < 0.5, -1.0, 1.0)
    rows = torch.empty(n_tie, M)
    rows.scatter_(1, perm, mags * sign)
    out[tie_groups] = rows
    if all_equal_groups:
        esign = torch.where(torch.rand(len(eq_groups), M, generator=g) < 0.5, -1.0, 1.0)
        out[eq_groups] = 1.5 * s * esign
    # 1.5 s, 2 s .. 3 s are rounded to bf16 once here; equal inputs stay equal.
    return out.reshape(d_out, d_in).to(torch.bfloat16)


def optimizer_state(d_out: int, d_in: int, seed: int = 0, tensor_id: int = 400,
                    g_std: float = 1e-3):
    """(dW, m, v) fp32 CPU tensors [d_out, d_in] for one AdamW step: the
    gradient ~ N(0, g_std), the first moment ~ N(0, 0.3 g_std) and the second
    moment (g_std * z)^2 with z ~ N(0, 1)."""
    g = gen(seed, tensor_id)
    dw = torch.randn(d_out, d_in, generator=g, dtype=torch.float32) * g_std
    m = torch.randn(d_out, d_in, generator=g, dtype=torch.float32) * (0.3 * g_std)
    z = torch.randn(d_out, d_in, generator=g, dtype=torch.float32) * g_std
    return dw, m, z * z


def bits(t: torch.Tensor) -> np.ndarray:
    """Raw bf16 bit patterns of a CPU bf16 tensor as a numpy uint16 array."""
    assert t.dtype == torch.bfloat16
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def from_bits(u16: np.ndarray) -> torch.Tensor:
    """Inverse of :func:`bits`."""
    return torch.from_numpy(np.ascontiguousarray(u16).view(np.int16)).view(torch.bfloat16)


@dataclass(frozen=True)
class Projection:
    """One linear projection of a transformer block: W is [d_out, d_in]."""
    name: str
    d_out: int
    d_in: int
    input_name: str  # which activation tensor feeds it


@dataclass(frozen=True)
class LayerSet:
    name: str
    hidden: int
    intermediate: int
    kv_dim: int
    projections: tuple

    @property
    def params(self) -> int:
        return sum(p.d_out * p.d_in for p in self.projections)

    @property
    def inputs(self) -> dict:
        """Distinct activation inputs: name -> d_in."""
        d = {}
        for p in self.projections:
            d.setdefault(p.input_name, p.d_in)
        return d


def layer_set(name: str) -> LayerSet:
    """The seven projections of one Qwen2.5-shaped transformer block.

    q/o: hidden x hidden, k/v: kv_dim x hidden, gate/up: intermediate x
    hidden, down: hidden x intermediate.  q, k and v read the attention input;
    gate and up read the MLP input.  "qwen2.5-3b-up" is the up projection of
    the 3B block alone (11008 x 2048).
    """
    shapes = {
        "qwen2.5-0.5b": (896, 4864, 128),
        "qwen2.5-3b": (2048, 11008, 256),
    }
    if name == "qwen2.5-3b-up":
        return LayerSet(name, 2048, 11008, 256, (Projection("up", 11008, 2048, "mlp_in"),))
    h, i, kv = shapes[name]
    projs = (
        Projection("q", h, h, "attn_in"),
        Projection("k", kv, h, "attn_in"),
        Projection("v", kv, h, "attn_in"),
        Projection("o", h, h, "o_in"),
        Projection("gate", i, h, "mlp_in"),
        Projection("up", i, h, "mlp_in"),
        Projection("down", h, i, "down_in"),
    )
    return LayerSet(name, h, i, kv, projs)
