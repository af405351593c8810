"""CPU oracle for the Sparse-BitLinear operator (test infrastructure).

This module is test infrastructure.  Only the tests under ``tests/``,
``__graft_entry__.smoke()`` and the ``cpu_baseline`` / ``--impl reference``
legs of ``bench.py`` may import or call it.  The CUDA library
(``semi_structured_sparsity_step_b200``) never imports it, and it imports
nothing from the CUDA library: the two share no code.  Inputs come from the
seeded generators in ``synth`` as raw bf16 bit patterns (numpy ``uint16``).

It is a plain, slow restatement of what the operator computes, written in
numpy so that each step can be checked against the pages by eye.  Floating
point steps that decide integers (ternary codes, int8 activations) are
written as explicit IEEE fp32 operations, in the order given below, so that
a GPU implementation can reproduce them bit for bit; the reductions that only
feed float outputs (the backward products) are done in fp64.

Pages cited (titles as they appear on the pages):

* [summary]   "Sparse-BitNet：1.58-bit 大模型天然兼容半结构化稀疏" -- the
  structured summary of arXiv 2603.05168 (sections 前置知识, 核心方法,
  方法步骤详情 / Algorithm 1, 局限与改进, 独立分析的弱点, 论文图表).
* [gist]      the gist.science technical summary of the same paper
  (section 2.2 "Sparse-BitNet 框架").
* [explainer] "什麼是 Sparse-BitNet？核心概念一次搞懂" (sections
  "1.58 位元量化的技術原理", "N:M 半結構化稀疏性的運作機制").
* [article]   "突破性发现：极低位量化与稀疏化的完美协同" (section 7.1,
  "推理优化技巧").

Readings taken where the pages are silent (each is pinned by a test):

* ties in |W| inside a group go to the lowest index;
* the quantiser divides by (gamma + 1e-5); outputs are scaled by gamma;
* gamma is the exact mean of |W| over the whole tensor, rounded once to
  fp64 (correctly rounded sum, then an fp64 division), then to fp32;
* an all-zero activation row uses max|x| = 1e-5 (so it quantises to zeros);
* the straight-through estimator is the identity through the activation
  quantiser, RoundClip and the N:M selector; no gradient flows through gamma.

Parity status: every function here is pinned by ``tests/test_oracle_pins.py``
or, for the optimizer step, ``tests/test_oracle_adamw_pins.py`` (none is
"parity unpinned").
"""
from __future__ import annotations

import math

import numpy as np

EPS = np.float32(1e-5)          # quantiser epsilon (denominator only)
ACT_FLOOR = np.float32(1e-5)    # floor for max|x| of a token
QMAX = np.float32(127.0)        # int8 absmax level


# --------------------------------------------------------------------------
# bf16 decoding (format plumbing, exact)
# --------------------------------------------------------------------------
def bf16_to_f32(u16: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> the same values as fp32 (exact widening)."""
    u16 = np.ascontiguousarray(u16, dtype=np.uint16)
    return (u16.astype(np.uint32) << np.uint32(16)).view(np.float32)


# --------------------------------------------------------------------------
# (a1) N:M magnitude mask  M_{N:M} = Pi_{N:M}(|W|)
# [summary] 半结构化 N:M 稀疏 (||M_group||_0 = N per M consecutive weights);
# [summary] 核心方法 (i) and Algorithm 1 step (2): top-N by magnitude of the
# continuous master weight, recomputed every step; [gist] 2.2 (mask from
# master weights, not from ternary weights).
# --------------------------------------------------------------------------
def nm_mask(w_bits: np.ndarray, N: int, M: int, chunk: int = 1 << 18) -> np.ndarray:
    """Keep-mask (bool, same shape as W): top-N of |W| in each group of M
    consecutive weights along d_in.

    Rank of position j in its group: the number of members with a strictly
    larger magnitude plus the number of earlier members with an equal one.
    Position j is kept iff rank_j < N.  This keeps exactly N per group and
    breaks ties toward the lowest index.
    """
    return top_n_mask(np.abs(bf16_to_f32(w_bits)), N, M, chunk)


def top_n_mask(mag: np.ndarray, N: int, M: int, chunk: int = 1 << 18) -> np.ndarray:
    """The rank rule of nm_mask on any array of magnitudes [d_out, d_in]."""
    d_out, d_in = mag.shape
    assert d_in % M == 0 and 1 <= N <= M
    a_all = mag.reshape(-1, M)
    earlier = np.tri(M, k=-1, dtype=bool)          # earlier[j, k] = (k < j)
    keep = np.empty(a_all.shape, dtype=bool)
    for s in range(0, a_all.shape[0], chunk):
        a = a_all[s:s + chunk]
        aj = a[:, :, None]
        ak = a[:, None, :]
        rank = (ak > aj).sum(axis=2) + ((ak == aj) & earlier).sum(axis=2)
        keep[s:s + chunk] = rank < N
    return keep.reshape(d_out, d_in)


# --------------------------------------------------------------------------
# (a2) absmean scale  gamma = ||W||_1 / (d_out * d_in)
# [summary] 前置知识, "1.58-bit BitNet 量化".
# --------------------------------------------------------------------------
def absmean_gamma(w_bits: np.ndarray) -> np.float32:
    """gamma = fp32( fp64( sum |W| ) / n ), the sum rounded once.

    math.fsum returns the correctly rounded (round-half-even) fp64 value of
    the exact sum of its inputs; bf16 magnitudes are exact in fp64.
    """
    n = w_bits.size
    mags = np.abs(bf16_to_f32(w_bits).astype(np.float64)).ravel()
    total = math.fsum(mags)
    return np.float32(total / float(n))


# --------------------------------------------------------------------------
# (a3) ternary quantiser and quant-then-mask
# [summary] 前置知识: W_q = RoundClip(W / gamma, -1, +1); epsilon in the
# denominator per the plain reading of the operator spec; [summary] 核心方法
# (iii): W_eff = W_q (.) M_{N:M}; [explainer] "1.58 位元量化的技術原理"
# (threshold form -1 / 0 / +1 at -gamma/2, +gamma/2).
# --------------------------------------------------------------------------
def ternary(w_bits: np.ndarray, gamma: np.float32) -> np.ndarray:
    """W_q = clip(rint(fp32(w / fp32(gamma + eps))), -1, 1) as int8.

    rint rounds half to even, so |w / den| = 0.5 maps to 0.
    """
    w = bf16_to_f32(w_bits)
    den = np.float32(np.float32(gamma) + EPS)
    r = np.divide(w, den, dtype=np.float32)
    return np.clip(np.rint(r), -1.0, 1.0).astype(np.int8)


def effective_weight(w_bits: np.ndarray, N: int, M: int):
    """Algorithm 1 steps (2), (4), (5): returns (W_eff int8, gamma fp32,
    keep bool).  The mask comes from |W|, not from W_q."""
    keep = nm_mask(w_bits, N, M)
    gamma = absmean_gamma(w_bits)
    wq = ternary(w_bits, gamma)
    weff = np.where(keep, wq, np.int8(0)).astype(np.int8)
    return weff, gamma, keep


# --------------------------------------------------------------------------
# Ablations the pages evaluate (NEXT rank 3)
# [summary] 核心方法 / Dual-STE (masked weights keep their gradient; the
# ablation without it multiplies dW by the mask), [gist] 2.2 and the
# ablation of the mask source (Pi_N:M of |W_q| instead of |W|).
# --------------------------------------------------------------------------
def effective_weight_mask_from_quantised(w_bits: np.ndarray, N: int, M: int):
    """Ablation: the mask is the top-N of |W_q| (values 0 or 1) per group,
    ties to the lowest index; returns (W_eff, gamma, keep)."""
    gamma = absmean_gamma(w_bits)
    wq = ternary(w_bits, gamma)
    keep = top_n_mask(np.abs(wq.astype(np.float32)), N, M)
    weff = np.where(keep, wq, np.int8(0)).astype(np.int8)
    return weff, gamma, keep


def masked_grad(dw: np.ndarray, keep: np.ndarray) -> np.ndarray:
    """Ablation without the Dual-STE: dW (.) M (masked weights get zero)."""
    return np.where(keep, dw, np.float32(0.0)).astype(dw.dtype)


# --------------------------------------------------------------------------
# (a4) per-token absmax int8 activation quantisation
# [summary] 前置知识 ("激活值另用 absmax 量化到 8-bit 整数") and Algorithm 1
# step (3).
# --------------------------------------------------------------------------
def act_quant(x_bits: np.ndarray):
    """Returns (X_q int8 [T, d_in], amax fp32 [T]).

    amax_t = max(max_j |x_tj|, 1e-5); s_t = fp32(127 / amax_t);
    X_q = clip(rint(fp32(x * s_t)), -128, 127).
    """
    x = bf16_to_f32(x_bits)
    if x.shape[0] == 0:
        return np.zeros(x.shape, np.int8), np.zeros((0,), np.float32)
    a = np.abs(x).max(axis=1).astype(np.float32)
    a = np.maximum(a, ACT_FLOOR)
    s = np.divide(QMAX, a, dtype=np.float32)
    xs = np.multiply(x, s[:, None], dtype=np.float32)
    xq = np.clip(np.rint(xs), -128.0, 127.0).astype(np.int8)
    return xq, a


def f32_to_bf16(x: np.ndarray) -> np.ndarray:
    """fp32 values -> bf16 bit patterns, round to nearest even (finite inputs)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = (u + np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)
    return r.astype(np.uint16)


# --------------------------------------------------------------------------
# Norm before the activation quantiser: x~ = Q_a(Norm(x))
# [summary] Algorithm 1 step (3).  The pages do not name the norm; the
# reading taken is RMSNorm with a per-channel gain g (the norm BitNet-style
# layers put in front of Q_a), with the arithmetic fixed so that the int8
# codes do not depend on a summation order:
#   ss = sum_j x_j^2 in fp64 (each bf16 square is exact in fp64),
#   v = fl32(ss / d + eps) (fp64 division and sum, rounded once; eps is the
#       fp32 value the operator is given),
#   r = fl32(1 / fl32(sqrt(v))) (IEEE sqrt and divide in fp32),
#   xn_j = bf16(fl32(fl32(x_j * r) * g_j)) (round to nearest even),
# then Q_a of the bf16 row xn exactly as act_quant.
# --------------------------------------------------------------------------
def rms_norm(x_bits: np.ndarray, g_bits: np.ndarray, eps: float):
    """(xn bf16 bits [T, d], r fp32 [T])."""
    x = bf16_to_f32(x_bits)
    g = bf16_to_f32(g_bits)
    d = x.shape[1]
    ss = np.square(x.astype(np.float64)).sum(axis=1)
    v = (ss / d + float(np.float32(eps))).astype(np.float32)
    r = np.divide(np.float32(1.0), np.sqrt(v, dtype=np.float32), dtype=np.float32)
    t = np.multiply(x, r[:, None], dtype=np.float32)
    xn = np.multiply(t, g[None, :], dtype=np.float32)
    return f32_to_bf16(xn), r


def rms_norm_act_quant(x_bits: np.ndarray, g_bits: np.ndarray, eps: float):
    """(xn bf16 bits, X_q int8, amax fp32) of x~ = Q_a(RMSNorm(x))."""
    xn, _ = rms_norm(x_bits, g_bits, eps)
    xq, amax = act_quant(xn)
    return xn, xq, amax


# --------------------------------------------------------------------------
# (a5) forward: y = (X_q . W_eff^T) * gamma * amax / 127, int32 accumulation
# [summary] Algorithm 1 step (6) ("y ~ s * W_eff x~", s absorbs the scales);
# [summary] 半结构化 N:M 稀疏 (y = (W (.) M) x).
# --------------------------------------------------------------------------
def forward_acc(xq: np.ndarray, weff: np.ndarray) -> np.ndarray:
    """acc[t, o] = sum_j xq[t, j] * W_eff[o, j], exact integers (int32)."""
    acc = xq.astype(np.int64) @ weff.astype(np.int64).T
    return acc.astype(np.int32)


def forward_out(acc: np.ndarray, gamma: np.float32, amax: np.ndarray) -> np.ndarray:
    """y = fp32( fp32(acc) * fp32(gamma * fp32(amax / 127)) )."""
    c = np.divide(amax.astype(np.float32), QMAX, dtype=np.float32)
    sc = np.multiply(np.float32(gamma), c, dtype=np.float32)
    return np.multiply(acc.astype(np.float32), sc[:, None], dtype=np.float32)


def forward(x_bits: np.ndarray, w_bits: np.ndarray, N: int, M: int):
    """Whole forward of one Sparse-BitLinear layer.  Returns a dict."""
    weff, gamma, keep = effective_weight(w_bits, N, M)
    xq, amax = act_quant(x_bits)
    acc = forward_acc(xq, weff)
    y = forward_out(acc, gamma, amax)
    return dict(weff=weff, gamma=gamma, keep=keep, xq=xq, amax=amax, acc=acc, y=y)


# --------------------------------------------------------------------------
# (a6, a7) Dual-STE backward
# [summary] Straight-Through Estimator (Q replaced by the identity in the
# backward; Dual STE extends it to Pi_{N:M}); [summary] 核心方法 (masked
# weights receive the full gradient); Algorithm 1 step (7); [gist] 2.2.
# --------------------------------------------------------------------------
def backward_dx(dy_bits: np.ndarray, weff: np.ndarray, gamma: np.float32) -> np.ndarray:
    """dX = dY . (gamma * W_eff), fp64 accumulation, fp32 result."""
    dy = bf16_to_f32(dy_bits).astype(np.float64)
    return (float(gamma) * (dy @ weff.astype(np.float64))).astype(np.float32)


def backward_dw(dy_bits: np.ndarray, x_bits: np.ndarray) -> np.ndarray:
    """dW = dY^T . X (dense, unmasked), fp64 accumulation, fp32 result."""
    dy = bf16_to_f32(dy_bits).astype(np.float64)
    x = bf16_to_f32(x_bits).astype(np.float64)
    return (dy.T @ x).astype(np.float32)


# --------------------------------------------------------------------------
# (a9) packed inference format: 2-bit ternary codes + N:M index
# [article] 7.1 推理优化技巧 (pre-compute and cache the sparse format; bit
# operations for ternary products); [summary] 核心方法 (the deployed ternary
# weights are N:M-structured).  The pages fix only "2-bit ternary codes plus
# an N:M index"; the bit layout below is this library's.
#
# Per weight row, two planes, each padded to a multiple of 16 bytes:
#   index plane: for every group, an M-bit slot mask (bit p = position p is a
#     slot), little-endian bit stream (group g at bit g*M);
#   codes plane: the row is cut into chunks of 8 consecutive positions (one
#     group when M = 8, two when M = 4).  A chunk has K = 8N/M slots s_0 <
#     ... < s_(K-1) (its groups' slots in ascending position order) and a
#     field of 2K bits; chunk c's field starts at bit 2K*c of a little-endian
#     bit stream.  With H = ceil(K/2), the code of slot s_q (q < H) sits at
#     field bits 4q, 4q+1 and the code of slot s_(H+q) at bits 4q+2, 4q+3.
#   Code of a value: +1 -> 00, -1 -> 01, 0 -> 10 (bit 0 = negative, bit 1 =
#     zero); 11 is never written.
# Slots are all nonzero positions of the group plus, if there are fewer
# than N, the lowest-index zero positions.  The buffer holds all code rows
# first, then all index rows.
# --------------------------------------------------------------------------
def _ceil16(n: int) -> int:
    return (n + 15) // 16 * 16


def packed_layout(d_out: int, d_in: int, N: int, M: int):
    """(codes_row_bytes, index_row_bytes, total_bytes)."""
    G = d_in // M
    crow = _ceil16((G * N * 2 + 7) // 8)
    irow = _ceil16((G * M + 7) // 8)
    return crow, irow, d_out * (crow + irow)


def _put_bits(buf: bytearray, bitpos: int, value: int, nbits: int) -> None:
    for b in range(nbits):
        if (value >> b) & 1:
            buf[(bitpos + b) // 8] |= 1 << ((bitpos + b) % 8)


def _get_bits(buf, bitpos: int, nbits: int) -> int:
    v = 0
    for b in range(nbits):
        if (buf[(bitpos + b) // 8] >> ((bitpos + b) % 8)) & 1:
            v |= 1 << b
    return v


_CODE = {1: 0b00, -1: 0b01, 0: 0b10}
_VALUE = {0b00: 1, 0b01: -1, 0b10: 0}


def _slot_bit(i: int, K: int) -> int:
    """Bit offset, inside its chunk's field, of the code of slot i."""
    H = (K + 1) // 2
    return 4 * i if i < H else 4 * (i - H) + 2


def _group_slots(grp, N: int):
    """The slots of one group: nonzero positions, then lowest zero positions."""
    nz = [p for p in range(len(grp)) if grp[p] != 0]
    zeros = [p for p in range(len(grp)) if grp[p] == 0]
    return sorted(nz + zeros[: max(0, N - len(nz))])


def pack(weff: np.ndarray, N: int, M: int) -> np.ndarray:
    """Pack W_eff (int8 in {-1,0,1}, at most N nonzeros per group)."""
    d_out, d_in = weff.shape
    crow, irow, total = packed_layout(d_out, d_in, N, M)
    G = d_in // M
    K = 8 * N // M
    out = bytearray(total)
    for o in range(d_out):
        codes = bytearray(crow)
        index = bytearray(irow)
        for c in range(d_in // 8):
            chunk_slots = []                      # positions within the chunk
            for g in range(c * 8 // M, (c + 1) * 8 // M):
                grp = [int(v) for v in weff[o, g * M:(g + 1) * M]]
                if sum(v != 0 for v in grp) > N:
                    raise ValueError(f"row {o} group {g}: more than N={N} nonzeros")
                slots = _group_slots(grp, N)
                _put_bits(index, g * M, sum(1 << p for p in slots), M)
                chunk_slots += [g * M + p - 8 * c for p in slots]
            for i, p in enumerate(chunk_slots):
                _put_bits(codes, 2 * K * c + _slot_bit(i, K), _CODE[int(weff[o, 8 * c + p])], 2)
        out[o * crow:(o + 1) * crow] = codes
        base = d_out * crow
        out[base + o * irow: base + (o + 1) * irow] = index
    assert G * M == d_in
    return np.frombuffer(bytes(out), dtype=np.uint8).copy()


def unpack(packed: np.ndarray, d_out: int, d_in: int, N: int, M: int) -> np.ndarray:
    """Inverse of :func:`pack` (raises on an invalid code or slot count)."""
    crow, irow, total = packed_layout(d_out, d_in, N, M)
    assert packed.size == total
    K = 8 * N // M
    buf = packed.tobytes()
    w = np.zeros((d_out, d_in), dtype=np.int8)
    base = d_out * crow
    for o in range(d_out):
        codes = buf[o * crow:(o + 1) * crow]
        index = buf[base + o * irow: base + (o + 1) * irow]
        for c in range(d_in // 8):
            chunk_slots = []
            for g in range(c * 8 // M, (c + 1) * 8 // M):
                m = _get_bits(index, g * M, M)
                slots = [p for p in range(M) if (m >> p) & 1]
                if len(slots) != N:
                    raise ValueError(f"row {o} group {g}: {len(slots)} slots != N={N}")
                chunk_slots += [g * M + p - 8 * c for p in slots]
            for i, p in enumerate(chunk_slots):
                code = _get_bits(codes, 2 * K * c + _slot_bit(i, K), 2)
                if code not in _VALUE:
                    raise ValueError(f"row {o} chunk {c}: invalid code {code:#b}")
                w[o, 8 * c + p] = _VALUE[code]
    return w


# --------------------------------------------------------------------------
# Dense 2-bit ternary layout (a denser decode format)
# [article] 7.1 推理优化技巧 (a cached low-bit format for inference).  Every
# position keeps its 2-bit code and there is no index plane: for an N:M
# weight the dropped positions simply hold the code of 0.  Per row, d_in / 8
# chunks of 16 bits (little-endian halfwords, rows padded to 16 bytes); in a
# chunk the code of position q (q < 4) sits at bits 4q..4q+1 and the code of
# position q + 4 at bits 4q+2..4q+3 -- the chunk layout of the packed format
# with all eight positions as slots.  Codes as above: +1 00, -1 01, 0 10.
# --------------------------------------------------------------------------
def dense2_row_bytes(d_in: int) -> int:
    return _ceil16(d_in // 4)


def pack_dense2(weff: np.ndarray) -> np.ndarray:
    """W_eff (int8 in {-1, 0, 1}) -> dense 2-bit codes, [d_out, row bytes]."""
    d_out, d_in = weff.shape
    rb = dense2_row_bytes(d_in)
    out = bytearray(d_out * rb)
    for o in range(d_out):
        row = bytearray(rb)
        for pos in range(d_in):
            c, p = divmod(pos, 8)
            bit = 16 * c + (4 * p if p < 4 else 4 * (p - 4) + 2)
            _put_bits(row, bit, _CODE[int(weff[o, pos])], 2)
        out[o * rb:(o + 1) * rb] = row
    return np.frombuffer(bytes(out), dtype=np.uint8).copy()


def unpack_dense2(buf: np.ndarray, d_out: int, d_in: int) -> np.ndarray:
    """Inverse of :func:`pack_dense2` (raises on the unused code 11)."""
    rb = dense2_row_bytes(d_in)
    assert buf.size == d_out * rb
    data = buf.tobytes()
    w = np.zeros((d_out, d_in), dtype=np.int8)
    for o in range(d_out):
        row = data[o * rb:(o + 1) * rb]
        for pos in range(d_in):
            c, p = divmod(pos, 8)
            code = _get_bits(row, 16 * c + (4 * p if p < 4 else 4 * (p - 4) + 2), 2)
            if code not in _VALUE:
                raise ValueError(f"row {o} position {pos}: invalid code {code:#b}")
            w[o, pos] = _VALUE[code]
    return w


# --------------------------------------------------------------------------
# (a10) decode GEMV on the packed format
# [summary] 实验结果 / Table 3 (decode on the deployed 6:8 ternary model).
# --------------------------------------------------------------------------
def gemv_packed(xq: np.ndarray, amax: np.ndarray, packed: np.ndarray,
                gamma: np.float32, d_in: int, d_out: int, N: int, M: int) -> np.ndarray:
    """y = forward_out(X_q . unpack(packed)^T, gamma, amax)."""
    w = unpack(packed, d_out, d_in, N, M)
    return forward_out(forward_acc(xq, w), gamma, amax)


# --------------------------------------------------------------------------
# (a8) 2:4 compressed weight for the sparse tensor core
# [summary] 前置知识 / 半结构化 N:M 稀疏 (2:4 -- two kept of every four --
# is the pattern NVIDIA's sparse tensor cores accelerate) and 核心方法
# (masking after quantisation keeps the deployed weight N:M-structured so it
# can go to the sparse tensor core as it is).
#
# The format (this library's, the pages fix none) has two planes:
#   values plane: d_out rows of vrow = ceil16(d_in / 2) bytes; row o holds,
#     for every group g of four weights, the int8 values of its two slots in
#     ascending position order at bytes 2g and 2g + 1; bytes past d_in / 2
#     are zero;
#   selector plane (from the first 1024-byte boundary at or after the end
#     of the values plane): for every row and group a 4-bit selector
#     i0 | (i1 << 2), i0 < i1 the two slot positions.  It is tiled for the
#     tensor core: blocks of 128 rows x 256 weights (4096 bytes), block
#     (mb, kb) at (mb * KB + kb) * 4096; inside a block, two halves of 128
#     weights each (2048 bytes), row r of a half at 16 r, and the selector of
#     group j of that half in byte j // 2, low nibble for even j.  Rows are
#     padded to a multiple of 256 and weights to a multiple of 256; padding
#     groups get the selector of slots (0, 1) and zero values.
# Slots are the group's nonzero positions plus, if fewer than two, its
# lowest zero positions (the rule of the packed format above).
# --------------------------------------------------------------------------
SP24_PAD_NIBBLE = 0x4   # slots (0, 1)


def sparse24_layout(d_out: int, d_in: int):
    """(vrow, meta_off, total_bytes, KB, MB): values row bytes, selector-plane
    offset, buffer size, 256-weight blocks per row, 128-row blocks."""
    vrow = _ceil16(d_in // 2)
    KB = -(-d_in // 256)
    MB = 2 * (-(-d_out // 256))
    meta_off = -(-(d_out * vrow) // 1024) * 1024
    return vrow, meta_off, meta_off + MB * KB * 4096, KB, MB


def _selector_plane(nib: np.ndarray, KB: int, MB: int) -> np.ndarray:
    """Selector nibbles on the padded grid [MB * 128, KB * 64] -> the plane's
    bytes: two groups per byte (low nibble = even group), then the blocks of
    128 rows x 256 weights in (mb, kb) order, each as two halves of 128 rows
    x 16 bytes."""
    byte = (nib[:, 0::2] | (nib[:, 1::2] << 4)).astype(np.uint8)          # [MB*128, KB*32]
    blocks = byte.reshape(MB, 128, KB, 2, 16).transpose(0, 2, 3, 1, 4)    # mb, kb, half, r, q
    return np.ascontiguousarray(blocks).reshape(-1)


def _selector_grid(plane: np.ndarray, KB: int, MB: int) -> np.ndarray:
    """Inverse of :func:`_selector_plane`: nibbles [MB * 128, KB * 64]."""
    byte = plane.reshape(MB, KB, 2, 128, 16).transpose(0, 3, 1, 2, 4).reshape(MB * 128, KB * 32)
    nib = np.empty((MB * 128, KB * 64), dtype=np.uint8)
    nib[:, 0::2] = byte & 0xF
    nib[:, 1::2] = byte >> 4
    return nib


def compress24(weff: np.ndarray) -> np.ndarray:
    """W_eff (int8 [d_out, d_in], at most two nonzeros per group of four)
    -> the compressed buffer (uint8)."""
    d_out, d_in = weff.shape
    assert d_in % 4 == 0
    vrow, meta_off, total, KB, MB = sparse24_layout(d_out, d_in)
    G = d_in // 4
    grp = weff.reshape(d_out, G, 4).astype(np.int64)
    nz = grp != 0
    if (nz.sum(axis=-1) > 2).any():
        o, g = np.argwhere(nz.sum(axis=-1) > 2)[0]
        raise ValueError(f"row {o} group {g}: more than 2 nonzeros")
    # nonzero positions first, then zero positions, each by index; take two
    key = np.where(nz, 0, 4) + np.arange(4)
    slots = np.sort(np.argsort(key, axis=-1)[..., :2], axis=-1)      # [d_out, G, 2]
    vals = np.take_along_axis(grp, slots, axis=-1).astype(np.int8)    # [d_out, G, 2]
    out = np.zeros(total, dtype=np.uint8)
    vplane = np.zeros((d_out, vrow), dtype=np.uint8)
    vplane[:, :2 * G] = vals.reshape(d_out, 2 * G).view(np.uint8)
    out[:d_out * vrow] = vplane.reshape(-1)
    nib = np.full((MB * 128, KB * 64), SP24_PAD_NIBBLE, dtype=np.uint8)
    nib[:d_out, :G] = slots[..., 0] | (slots[..., 1] << 2)
    out[meta_off:] = _selector_plane(nib, KB, MB)
    return out


def _selectors(buf: np.ndarray, d_out: int, d_in: int):
    """(i0, i1) arrays [d_out, d_in / 4] read back from the selector plane."""
    vrow, meta_off, total, KB, MB = sparse24_layout(d_out, d_in)
    nib = _selector_grid(buf[meta_off:], KB, MB)[:d_out, :d_in // 4]
    return nib & 3, nib >> 2


def decompress24(buf: np.ndarray, d_out: int, d_in: int) -> np.ndarray:
    """Inverse of :func:`compress24` (raises on a selector with i0 >= i1)."""
    vrow, meta_off, total, KB, MB = sparse24_layout(d_out, d_in)
    assert buf.size == total
    G = d_in // 4
    i0, i1 = _selectors(buf, d_out, d_in)
    if (i0 >= i1).any():
        raise ValueError("selector with i0 >= i1")
    vals = buf[:d_out * vrow].reshape(d_out, vrow)[:, :2 * G].view(np.int8).reshape(d_out, G, 2)
    w = np.zeros((d_out, G, 4), dtype=np.int8)
    o_idx, g_idx = np.meshgrid(np.arange(d_out), np.arange(G), indexing="ij")
    w[o_idx, g_idx, i0] = vals[..., 0]
    w[o_idx, g_idx, i1] = vals[..., 1]
    return w.reshape(d_out, d_in)


def forward_acc_sparse24(xq: np.ndarray, buf: np.ndarray, d_out: int, d_in: int) -> np.ndarray:
    """acc[t, o] = sum_g sum_s value[o, g, s] * xq[t, 4 g + i_s[o, g]]: the
    product as a sparse tensor core forms it, from the two kept values of
    each group and the activations its selector picks (exact integers)."""
    vrow, meta_off, total, KB, MB = sparse24_layout(d_out, d_in)
    G = d_in // 4
    i0, i1 = _selectors(buf, d_out, d_in)
    vals = buf[:d_out * vrow].reshape(d_out, vrow)[:, :2 * G].view(np.int8).reshape(d_out, G, 2).astype(np.int64)
    xg = xq.astype(np.int64).reshape(xq.shape[0], G, 4)
    acc = np.zeros((xq.shape[0], d_out), dtype=np.int64)
    base = np.arange(G)
    for o in range(d_out):
        acc[:, o] = (xg[:, base, i0[o]] * vals[o, :, 0]).sum(axis=1) + (xg[:, base, i1[o]] * vals[o, :, 1]).sum(axis=1)
    return acc.astype(np.int32)


# --------------------------------------------------------------------------
# The optimizer step after the backward pass (AdamW on the master weight),
# gradient-norm clipping, and the mask flip count between consecutive steps.
# [summary] Algorithm 1 step (8) (AdamW, beta = (0.9, 0.95), eps = 1e-5,
# weight decay 0.1, grad clip 1.0, BF16 master weight W) and 局限与改进 /
# 独立分析的弱点 (the mask flip rate of Fig. 3b: how many mask entries change
# from one step to the next).
#
# Readings (the pages give only the hyperparameters):
# * AdamW is the decoupled-decay form with bias-corrected moments;
# * the per-step scalars are computed in fp64 from the hyperparameters and
#   rounded once to fp32:  alpha = lr / (1 - beta1^t),
#   b2s = sqrt(1 - beta2^t),  decay = 1 - lr * wd,  omb1 = 1 - beta1,
#   omb2 = 1 - beta2 (beta1, beta2, eps themselves rounded to fp32);
# * each element is updated with IEEE fp32 operations, in this order:
#     g  = dW * c                      (c: the clipping factor, fp32)
#     m' = beta1 * m + omb1 * g
#     v' = beta2 * v + (omb2 * g) * g
#     u  = m' / (sqrt(v') / b2s + eps)
#     w' = w * decay - alpha * u
#   every product, sum, quotient and square root rounded to fp32 on its own;
# * the master weight is either the bf16 W itself (the pages' "BF16 master
#   weight"; the new W is bf16_rn(w')) or an fp32 copy W32 kept beside it
#   (the new W32 is w' and the bf16 W becomes bf16_rn(w'));
# * clipping is by the global L2 norm of all gradients:
#   c = fl32(min(1, max_norm / (sqrt(S) + 1e-6))) with S the sum of squares
#   in fp64 and the sqrt and divide in fp64;
# * the flip count is the number of positions whose keep flag differs
#   between the mask of W before and the mask of W after the update.
# --------------------------------------------------------------------------
def grad_sqnorm(*grads: np.ndarray) -> float:
    """S = sum of g^2 over every element of every gradient, correctly
    rounded to fp64 (each fp32 square is exact in fp64; math.fsum rounds
    the exact sum once)."""
    parts = [np.square(np.asarray(g, np.float32).astype(np.float64)).ravel() for g in grads]
    return math.fsum(np.concatenate(parts)) if parts else 0.0


def grad_clip_scale(sumsq: float, max_norm: float) -> np.float32:
    """c = fl32(min(1, max_norm / (sqrt(S) + 1e-6))), in fp64."""
    return np.float32(min(1.0, float(max_norm) / (math.sqrt(float(sumsq)) + 1e-6)))


def adamw_scalars(lr: float, beta1: float, beta2: float, eps: float, weight_decay: float, step: int) -> dict:
    """The fp32 per-step scalars of AdamW at step t = step (t >= 1)."""
    t = int(step)
    f = np.float32
    return {
        "beta1": f(beta1), "beta2": f(beta2), "eps": f(eps),
        "omb1": f(1.0 - float(beta1)), "omb2": f(1.0 - float(beta2)),
        "alpha": f(float(lr) / (1.0 - float(beta1) ** t)),
        "b2s": f(math.sqrt(1.0 - float(beta2) ** t)),
        "decay": f(1.0 - float(lr) * float(weight_decay)),
    }


def adamw_update(w: np.ndarray, dw: np.ndarray, m: np.ndarray, v: np.ndarray, sc: dict,
                 clip: np.float32 = np.float32(1.0)):
    """One AdamW update of fp32 values w with gradient dw; returns
    (w', m', v') as fp32 arrays, each step rounded to fp32."""
    f32 = np.float32
    w = np.asarray(w, f32)
    g = np.multiply(np.asarray(dw, f32), f32(clip), dtype=f32)
    m1 = np.add(np.multiply(sc["beta1"], np.asarray(m, f32), dtype=f32),
                np.multiply(sc["omb1"], g, dtype=f32), dtype=f32)
    v1 = np.add(np.multiply(sc["beta2"], np.asarray(v, f32), dtype=f32),
                np.multiply(np.multiply(sc["omb2"], g, dtype=f32), g, dtype=f32), dtype=f32)
    den = np.add(np.divide(np.sqrt(v1, dtype=f32), sc["b2s"], dtype=f32), sc["eps"], dtype=f32)
    u = np.divide(m1, den, dtype=f32)
    w1 = np.subtract(np.multiply(w, sc["decay"], dtype=f32), np.multiply(sc["alpha"], u, dtype=f32), dtype=f32)
    return w1, m1, v1


def mask_flips(keep_before: np.ndarray, keep_after: np.ndarray) -> int:
    """Number of positions whose keep flag changed."""
    return int(np.count_nonzero(np.asarray(keep_before, bool) != np.asarray(keep_after, bool)))


def adamw_weight_step(w_bits: np.ndarray, dw: np.ndarray, m: np.ndarray, v: np.ndarray, N: int, M: int,
                      sc: dict, clip: np.float32 = np.float32(1.0), w32: np.ndarray | None = None):
    """Algorithm 1 step (8) followed by the next step's (2), (4), (5).

    Returns a dict with the new bf16 W bits, the new fp32 master (or None),
    m', v', and the next step's W_eff, gamma and keep-mask, plus the number
    of mask flips between the mask of the old W and that of the new W.
    """
    master = bf16_to_f32(w_bits) if w32 is None else np.asarray(w32, np.float32)
    w1, m1, v1 = adamw_update(master, dw, m, v, sc, clip)
    new_bits = f32_to_bf16(w1)
    weff, gamma, keep = effective_weight(new_bits, N, M)
    flips = mask_flips(nm_mask(w_bits, N, M), keep)
    return {"w_bits": new_bits, "w32": None if w32 is None else w1, "m": m1, "v": v1,
            "weff": weff, "gamma": gamma, "keep": keep, "flips": flips}
