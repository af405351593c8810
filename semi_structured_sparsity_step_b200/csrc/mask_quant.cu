// mask_quant.cu -- weight side of Sparse-BitLinear on sm_100a:
//   (a1) N:M magnitude mask, (a2) exact absmean scale gamma,
//   (a3) ternary quantiser and quant-then-mask.
//
// Sparse-BitNet summary ("Sparse-BitNet：1.58-bit 大模型天然兼容半结构化稀疏"):
//   前置知识 / 1.58-bit BitNet 量化 -- gamma = ||W||_1 / (d_out d_in),
//     W_q = RoundClip(W / gamma, -1, +1) (eps = 1e-5 in the denominator);
//   半结构化 N:M 稀疏, 核心方法 (i)-(iii), Algorithm 1 steps (2), (4), (5) --
//     keep the top-N of |W| in each group of M along d_in, every step, from
//     the bf16 master weight; W_eff = W_q (.) mask.
//
// Two launches over W (both memory bound, 128-bit loads):
//   1. gamma_reduce_kernel: exact sum of |W|.  A bf16 magnitude is
//      m * 2^(e - 134) with an 8-bit integer m and biased exponent e
//      (e := 1 for subnormals).  Magnitudes with e in [96, 128) (|w| in
//      [2^-31, 2)) are added exactly into a per-thread uint64 as
//      m << (e - 96); all others go to 256 per-exponent uint64 buckets
//      (shared-memory atomics, then global).  The last block to finish adds
//      the per-block window sums in 128 bits, folds everything into one
//      320-bit integer (unit 2^-133), rounds it once to fp64 (nearest-even),
//      divides by n in fp64 and rounds to fp32.  The result does not depend
//      on the order of the additions.  The ternary code only depends on
//      whether fp32(|w| / den) > 0.5 (den = fp32(gamma + 1e-5)), which is
//      monotone in |w|, so the same block also finds, by binary search with
//      the IEEE divide, the largest bf16 magnitude that still maps to 0 and
//      leaves it in the workspace.
//   2. ternary_mask_kernel: one thread per 8 weights (one uint4); each
//      ternary code is one integer compare against that threshold.  The
//      mask ranks the 15-bit magnitudes with the position as tie-break
//      (lower index wins), using pairwise compares in registers.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cmath>
#include <cstdint>
#include <mutex>

#include "../../include/sbl.h"
#include "sbl_device.cuh"
#include "sbl_internal.h"

namespace sbl {
namespace {

constexpr int kGammaThreads = 256;
constexpr int kWinLo = 96;  // window exponents [96, 128)

__device__ __forceinline__ void gamma_add_bf16(uint32_t h, uint64_t& acc, unsigned long long* sbucket) {
  const uint32_t e = (h >> 7) & 0xFFu;
  const uint32_t m = (h & 0x7Fu) | (e ? 0x80u : 0u);
  const uint32_t ee = e ? e : 1u;
  if (ee - kWinLo < 32u) {
    acc += static_cast<uint64_t>(m) << (ee - kWinLo);
  } else if (m != 0u) {
    atomicAdd(&sbucket[ee], static_cast<unsigned long long>(m));
  }
}

// Same split as gamma_add_bf16, with the in-window magnitude added to an fp64
// partial sum (exact: see gamma_reduce_kernel).
__device__ __forceinline__ void gamma_add_bf16_f64(uint32_t h, double& dacc, unsigned long long* sbucket) {
  const uint32_t mag = h & 0x7FFFu;
  if (mag - (static_cast<uint32_t>(kWinLo) << 7) < (32u << 7)) {
    dacc += static_cast<double>(__uint_as_float(mag << 16));
  } else {
    const uint32_t e = mag >> 7;
    const uint32_t m = (mag & 0x7Fu) | (e ? 0x80u : 0u);
    if (m != 0u) atomicAdd(&sbucket[e ? e : 1u], static_cast<unsigned long long>(m));
  }
}

// limbs (10 x 32 bit, little-endian) += v << shift, 0 <= shift < 256.
__device__ void bigint_add_shifted(uint32_t* limbs, uint64_t v, int shift) {
  if (v == 0) return;
  const int li = shift >> 5;
  const int off = shift & 31;
  const unsigned __int128 x = static_cast<unsigned __int128>(v) << off;
  uint32_t w[3] = {static_cast<uint32_t>(x), static_cast<uint32_t>(x >> 32), static_cast<uint32_t>(x >> 64)};
  uint64_t carry = 0;
  for (int i = li; i < kGammaLimbs; ++i) {
    const uint64_t add = (i - li < 3) ? w[i - li] : 0u;
    const uint64_t s = static_cast<uint64_t>(limbs[i]) + add + carry;
    limbs[i] = static_cast<uint32_t>(s);
    carry = s >> 32;
    if (i - li >= 2 && carry == 0) break;
  }
}

// Correctly rounded (nearest-even) fp64 value of limbs * 2^-133.
__device__ double bigint_to_double(const uint32_t* limbs) {
  int L = kGammaLimbs - 1;
  while (L >= 0 && limbs[L] == 0u) --L;
  if (L < 0) return 0.0;
  const int top = 32 * L + (31 - __clz(limbs[L]));  // index of the leading one
  // 96-bit window of limbs L, L-1, L-2 (missing limbs read as 0).
  const uint32_t l1 = L >= 1 ? limbs[L - 1] : 0u;
  const uint32_t l2 = L >= 2 ? limbs[L - 2] : 0u;
  const unsigned __int128 v = (static_cast<unsigned __int128>(limbs[L]) << 64) |
                              (static_cast<unsigned __int128>(l1) << 32) | l2;
  const int p = 64 + (31 - __clz(limbs[L]));        // leading one inside the window
  const int sh = p - 63;                             // 1..32
  const uint64_t mant64 = static_cast<uint64_t>(v >> sh);  // bits [top-63, top]
  bool sticky = (v & ((static_cast<unsigned __int128>(1) << sh) - 1)) != 0;
  for (int i = 0; i < L - 2; ++i) sticky |= limbs[i] != 0u;
  uint64_t mant = mant64 >> 11;                      // 53 bits
  const uint32_t rest = static_cast<uint32_t>(mant64 & 0x7FFu);
  sticky |= (rest & 0x3FFu) != 0u;
  int exp2 = top - 52;
  if ((rest & 0x400u) && (sticky || (mant & 1ull))) {
    mant += 1;
    if (mant == (1ull << 53)) {
      mant >>= 1;
      exp2 += 1;
    }
  }
  return scalbn(static_cast<double>(mant), exp2 - 133);
}

// Largest bf16 magnitude pattern b (0 <= b < 0x7F80) with fp32(bf16(b) / den) <= 0.5.
// fp32(|w| / den) is monotone in |w|, so W_q = 0 exactly when |w|'s pattern <= b.
__device__ uint32_t zero_threshold_bits_serial(float den) {
  uint32_t lo = 0u, hi = 0x7F80u;  // cond(lo) holds; cond(hi) fails (inf)
  while (hi - lo > 1u) {
    const uint32_t mid = (lo + hi) >> 1;
    const float v = __uint_as_float(mid << 16);
    if (__fdiv_rn(v, den) <= 0.5f) lo = mid; else hi = mid;
  }
  return lo;
}

// The same threshold found by one warp: the boundary lies within a bf16 ulp
// of den / 2, so the 32 lanes test the 32 patterns around it with the IEEE
// divide at once and the boundary is the last lane that passes.  If the
// window does not bracket the boundary (not expected), lane 0 falls back to
// the serial search.  Must be called by all 32 lanes; returns in every lane.
__device__ uint32_t zero_threshold_bits_warp(float den) {
  const uint32_t lane = threadIdx.x & 31u;
  const uint32_t centre = __float_as_uint(__fmul_rn(den, 0.5f)) >> 16;  // truncated to bf16
  const int base = static_cast<int>(centre) - 16;
  const int cand = base + static_cast<int>(lane);
  bool ok = false;
  if (cand >= 0 && cand < 0x7F80) ok = __fdiv_rn(__uint_as_float(static_cast<uint32_t>(cand) << 16), den) <= 0.5f;
  const uint32_t pass = __ballot_sync(0xFFFFFFFFu, ok);
  uint32_t thr;
  const bool bracketed = (pass & 1u) && !(pass >> 31) && ((pass & (pass + 1u)) == 0u);  // a prefix 0..k, k < 31
  if (bracketed) {
    thr = static_cast<uint32_t>(base + (31 - __clz(pass)));
  } else {
    thr = lane == 0 ? zero_threshold_bits_serial(den) : 0u;
    thr = __shfl_sync(0xFFFFFFFFu, thr, 0);
  }
  return thr;
}

// End of an exact gamma pass, called by every thread of each block (256
// threads) once its share of W has been added: `acc` is the thread's window
// sum (units of 2^-38), `sbucket` the block's shared exponent buckets.  The
// block's partials go to the workspace; the last block to finish adds all
// partials exactly (320-bit integer), writes gamma = fp32(fp64(sum) / n) and
// the zero threshold of the ternary quantiser into the workspace.
__device__ void gamma_block_done(uint64_t acc, unsigned long long* sbucket, GammaWorkspace* ws, size_t n_elems,
                                 float* __restrict__ gamma_out) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xFFFFFFFFu, acc, o);
  __shared__ uint64_t swarp[kGammaThreads / 32];
  __shared__ int s_last;
  if ((threadIdx.x & 31) == 0) swarp[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    uint64_t s = 0;
    for (int w = 0; w < kGammaThreads / 32; ++w) s += swarp[w];
    ws->block_window[blockIdx.x] = s;
  }
  if (sbucket[threadIdx.x] != 0ull) atomicAdd(&ws->bucket[threadIdx.x], sbucket[threadIdx.x]);
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) s_last = (atomicAdd(&ws->ticket, 1u) == gridDim.x - 1);
  __syncthreads();
  if (!s_last) return;
  __threadfence();

  // Last block: 128-bit sum of the per-block window sums, one lane per
  // partial, then a shuffle tree; carries are tracked in the high word.
  __shared__ uint64_t s_lo[kGammaThreads / 32], s_hi[kGammaThreads / 32];
  __shared__ uint32_t s_occ[256 / 32];
  __shared__ float s_gamma;
  uint64_t lo = 0, hi = 0;
  for (unsigned b = threadIdx.x; b < gridDim.x; b += blockDim.x) {
    const uint64_t p = __ldcg(&ws->block_window[b]);
    lo += p;
    hi += (lo < p) ? 1u : 0u;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const uint64_t olo = __shfl_xor_sync(0xFFFFFFFFu, lo, o);
    const uint64_t ohi = __shfl_xor_sync(0xFFFFFFFFu, hi, o);
    lo += olo;
    hi += ohi + ((lo < olo) ? 1u : 0u);
  }
  const uint64_t bucket = __ldcg(&ws->bucket[threadIdx.x]);
  sbucket[threadIdx.x] = bucket;
  const uint32_t occ = __ballot_sync(0xFFFFFFFFu, bucket != 0ull);
  if ((threadIdx.x & 31) == 0) {
    s_lo[threadIdx.x >> 5] = lo;
    s_hi[threadIdx.x >> 5] = hi;
    s_occ[threadIdx.x >> 5] = occ;
  }
  __syncthreads();
  if (threadIdx.x < 32) {
    if (threadIdx.x == 0) {
      lo = 0;
      hi = 0;
      for (int w = 0; w < kGammaThreads / 32; ++w) {
        lo += s_lo[w];
        hi += s_hi[w] + ((lo < s_lo[w]) ? 1u : 0u);
      }
      uint32_t limbs[kGammaLimbs];
#pragma unroll
      for (int i = 0; i < kGammaLimbs; ++i) limbs[i] = 0u;
      // value = m * 2^(ee-134) = m * 2^(ee-1) units of 2^-133; window sums carry 2^(96-1).
      bigint_add_shifted(limbs, lo, kWinLo - 1);
      bigint_add_shifted(limbs, hi, kWinLo - 1 + 64);
      for (int w = 0; w < 256 / 32; ++w) {
        uint32_t m = s_occ[w];
        while (m != 0u) {  // only the occupied exponent buckets
          const int ee = 32 * w + (__ffs(m) - 1);
          m &= m - 1u;
          if (ee >= 1) bigint_add_shifted(limbs, sbucket[ee], ee - 1);
        }
      }
      const double total = bigint_to_double(limbs);
      const double mean = __ddiv_rn(total, static_cast<double>(n_elems));
      s_gamma = __double2float_rn(mean);
      *gamma_out = s_gamma;
    }
    __syncwarp();
    const uint32_t thr = zero_threshold_bits_warp(__fadd_rn(s_gamma, 1e-5f));
    if (threadIdx.x == 0) ws->zero_threshold = thr;
  }
}

__global__ void __launch_bounds__(kGammaThreads) gamma_reduce_kernel(const uint4* __restrict__ W, size_t n_vec,
                                                                      size_t n_elems, GammaWorkspace* ws,
                                                                      float* __restrict__ gamma_out) {
  __shared__ unsigned long long sbucket[256];
  sbucket[threadIdx.x] = 0ull;
  __syncthreads();

  // In-window magnitudes (|w| in [2^-31, 2), bf16 pattern in [0x3000, 0x4000))
  // are added as fp64: each is a multiple of 2^-38 below 2, so a sum of up to
  // 512 of them stays below 2^10 and needs at most 48 significant bits --
  // every fp64 addition is exact.  The partial sum is moved into the uint64
  // `acc` (units of 2^-38) every 512 elements.
  uint64_t acc = 0;
  const size_t stride = static_cast<size_t>(gridDim.x) * blockDim.x;
  size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x;
  while (i + 3 * stride < n_vec) {
    double dacc = 0.0;
    for (int rep = 0; rep < 16 && i + 3 * stride < n_vec; ++rep, i += 4 * stride) {  // 16 x 32 elements
      uint4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) v[u] = __ldg(W + i + u * stride);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const uint32_t w4[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          gamma_add_bf16_f64(w4[k] & 0xFFFFu, dacc, sbucket);
          gamma_add_bf16_f64(w4[k] >> 16, dacc, sbucket);
        }
      }
    }
    acc += static_cast<uint64_t>(scalbn(dacc, 38));
  }
  for (; i < n_vec; i += stride) {
    const uint4 v = __ldg(W + i);
    const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      gamma_add_bf16(w4[k] & 0xFFFFu, acc, sbucket);
      gamma_add_bf16(w4[k] >> 16, acc, sbucket);
    }
  }
  gamma_block_done(acc, sbucket, ws, n_elems, gamma_out);
}


// Keep flags of one group of M positions (bit j = position j).  Each
// position gets the key (|w| pattern << 3) | (M-1-j): all keys of a group
// differ, and a larger key means "kept first" (larger magnitude, then lower
// index).  The group keeps its N largest keys.  Whichever side is smaller is
// selected by repeated minimum/maximum reductions: with d = M - N <= N the d
// smallest keys are dropped, otherwise the N largest are kept.  Subtracting
// (last + 1) with unsigned wrap-around moves the keys already taken to the
// top (for the minimum) so each round is one sub and one min per key.
template <int M, int N>
__device__ __forceinline__ uint32_t keep_group(const uint32_t (&key)[M]) {
  constexpr int d = M - N;
  if constexpr (d == 0) return (1u << M) - 1u;
  if constexpr (d <= N) {
    uint32_t dropped = 0u, last = 0u;
#pragma unroll
    for (int r = 0; r < d; ++r) {
      const uint32_t off = r == 0 ? 0u : last + 1u;
      uint32_t mn = 0xFFFFFFFFu;
#pragma unroll
      for (int j = 0; j < M; ++j) mn = min(mn, key[j] - off);
      last = mn + off;
      dropped |= 1u << (M - 1 - static_cast<int>(last & 7u));
    }
    return ((1u << M) - 1u) & ~dropped;
  }
  uint32_t kept = 0u, last = 0xFFFFFFFFu;
#pragma unroll
  for (int r = 0; r < N; ++r) {
    uint32_t mx = 0u;
#pragma unroll
    for (int j = 0; j < M; ++j) mx = max(mx, key[j] < last ? key[j] : 0u);
    last = mx;
    kept |= 1u << (M - 1 - static_cast<int>(mx & 7u));
  }
  return kept;
}

// FROMQ (an ablation): the mask keys use whether the ternary code is nonzero
// instead of the magnitude, so the mask is the top-N of |W_q|, ties to the
// lowest index.
template <int M, int N, bool FROMQ>
__global__ void __launch_bounds__(256) ternary_mask_kernel(const uint4* __restrict__ W, size_t n_vec,
                                                           const GammaWorkspace* __restrict__ ws,
                                                           uint2* __restrict__ w_eff,
                                                           uint4* __restrict__ w_eff_bf16,
                                                           uint8_t* __restrict__ mask_bits) {
  const uint32_t thr = ws->zero_threshold;
  const uint32_t thr2 = thr | (thr << 16);
  auto one = [&](size_t i, const uint4 v) {
    const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
    // ---- N:M mask from the 15-bit magnitudes
    uint32_t keep = 0u;
#pragma unroll
    for (int g = 0; g < 8 / M; ++g) {
      uint32_t key[M];
#pragma unroll
      for (int j = 0; j < M; ++j) {
        const int pos = g * M + j;
        uint32_t h = (w4[pos >> 1] >> (16 * (pos & 1))) & 0x7FFFu;
        if constexpr (FROMQ) h = h > thr ? 1u : 0u;  // |W_q|
        key[j] = (h << 3) | static_cast<uint32_t>(M - 1 - j);
      }
      keep |= keep_group<M, N>(key) << (g * M);
    }
    // ---- ternary codes, two bf16 per 32-bit word
    uint32_t qb[4], q16[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const uint32_t mag = w4[k] & 0x7FFF7FFFu;
      const uint32_t gt = __vcmpgtu2(mag, thr2);                           // 0xFFFF where |w| maps to +-1
      const uint32_t kb = (keep >> (2 * k)) & 3u;
      const uint32_t kh = ((kb & 1u) | ((kb & 2u) << 15)) * 0xFFFFu;        // keep flags as 16-bit lanes
      const uint32_t nz = gt & kh;
      const uint32_t neg = ((w4[k] >> 15) & 0x00010001u) * 0xFFFFu;         // sign as 16-bit lanes
      qb[k] = nz & (0x3F803F80u | (w4[k] & 0x80008000u));                  // +-1.0 in bf16
      q16[k] = nz & (0x00010001u | neg);                                   // +-1 in int16 lanes
    }
    w_eff[i] = make_uint2(__byte_perm(q16[0], q16[1], 0x6420), __byte_perm(q16[2], q16[3], 0x6420));
    if (w_eff_bf16 != nullptr) w_eff_bf16[i] = make_uint4(qb[0], qb[1], qb[2], qb[3]);
    if (mask_bits != nullptr) mask_bits[i] = static_cast<uint8_t>(keep);
  };
  // two vectors per thread and iteration, both loads issued first
  const size_t stride = static_cast<size_t>(gridDim.x) * blockDim.x;
  size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x;
  for (; i + stride < n_vec; i += 2 * stride) {
    const uint4 v0 = __ldg(W + i), v1 = __ldg(W + i + stride);
    one(i, v0);
    one(i + stride, v1);
  }
  if (i < n_vec) one(i, __ldg(W + i));
}

// ---------------------------------------------------------------------------
// The optimizer step fused with the first pass of the next weight step.
// Sparse-BitNet summary, Algorithm 1 step (8): AdamW on the bf16 master
// weight (beta = (0.9, 0.95), eps = 1e-5, weight decay 0.1, grad clip 1.0),
// and 独立分析的弱点 (the mask flip rate of Fig. 3b).
//
// One thread per 8 weights: it loads the master values (8 bf16, or 8 fp32
// when an fp32 copy is kept), 8 fp32 gradients and both fp32 moments,
// updates them with IEEE fp32 operations in a fixed order (no contraction):
//   g = dW * c;  m' = b1 m + (1 - b1) g;  v' = b2 v + ((1 - b2) g) g;
//   w' = w * (1 - lr wd) - alpha * (m' / (sqrt(v') / sqrt(1 - b2^t) + eps)),
// alpha = lr / (1 - b1^t), stores them, rounds w' to bf16 (nearest even),
// and from the new bf16 values adds |W'| to the exact gamma sum (the same
// integer windows and buckets as gamma_reduce_kernel) and, when asked,
// counts the positions whose N:M keep flag differs from the mask stored for
// the old W.  The last block finishes gamma and the ternary threshold, so
// the next launch is the ternary pass alone: the update and the next step's
// gamma pass share one read of W.
struct AdamwScalars {
  float beta1, beta2, omb1, omb2, eps, alpha, b2s, decay;
  double max_norm;  // clipping bound (used when a squared norm is given)
};

template <int M, int N, bool MASTER32>
__global__ void __launch_bounds__(kGammaThreads) adamw_gamma_kernel(
    uint4* __restrict__ W, float4* __restrict__ W32, const float4* __restrict__ dW, float4* __restrict__ m,
    float4* __restrict__ v, const uint8_t* __restrict__ old_bits, size_t n_vec, size_t n_elems, AdamwScalars sc,
    const double* __restrict__ sumsq, GammaWorkspace* ws, float* __restrict__ gamma_out,
    unsigned long long* __restrict__ flips) {
  __shared__ unsigned long long sbucket[256];
  sbucket[threadIdx.x] = 0ull;
  __syncthreads();
  // clipping factor c = fl32(min(1, max_norm / (sqrt(S) + 1e-6))), in fp64
  float c = 1.0f;
  if (sumsq != nullptr) {
    const double q = __ddiv_rn(sc.max_norm, __dadd_rn(__dsqrt_rn(*sumsq), 1e-6));
    c = q < 1.0 ? __double2float_rn(q) : 1.0f;
  }
  uint64_t acc = 0;
  uint32_t nflip = 0;
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n_vec;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    float w[8], g[8], mv[8], vv[8];
    {
      const float4 g0 = __ldcs(dW + 2 * i), g1 = __ldcs(dW + 2 * i + 1);
      const float4 m0 = __ldcs(m + 2 * i), m1 = __ldcs(m + 2 * i + 1);
      const float4 v0 = __ldcs(v + 2 * i), v1 = __ldcs(v + 2 * i + 1);
      g[0] = g0.x; g[1] = g0.y; g[2] = g0.z; g[3] = g0.w; g[4] = g1.x; g[5] = g1.y; g[6] = g1.z; g[7] = g1.w;
      mv[0] = m0.x; mv[1] = m0.y; mv[2] = m0.z; mv[3] = m0.w; mv[4] = m1.x; mv[5] = m1.y; mv[6] = m1.z; mv[7] = m1.w;
      vv[0] = v0.x; vv[1] = v0.y; vv[2] = v0.z; vv[3] = v0.w; vv[4] = v1.x; vv[5] = v1.y; vv[6] = v1.z; vv[7] = v1.w;
      if constexpr (MASTER32) {
        const float4 a = __ldcs(W32 + 2 * i), b = __ldcs(W32 + 2 * i + 1);
        w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w; w[4] = b.x; w[5] = b.y; w[6] = b.z; w[7] = b.w;
      } else {
        const uint4 q = W[i];
        const uint32_t q4[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          w[2 * k] = __uint_as_float(q4[k] << 16);
          w[2 * k + 1] = __uint_as_float(q4[k] & 0xFFFF0000u);
        }
      }
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const float gk = __fmul_rn(g[k], c);
      mv[k] = __fadd_rn(__fmul_rn(sc.beta1, mv[k]), __fmul_rn(sc.omb1, gk));
      vv[k] = __fadd_rn(__fmul_rn(sc.beta2, vv[k]), __fmul_rn(__fmul_rn(sc.omb2, gk), gk));
      const float den = __fadd_rn(__fdiv_rn(__fsqrt_rn(vv[k]), sc.b2s), sc.eps);
      w[k] = __fsub_rn(__fmul_rn(w[k], sc.decay), __fmul_rn(sc.alpha, __fdiv_rn(mv[k], den)));
    }
    __stcs(m + 2 * i, make_float4(mv[0], mv[1], mv[2], mv[3]));
    __stcs(m + 2 * i + 1, make_float4(mv[4], mv[5], mv[6], mv[7]));
    __stcs(v + 2 * i, make_float4(vv[0], vv[1], vv[2], vv[3]));
    __stcs(v + 2 * i + 1, make_float4(vv[4], vv[5], vv[6], vv[7]));
    if constexpr (MASTER32) {
      __stcs(W32 + 2 * i, make_float4(w[0], w[1], w[2], w[3]));
      __stcs(W32 + 2 * i + 1, make_float4(w[4], w[5], w[6], w[7]));
    }
    uint32_t nb[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const __nv_bfloat162 p = __floats2bfloat162_rn(w[2 * k], w[2 * k + 1]);
      nb[k] = *reinterpret_cast<const uint32_t*>(&p);
    }
    W[i] = make_uint4(nb[0], nb[1], nb[2], nb[3]);  // kept in L2 for the ternary pass
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      gamma_add_bf16(nb[k] & 0xFFFFu, acc, sbucket);
      gamma_add_bf16(nb[k] >> 16, acc, sbucket);
    }
    if (old_bits != nullptr) {
      uint32_t keep = 0u;
#pragma unroll
      for (int gi = 0; gi < 8 / M; ++gi) {
        uint32_t key[M];
#pragma unroll
        for (int j = 0; j < M; ++j) {
          const int pos = gi * M + j;
          const uint32_t h = (nb[pos >> 1] >> (16 * (pos & 1))) & 0x7FFFu;
          key[j] = (h << 3) | static_cast<uint32_t>(M - 1 - j);
        }
        keep |= keep_group<M, N>(key) << (gi * M);
      }
      nflip += __popc((keep ^ static_cast<uint32_t>(old_bits[i])) & 0xFFu);
    }
  }
  if (old_bits != nullptr) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) nflip += __shfl_xor_sync(0xFFFFFFFFu, nflip, o);
    if ((threadIdx.x & 31) == 0 && nflip != 0u) atomicAdd(flips, static_cast<unsigned long long>(nflip));
  }
  gamma_block_done(acc, sbucket, ws, n_elems, gamma_out);
}

// Sum of squares of an fp32 gradient in fp64 (each square is exact in fp64),
// added to *sumsq.  Each block sums a fixed grid-stride share and the last
// block adds the per-block partials in block order, so the result depends
// only on n and the grid, not on scheduling.
__global__ void __launch_bounds__(kGammaThreads) grad_sqnorm_kernel(const float4* __restrict__ g, size_t n4,
                                                                    const float* __restrict__ tail, int n_tail,
                                                                    GammaWorkspace* ws, double* sumsq) {
  __shared__ double s_w[kGammaThreads / 32];
  // four independent 16-byte loads in flight per thread, two accumulators
  const size_t stride = static_cast<size_t>(gridDim.x) * blockDim.x;
  size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x;
  double s0 = 0.0, s1 = 0.0;
  for (; i + 3 * stride < n4; i += 4 * stride) {
    float4 a[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) a[u] = __ldcs(g + i + u * stride);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      s0 = fma(static_cast<double>(a[u].x), static_cast<double>(a[u].x), s0);
      s1 = fma(static_cast<double>(a[u].y), static_cast<double>(a[u].y), s1);
      s0 = fma(static_cast<double>(a[u].z), static_cast<double>(a[u].z), s0);
      s1 = fma(static_cast<double>(a[u].w), static_cast<double>(a[u].w), s1);
    }
  }
  for (; i < n4; i += stride) {
    const float4 a = __ldcs(g + i);
    s0 = fma(static_cast<double>(a.x), static_cast<double>(a.x), s0);
    s1 = fma(static_cast<double>(a.y), static_cast<double>(a.y), s1);
    s0 = fma(static_cast<double>(a.z), static_cast<double>(a.z), s0);
    s1 = fma(static_cast<double>(a.w), static_cast<double>(a.w), s1);
  }
  double s = s0 + s1;
  if (blockIdx.x == 0 && static_cast<int>(threadIdx.x) < n_tail) {
    const double t = static_cast<double>(tail[threadIdx.x]);
    s = fma(t, t, s);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xFFFFFFFFu, s, o);
  if ((threadIdx.x & 31) == 0) s_w[threadIdx.x >> 5] = s;
  __syncthreads();
  double* part = reinterpret_cast<double*>(ws->block_window);
  __shared__ int s_last;
  if (threadIdx.x == 0) {
    double b = 0.0;
    for (int w = 0; w < kGammaThreads / 32; ++w) b += s_w[w];
    part[blockIdx.x] = b;
    __threadfence();
    s_last = atomicAdd(&ws->ticket, 1u) == gridDim.x - 1;
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  // last block: the partials in a fixed tree (thread k takes k, k + 256, ...;
  // then the butterfly and the warps in order), so the sum does not depend
  // on which block finished last
  double t = 0.0;
  for (unsigned k = threadIdx.x; k < gridDim.x; k += blockDim.x) t += __ldcg(part + k);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xFFFFFFFFu, t, o);
  if ((threadIdx.x & 31) == 0) s_w[threadIdx.x >> 5] = t;
  __syncthreads();
  if (threadIdx.x == 0) {
    double u = 0.0;
    for (int w = 0; w < kGammaThreads / 32; ++w) u += s_w[w];
    *sumsq += u;
  }
}

}  // namespace

size_t mask_quant_workspace_bytes() { return sizeof(GammaWorkspace); }

// The second pass of the weight step (ternary codes, W_eff, mask) for a W
// whose gamma pass has left its threshold in ws.
static cudaError_t launch_ternary(const void* W, size_t n_vec, int N, int M, const GammaWorkspace* ws,
                                  int8_t* W_eff, void* W_eff_bf16, uint8_t* mask_bits, bool from_quantised,
                                  cudaStream_t stream, int num_sms) {
  size_t qblocks = (n_vec + 255) / 256;
  const size_t qmax = static_cast<size_t>(num_sms) * 8;
  if (qblocks > qmax) qblocks = qmax;
  if (qblocks < 1) qblocks = 1;
  const unsigned qb = static_cast<unsigned>(qblocks);
  const uint4* w4 = static_cast<const uint4*>(W);
  uint2* we = reinterpret_cast<uint2*>(W_eff);
  uint4* wb = static_cast<uint4*>(W_eff_bf16);
#define SBL_TERNARY(MM, NN)                                                                   \
  (from_quantised ? ternary_mask_kernel<MM, NN, true><<<qb, 256, 0, stream>>>(w4, n_vec, ws, we, wb, mask_bits) \
                  : ternary_mask_kernel<MM, NN, false><<<qb, 256, 0, stream>>>(w4, n_vec, ws, we, wb, mask_bits))
  if (M == 8) {
    switch (N) {
      case 1: SBL_TERNARY(8, 1); break;
      case 2: SBL_TERNARY(8, 2); break;
      case 3: SBL_TERNARY(8, 3); break;
      case 4: SBL_TERNARY(8, 4); break;
      case 5: SBL_TERNARY(8, 5); break;
      case 6: SBL_TERNARY(8, 6); break;
      case 7: SBL_TERNARY(8, 7); break;
      default: SBL_TERNARY(8, 8); break;
    }
  } else {
    switch (N) {
      case 1: SBL_TERNARY(4, 1); break;
      case 2: SBL_TERNARY(4, 2); break;
      case 3: SBL_TERNARY(4, 3); break;
      default: SBL_TERNARY(4, 4); break;
    }
  }
#undef SBL_TERNARY
  return cudaGetLastError();
}

cudaError_t launch_mask_quant(const void* W, int d_out, int d_in, int N, int M, int8_t* W_eff, void* W_eff_bf16,
                              uint8_t* mask_bits, float* gamma, void* workspace, cudaStream_t stream,
                              int num_sms, bool from_quantised) {
  const size_t n = static_cast<size_t>(d_out) * d_in;
  const size_t n_vec = n / 8;
  auto* ws = static_cast<GammaWorkspace*>(workspace);
  cudaError_t e = cudaMemsetAsync(ws, 0, offsetof(GammaWorkspace, block_window), stream);
  if (e != cudaSuccess) return e;
  int blocks = static_cast<int>((n_vec + kGammaThreads - 1) / kGammaThreads);
  if (blocks > kGammaMaxBlocks) blocks = kGammaMaxBlocks;
  if (blocks < 1) blocks = 1;
  (void)num_sms;
  gamma_reduce_kernel<<<blocks, kGammaThreads, 0, stream>>>(static_cast<const uint4*>(W), n_vec, n, ws, gamma);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_ternary(W, n_vec, N, M, ws, W_eff, W_eff_bf16, mask_bits, from_quantised, stream, num_sms);
}

// fp32 per-step scalars of AdamW, computed in fp64 from the hyperparameters
// and rounded once each (beta^t by the C library's pow).
static AdamwScalars adamw_scalars(const AdamwParams& p) {
  AdamwScalars sc;
  const double t = static_cast<double>(p.step);
  sc.beta1 = static_cast<float>(p.beta1);
  sc.beta2 = static_cast<float>(p.beta2);
  sc.omb1 = static_cast<float>(1.0 - p.beta1);
  sc.omb2 = static_cast<float>(1.0 - p.beta2);
  sc.eps = static_cast<float>(p.eps);
  sc.alpha = static_cast<float>(p.lr / (1.0 - std::pow(p.beta1, t)));
  sc.b2s = static_cast<float>(std::sqrt(1.0 - std::pow(p.beta2, t)));
  sc.decay = static_cast<float>(1.0 - p.lr * p.weight_decay);
  sc.max_norm = p.max_norm;
  return sc;
}

template <int M, int N>
static void adamw_launch_mn(bool master32, unsigned blocks, cudaStream_t stream, uint4* W, float4* W32,
                            const float4* dW, float4* m, float4* v, const uint8_t* old_bits, size_t n_vec,
                            size_t n, const AdamwScalars& sc, const double* sumsq, GammaWorkspace* ws,
                            float* gamma, unsigned long long* flips) {
  if (master32)
    adamw_gamma_kernel<M, N, true><<<blocks, kGammaThreads, 0, stream>>>(W, W32, dW, m, v, old_bits, n_vec, n, sc,
                                                                          sumsq, ws, gamma, flips);
  else
    adamw_gamma_kernel<M, N, false><<<blocks, kGammaThreads, 0, stream>>>(W, W32, dW, m, v, old_bits, n_vec, n, sc,
                                                                           sumsq, ws, gamma, flips);
}

cudaError_t launch_adamw_step(void* W, float* W32, const float* dW, float* m, float* v, int d_out, int d_in, int N,
                              int M, const AdamwParams& hp, const double* grad_sqnorm, int8_t* W_eff,
                              void* W_eff_bf16, uint8_t* mask_bits, float* gamma, unsigned long long* flips,
                              void* workspace, cudaStream_t stream, int num_sms) {
  const size_t n = static_cast<size_t>(d_out) * d_in;
  const size_t n_vec = n / 8;
  auto* ws = static_cast<GammaWorkspace*>(workspace);
  cudaError_t e = cudaMemsetAsync(ws, 0, offsetof(GammaWorkspace, block_window), stream);
  if (e != cudaSuccess) return e;
  int blocks = static_cast<int>((n_vec + kGammaThreads - 1) / kGammaThreads);
  if (blocks > kGammaMaxBlocks) blocks = kGammaMaxBlocks;
  if (blocks < 1) blocks = 1;
  const AdamwScalars sc = adamw_scalars(hp);
  const uint8_t* old_bits = flips != nullptr ? mask_bits : nullptr;
  auto* w4 = static_cast<uint4*>(W);
  auto* w32 = reinterpret_cast<float4*>(W32);
  auto* g4 = reinterpret_cast<const float4*>(dW);
  auto* m4 = reinterpret_cast<float4*>(m);
  auto* v4 = reinterpret_cast<float4*>(v);
  const bool master32 = W32 != nullptr;
  const unsigned ub = static_cast<unsigned>(blocks);
#define SBL_ADAMW(MM, NN) \
  adamw_launch_mn<MM, NN>(master32, ub, stream, w4, w32, g4, m4, v4, old_bits, n_vec, n, sc, grad_sqnorm, ws, gamma, flips)
  if (M == 8) {
    switch (N) {
      case 1: SBL_ADAMW(8, 1); break;
      case 2: SBL_ADAMW(8, 2); break;
      case 3: SBL_ADAMW(8, 3); break;
      case 4: SBL_ADAMW(8, 4); break;
      case 5: SBL_ADAMW(8, 5); break;
      case 6: SBL_ADAMW(8, 6); break;
      case 7: SBL_ADAMW(8, 7); break;
      default: SBL_ADAMW(8, 8); break;
    }
  } else {
    switch (N) {
      case 1: SBL_ADAMW(4, 1); break;
      case 2: SBL_ADAMW(4, 2); break;
      case 3: SBL_ADAMW(4, 3); break;
      default: SBL_ADAMW(4, 4); break;
    }
  }
#undef SBL_ADAMW
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_ternary(W, n_vec, N, M, ws, W_eff, W_eff_bf16, mask_bits, false, stream, num_sms);
}

cudaError_t launch_grad_sqnorm(const float* g, size_t n, double* sumsq, void* workspace, cudaStream_t stream) {
  auto* ws = static_cast<GammaWorkspace*>(workspace);
  cudaError_t e = cudaMemsetAsync(&ws->ticket, 0, sizeof(ws->ticket), stream);
  if (e != cudaSuccess) return e;
  const size_t n4 = n / 4;
  const int n_tail = static_cast<int>(n - 4 * n4);
  size_t blocks = (n4 + kGammaThreads - 1) / kGammaThreads;
  if (blocks > static_cast<size_t>(kGammaMaxBlocks)) blocks = kGammaMaxBlocks;
  if (blocks < 1) blocks = 1;
  grad_sqnorm_kernel<<<static_cast<unsigned>(blocks), kGammaThreads, 0, stream>>>(
      reinterpret_cast<const float4*>(g), n4, g + 4 * n4, n_tail, ws, sumsq);
  return cudaGetLastError();
}

}  // namespace sbl

// ---------------------------------------------------------------------------
// dW (.) M: the ablation in which masked weights receive no gradient.  One
// thread per 8 weights (two float4 and one mask byte); HBM bound.
namespace {
__global__ void __launch_bounds__(256) mask_grad_kernel(float4* __restrict__ dW, const uint8_t* __restrict__ bits,
                                                        size_t n8) {
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n8;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const uint32_t m = bits[i];
    float4 a = dW[2 * i], b = dW[2 * i + 1];
    a.x = (m & 1u) ? a.x : 0.0f;
    a.y = (m & 2u) ? a.y : 0.0f;
    a.z = (m & 4u) ? a.z : 0.0f;
    a.w = (m & 8u) ? a.w : 0.0f;
    b.x = (m & 16u) ? b.x : 0.0f;
    b.y = (m & 32u) ? b.y : 0.0f;
    b.z = (m & 64u) ? b.z : 0.0f;
    b.w = (m & 128u) ? b.w : 0.0f;
    dW[2 * i] = a;
    dW[2 * i + 1] = b;
  }
}
}  // namespace

namespace sbl {
cudaError_t launch_mask_grad(float* dW, const uint8_t* mask_bits, int d_out, int d_in, cudaStream_t stream,
                             int num_sms) {
  const size_t n8 = static_cast<size_t>(d_out) * d_in / 8;
  if (n8 == 0) return cudaSuccess;
  size_t blocks = (n8 + 255) / 256;
  const size_t cap = static_cast<size_t>(num_sms) * 8;
  if (blocks > cap) blocks = cap;
  mask_grad_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(reinterpret_cast<float4*>(dW), mask_bits, n8);
  return cudaGetLastError();
}
}  // namespace sbl

// ---------------------------------------------------------------------------
// Allocation-free variant of sbl_mask_quant.
//
// Some callers cannot allocate device memory at the point where they run
// the weight step: processes that reserve their whole device-memory budget
// at start-up and forbid any later cudaMalloc, and host frameworks whose
// plugin interface hands over only the input and output buffers, with no
// workspace.  For them the scratch of the gamma pass (exponent buckets, the
// finished-blocks ticket and one partial sum per block) lives in the fixed
// array below, part of the library's own static device memory: every device
// that loads the library holds these bytes until the process exits.
namespace {

static __device__ __align__(256) unsigned char g_mask_quant_scratch[sizeof(sbl::GammaWorkspace)];

constexpr int kNoAllocMaxDevices = 64;
void* g_scratch_ptr[kNoAllocMaxDevices] = {};
int g_scratch_sms[kNoAllocMaxDevices] = {};
std::mutex g_scratch_mu;

// Device address of the scratch array on the current device.  In host code
// the array's name is only a host-side stand-in, so the address is looked up
// once per device with that device current, and cached.
sbl_status scratch_for_current_device(void** ptr, int* num_sms) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SBL_ERR_CUDA;
  if (dev < 0 || dev >= kNoAllocMaxDevices) return SBL_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return SBL_ERR_CUDA;
    if (major != 10 || minor != 0) return SBL_ERR_UNSUPPORTED;
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_mask_quant_scratch) != cudaSuccess || p == nullptr) return SBL_ERR_CUDA;
    g_scratch_sms[dev] = sms;
    g_scratch_ptr[dev] = p;
  }
  *ptr = g_scratch_ptr[dev];
  *num_sms = g_scratch_sms[dev];
  return SBL_OK;
}

}  // namespace

extern "C" size_t sbl_mask_quant_noalloc_scratch_bytes(void) { return sizeof(sbl::GammaWorkspace); }

extern "C" sbl_status sbl_mask_quant_noalloc(const void* W, int d_out, int d_in, int N, int M, int8_t* W_eff,
                                             void* W_eff_bf16, uint8_t* mask_bits, float* gamma, void* stream) {
  if (!(M == 4 || M == 8) || N < 1 || N > M) return SBL_ERR_INVALID_ARG;
  if (W == nullptr || W_eff == nullptr || gamma == nullptr) return SBL_ERR_INVALID_ARG;
  if (d_out <= 0 || d_in <= 0 || d_in % 16 != 0 || d_out % 8 != 0 || d_in % M != 0) return SBL_ERR_SHAPE;
  // The fixed scratch serves any W up to 2^32 - 1 elements; larger W is refused.
  if (static_cast<unsigned long long>(d_out) * static_cast<unsigned long long>(d_in) >= (1ull << 32))
    return SBL_ERR_SHAPE;
  auto misaligned = [](const void* q) { return (reinterpret_cast<uintptr_t>(q) & 15u) != 0; };
  if (misaligned(W) || misaligned(W_eff) || misaligned(W_eff_bf16) || misaligned(mask_bits) ||
      (reinterpret_cast<uintptr_t>(gamma) & 3u) != 0)
    return SBL_ERR_ALIGN;
  void* scratch = nullptr;
  int num_sms = 0;
  const sbl_status st = scratch_for_current_device(&scratch, &num_sms);
  if (st != SBL_OK) return st;
  const cudaError_t e = sbl::launch_mask_quant(W, d_out, d_in, N, M, W_eff, W_eff_bf16, mask_bits, gamma, scratch,
                                               static_cast<cudaStream_t>(stream), num_sms);
  return e == cudaSuccess ? SBL_OK : SBL_ERR_CUDA;
}
