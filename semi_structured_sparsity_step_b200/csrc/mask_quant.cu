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
#include <cuda_runtime.h>
#include <cstdint>

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
__device__ uint32_t zero_threshold_bits(float den) {
  uint32_t lo = 0u, hi = 0x7F80u;  // cond(lo) holds; cond(hi) fails (inf)
  while (hi - lo > 1u) {
    const uint32_t mid = (lo + hi) >> 1;
    const float v = __uint_as_float(mid << 16);
    if (__fdiv_rn(v, den) <= 0.5f) lo = mid; else hi = mid;
  }
  return lo;
}

__global__ void __launch_bounds__(kGammaThreads) gamma_reduce_kernel(const uint4* __restrict__ W, size_t n_vec,
                                                                      size_t n_elems, GammaWorkspace* ws,
                                                                      float* __restrict__ gamma_out) {
  __shared__ unsigned long long sbucket[256];
  __shared__ uint64_t swarp[kGammaThreads / 32];
  __shared__ int s_last;
  sbucket[threadIdx.x] = 0ull;
  __syncthreads();

  uint64_t acc = 0;
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n_vec;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const uint4 v = __ldg(W + i);
    const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      gamma_add_bf16(w4[k] & 0xFFFFu, acc, sbucket);
      gamma_add_bf16(w4[k] >> 16, acc, sbucket);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xFFFFFFFFu, acc, o);
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

  // Last block: 128-bit sum of the per-block window sums.
  __shared__ uint64_t s_lo[kGammaThreads], s_hi[kGammaThreads];
  uint64_t lo = 0, hi = 0;
  for (unsigned b = threadIdx.x; b < gridDim.x; b += blockDim.x) {
    const uint64_t p = __ldcg(&ws->block_window[b]);
    lo += p;
    hi += (lo < p) ? 1u : 0u;
  }
  s_lo[threadIdx.x] = lo;
  s_hi[threadIdx.x] = hi;
  sbucket[threadIdx.x] = __ldcg(&ws->bucket[threadIdx.x]);
  __syncthreads();
  if (threadIdx.x != 0) return;
  lo = 0;
  hi = 0;
  for (int t = 0; t < kGammaThreads; ++t) {
    lo += s_lo[t];
    hi += s_hi[t] + ((lo < s_lo[t]) ? 1u : 0u);
  }
  uint32_t limbs[kGammaLimbs];
#pragma unroll
  for (int i = 0; i < kGammaLimbs; ++i) limbs[i] = 0u;
  // value = m * 2^(ee-134) = m * 2^(ee-1) units of 2^-133; window sums carry 2^(96-1).
  bigint_add_shifted(limbs, lo, kWinLo - 1);
  bigint_add_shifted(limbs, hi, kWinLo - 1 + 64);
  for (int ee = 1; ee < 256; ++ee) bigint_add_shifted(limbs, sbucket[ee], ee - 1);
  const double total = bigint_to_double(limbs);
  const double mean = __ddiv_rn(total, static_cast<double>(n_elems));
  const float gamma = __double2float_rn(mean);
  *gamma_out = gamma;
  ws->zero_threshold = zero_threshold_bits(__fadd_rn(gamma, 1e-5f));
}


template <int M>
__device__ __forceinline__ void rank_keep(const uint32_t (&mag)[8], int N, uint32_t& keep_bits) {
  // key = magnitude, then lower position first; all keys in a group differ.
  keep_bits = 0u;
#pragma unroll
  for (int g = 0; g < 8 / M; ++g) {
    uint32_t key[M];
    int rank[M];
#pragma unroll
    for (int j = 0; j < M; ++j) {
      key[j] = (mag[g * M + j] << 3) | static_cast<uint32_t>(M - 1 - j);
      rank[j] = 0;
    }
#pragma unroll
    for (int i = 0; i < M; ++i) {
#pragma unroll
      for (int j = i + 1; j < M; ++j) {
        const int gt = key[i] > key[j];
        rank[j] += gt;
        rank[i] += 1 - gt;
      }
    }
#pragma unroll
    for (int j = 0; j < M; ++j) keep_bits |= (rank[j] < N ? 1u : 0u) << (g * M + j);
  }
}

template <int M>
__global__ void __launch_bounds__(256) ternary_mask_kernel(const uint4* __restrict__ W, size_t n_vec, int N,
                                                           const GammaWorkspace* __restrict__ ws,
                                                           uint2* __restrict__ w_eff,
                                                           uint4* __restrict__ w_eff_bf16,
                                                           uint8_t* __restrict__ mask_bits) {
  const uint32_t thr = ws->zero_threshold;
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n_vec;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const uint4 v = __ldg(W + i);
    const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
    uint32_t h[8], mag[8];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      h[2 * k] = w4[k] & 0xFFFFu;
      h[2 * k + 1] = w4[k] >> 16;
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) mag[k] = h[k] & 0x7FFFu;
    uint32_t keep;
    rank_keep<M>(mag, N, keep);
    uint32_t q8[2] = {0u, 0u};
    uint32_t qb[4] = {0u, 0u, 0u, 0u};
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const bool nz = ((keep >> k) & 1u) && (mag[k] > thr);
      const bool neg = (h[k] >> 15) != 0u;
      const uint32_t byte = nz ? (neg ? 0xFFu : 0x01u) : 0u;
      const uint32_t bf = nz ? (neg ? 0xBF80u : 0x3F80u) : 0u;
      q8[k >> 2] |= byte << (8 * (k & 3));
      qb[k >> 1] |= bf << (16 * (k & 1));
    }
    w_eff[i] = make_uint2(q8[0], q8[1]);
    if (w_eff_bf16 != nullptr) w_eff_bf16[i] = make_uint4(qb[0], qb[1], qb[2], qb[3]);
    if (mask_bits != nullptr) mask_bits[i] = static_cast<uint8_t>(keep);
  }
}

}  // namespace

size_t mask_quant_workspace_bytes() { return sizeof(GammaWorkspace); }

cudaError_t launch_mask_quant(const void* W, int d_out, int d_in, int N, int M, int8_t* W_eff, void* W_eff_bf16,
                              uint8_t* mask_bits, float* gamma, void* workspace, cudaStream_t stream,
                              int num_sms) {
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
  size_t qblocks = (n_vec + 255) / 256;
  const size_t qmax = static_cast<size_t>(num_sms) * 16;
  if (qblocks > qmax) qblocks = qmax;
  if (qblocks < 1) qblocks = 1;
  if (M == 8) {
    ternary_mask_kernel<8><<<static_cast<unsigned>(qblocks), 256, 0, stream>>>(
        static_cast<const uint4*>(W), n_vec, N, ws, reinterpret_cast<uint2*>(W_eff),
        static_cast<uint4*>(W_eff_bf16), mask_bits);
  } else {
    ternary_mask_kernel<4><<<static_cast<unsigned>(qblocks), 256, 0, stream>>>(
        static_cast<const uint4*>(W), n_vec, N, ws, reinterpret_cast<uint2*>(W_eff),
        static_cast<uint4*>(W_eff_bf16), mask_bits);
  }
  return cudaGetLastError();
}

}  // namespace sbl
