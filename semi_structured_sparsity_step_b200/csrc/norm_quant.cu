// norm_quant.cu -- RMSNorm fused with the per-token absmax int8 activation
// quantiser: x~ = Q_a(Norm(x)) in one pass over X on sm_100a.
//
// Sparse-BitNet summary ("Sparse-BitNet：1.58-bit 大模型天然兼容半结构化稀疏"),
// Algorithm 1 step (3): the activation is normalised, then quantised to int8.
// Norm is read as RMSNorm with a per-channel gain g, with an arithmetic that
// does not depend on a summation order:
//   ss = sum_j x_j^2 in fp64 (each bf16 square is exact in fp64; the sum is
//   exact unless the squares span more than 2^37, and even then an order
//   of summation shows in v only when ss lies within a few fp64 ulps of an
//   fp32 rounding boundary),
//   v = fl32(ss / d + eps),  r = fl32(1 / fl32(sqrt(v))),
//   xn_j = bf16_rn(fl32(fl32(x_j * r) * g_j)),
// then Q_a of the bf16 row xn exactly as act_quant.cu (amax = max(max|xn|,
// 1e-5), one FADD of 1.5 * 2^23 rounds fl32(xn * fl32(127 / amax))).
//
// HBM bound: X is read once (2 B per element), Xq written once (1 B) and,
// when requested, the normalised row xn (2 B, the bf16 input of the dW
// product).  Compared with a separate norm kernel feeding act_quant this
// saves one read and one write of X.  Each row lives in registers (8, or 6
// for rows of 256 threads that fit, x 16 bytes per thread, TPR threads per
// row); longer rows re-read their tail from L2.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "sbl_device.cuh"
#include "sbl_internal.h"

namespace sbl {
namespace {

constexpr int kNqThreads = 256;
constexpr int kNqVpt = 8;
constexpr float kNqRoundMagic = 12582912.0f;  // 1.5 * 2^23

__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// fp64 value of |x| for the bf16 x in the low (t = w & 0x7FFF) or high half
// of a word, built with integer arithmetic instead of a conversion: the bf16
// exponent and mantissa bits move into the fp64 high word (shift by 13) and
// the exponent bias grows by 1023 - 127 = 896.  Exact for normal numbers; a
// zero or subnormal becomes a value below 2^-126, whose square (< 2^-252)
// cannot change fl32(ss / d + eps) for eps > 0.
__device__ __forceinline__ double absf64_lo(uint32_t w) {
  return __hiloint2double(static_cast<int>((w & 0x7FFFu) * 8192u + (896u << 20)), 0);
}
__device__ __forceinline__ double absf64_hi(uint32_t w) {
  return __hiloint2double(static_cast<int>(__umulhi(w & 0x7FFF0000u, 1u << 29) + (896u << 20)), 0);
}

// running fp64 sum of the squares of 8 bf16 values (each square is exact in
// fp64, so one fma per element adds it with a single rounding)
__device__ __forceinline__ double sumsq8(const uint4& v, double s) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const double a = absf64_lo(w[k]), b = absf64_hi(w[k]);
    s = fma(a, a, s);
    s = fma(b, b, s);
  }
  return s;
}

// bf16 round-to-nearest-even of fl32(fl32(x * r) * g) for the 8 values of v
// with gains gv; returns the 8 results packed like v
__device__ __forceinline__ uint4 norm8(const uint4& v, const uint4& gv, float r) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  const uint32_t gw[4] = {gv.x, gv.y, gv.z, gv.w};
  uint32_t o[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const float lo = __fmul_rn(__fmul_rn(bf_lo(w[k]), r), bf_lo(gw[k]));
    const float hi = __fmul_rn(__fmul_rn(bf_hi(w[k]), r), bf_hi(gw[k]));
    // one packed conversion (round to nearest even) for the pair
    const __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
    o[k] = *reinterpret_cast<const uint32_t*>(&p);
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

__device__ __forceinline__ uint32_t maxmag8(const uint4& v) {
  const uint32_t a = __vmaxu2(v.x & 0x7FFF7FFFu, v.y & 0x7FFF7FFFu);
  const uint32_t b = __vmaxu2(v.z & 0x7FFF7FFFu, v.w & 0x7FFF7FFFu);
  return __vmaxu2(a, b);
}

__device__ __forceinline__ uint32_t q1(float x, float s) {
  return __float_as_uint(__fadd_rn(__fmul_rn(x, s), kNqRoundMagic));
}

__device__ __forceinline__ uint2 quant8(const uint4& v, float s) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t o[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const uint32_t a = q1(bf_lo(w[2 * h]), s), b = q1(bf_hi(w[2 * h]), s);
    const uint32_t c = q1(bf_lo(w[2 * h + 1]), s), d = q1(bf_hi(w[2 * h + 1]), s);
    o[h] = __byte_perm(__byte_perm(a, b, 0x0040u), __byte_perm(c, d, 0x0040u), 0x5410u);
  }
  return make_uint2(o[0], o[1]);
}

// Sum (or max) of a value over the TPR threads of a row.  All threads of the
// block call it.  With WPR > 1 the warps meet at one barrier through the
// shared scratch; the sum and the max use different scratch arrays, and the
// barrier of one reduction is what keeps a fast warp from overwriting the
// other's scratch before every warp has read it, so no second barrier is
// needed.
template <int TPR, typename V>
__device__ __forceinline__ V row_reduce(V x, V* scratch, int rib, bool is_max) {
  constexpr int WPR = TPR / 32;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const V y = __shfl_xor_sync(0xFFFFFFFFu, x, o);
    x = is_max ? (x > y ? x : y) : x + y;
  }
  if constexpr (WPR > 1) {
    const int warp = threadIdx.x >> 5;
    if ((threadIdx.x & 31) == 0) scratch[warp] = x;
    __syncthreads();
    x = scratch[rib * WPR];
#pragma unroll
    for (int w = 1; w < WPR; ++w) {
      const V y = scratch[rib * WPR + w];
      x = is_max ? (x > y ? x : y) : x + y;
    }
  }
  return x;
}

template <int TPR, int VPT>
__global__ void __launch_bounds__(kNqThreads) norm_quant_kernel(const uint4* __restrict__ X,
                                                                const uint4* __restrict__ G, float eps, int T,
                                                                int nv, uint4* __restrict__ Xn,
                                                                uint2* __restrict__ Xq, float* __restrict__ amax) {
  constexpr int RPB = kNqThreads / TPR;  // rows per block
  __shared__ double s_sum[kNqThreads / 32];
  __shared__ uint32_t s_max[kNqThreads / 32];
  const int rib = threadIdx.x / TPR;
  const int tr = threadIdx.x % TPR;
  const int d = nv * 8;

  // Every vector's arithmetic runs unconditionally (a vector past the end of
  // the row is loaded as zeros: its squares are below 2^-252 and cannot move
  // fl32(ss / d + eps), and it normalises and quantises to zeros); only the
  // loads and stores are predicated, so the loops carry no divergent branches.
  // Rows past T re-read row T - 1 and store nothing.
  for (long long base = static_cast<long long>(blockIdx.x) * RPB; base < T;
       base += static_cast<long long>(gridDim.x) * RPB) {
    const long long row = base + rib;
    const bool active = row < T;
    const uint4* xr = X + (active ? row : static_cast<long long>(T) - 1) * static_cast<long long>(nv);
    uint4 v[VPT];
    double ss = 0.0;
#pragma unroll
    for (int k = 0; k < VPT; ++k) {
      const int idx = tr + k * TPR;
      v[k] = idx < nv ? __ldg(xr + idx) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int k = 0; k < VPT; ++k) ss = sumsq8(v[k], ss);
    for (int idx = tr + VPT * TPR; idx < nv; idx += TPR) ss = sumsq8(__ldg(xr + idx), ss);
    ss = row_reduce<TPR, double>(ss, s_sum, rib, false);
    const float vv = static_cast<float>(ss / static_cast<double>(d) + static_cast<double>(eps));
    const float r = __fdiv_rn(1.0f, __fsqrt_rn(vv));

    uint32_t mx = 0u;
#pragma unroll
    for (int k = 0; k < VPT; ++k) {
      const int idx = tr + k * TPR;
      const uint4 gk = idx < nv ? __ldg(G + idx) : make_uint4(0u, 0u, 0u, 0u);
      v[k] = norm8(v[k], gk, r);
      mx = __vmaxu2(mx, maxmag8(v[k]));
    }
    for (int idx = tr + VPT * TPR; idx < nv; idx += TPR)
      mx = __vmaxu2(mx, maxmag8(norm8(__ldg(xr + idx), __ldg(G + idx), r)));
    mx = max(mx & 0xFFFFu, mx >> 16);
    mx = row_reduce<TPR, uint32_t>(mx, s_max, rib, true);
    const float a = fmaxf(__uint_as_float(mx << 16), 1e-5f);
    const float sc = __fdiv_rn(127.0f, a);
    uint2* qr = Xq + row * static_cast<long long>(nv);
    uint4* nr = Xn != nullptr ? Xn + row * static_cast<long long>(nv) : nullptr;
#pragma unroll
    for (int k = 0; k < VPT; ++k) {
      const int idx = tr + k * TPR;
      const uint2 q = quant8(v[k], sc);
      if (active && idx < nv) {
        qr[idx] = q;
        if (nr != nullptr) nr[idx] = v[k];
      }
    }
    if (active) {
      for (int idx = tr + VPT * TPR; idx < nv; idx += TPR) {
        const uint4 u = norm8(__ldg(xr + idx), __ldg(G + idx), r);
        qr[idx] = quant8(u, sc);
        if (nr != nullptr) nr[idx] = u;
      }
      if (tr == 0) amax[row] = a;
    }
  }
}

template <int TPR, int VPT>
cudaError_t launch_nq_v(const void* X, const void* g, float eps, int T, int nv, void* Xn, int8_t* Xq, float* amax,
                        cudaStream_t stream, int num_sms) {
  constexpr int RPB = kNqThreads / TPR;
  long long blocks = (static_cast<long long>(T) + RPB - 1) / RPB;
  const long long cap = static_cast<long long>(num_sms) * 8;
  if (blocks > cap) blocks = cap;
  norm_quant_kernel<TPR, VPT><<<static_cast<unsigned>(blocks), kNqThreads, 0, stream>>>(
      static_cast<const uint4*>(X), static_cast<const uint4*>(g), eps, T, nv, static_cast<uint4*>(Xn),
      reinterpret_cast<uint2*>(Xq), amax);
  return cudaGetLastError();
}

// Vectors held in registers per thread.  A row of 256 threads that fits in
// 6 (such as 1376 vectors, d = 11008) holds 6 instead of 8, so it runs no
// arithmetic on two zero-filled vectors past its end; narrower rows keep 8.
template <int TPR>
cudaError_t launch_nq(const void* X, const void* g, float eps, int T, int nv, void* Xn, int8_t* Xq, float* amax,
                      cudaStream_t stream, int num_sms) {
  if constexpr (TPR == 256) {
    if (nv <= 6 * TPR) return launch_nq_v<TPR, 6>(X, g, eps, T, nv, Xn, Xq, amax, stream, num_sms);
  }
  return launch_nq_v<TPR, kNqVpt>(X, g, eps, T, nv, Xn, Xq, amax, stream, num_sms);
}

}  // namespace

cudaError_t launch_norm_act_quant(const void* X, const void* g, float eps, int T, int d_in, void* Xn, int8_t* Xq,
                                  float* amax, cudaStream_t stream, int num_sms) {
  if (T == 0) return cudaSuccess;
  const int nv = d_in / 8;
  if (nv <= 32 * kNqVpt) return launch_nq<32>(X, g, eps, T, nv, Xn, Xq, amax, stream, num_sms);
  if (nv <= 64 * kNqVpt) return launch_nq<64>(X, g, eps, T, nv, Xn, Xq, amax, stream, num_sms);
  if (nv <= 128 * kNqVpt) return launch_nq<128>(X, g, eps, T, nv, Xn, Xq, amax, stream, num_sms);
  return launch_nq<256>(X, g, eps, T, nv, Xn, Xq, amax, stream, num_sms);
}

}  // namespace sbl
