// gemm_tc.cu -- tensor-core products of Sparse-BitLinear on sm_100a (tcgen05).
//
//   (a5) forward, int8 x int8 -> int32 (kind::i8):
//        acc[t,o] = sum_j Xq[t,j] W_eff[o,j];  Y = fp32(acc) * fp32(gamma * fp32(amax_t / 127))
//        Sparse-BitNet summary, Algorithm 1 step (6).
//   (a6) dX = gamma * (dY . W_eff), bf16 x bf16 -> fp32 (kind::f16)
//   (a7) dW = dY^T . X (dense, every position of W), bf16 x bf16 -> fp32
//        Sparse-BitNet summary, STE (前置知识) and 核心方法, Algorithm 1 step (7).
//
// One kernel template, D[M,N] = sum_k A[m,k] B[n,k]:
//   * tile 128 x BN (BN = 256), K step of 128 bytes per stage (128 int8 or 64
//     bf16), STAGES-deep shared-memory ring filled by TMA with 128-byte swizzle;
//   * warp 0: one thread issues the TMA loads; warp 1: allocates tensor memory
//     and one thread issues tcgen05.mma (M = 128, N = BN, accumulator in TMEM),
//     committing each stage back to the producer; warps 2-5: epilogue, each
//     warp reads its 32-lane quarter of the accumulator with tcgen05.ld and
//     applies the scale / accumulate step while storing to global memory;
//   * operands may be K-major (K contiguous) or MN-major (M or N contiguous):
//     forward A = Xq and B = W_eff are K-major; for dX, A = dY is K-major and
//     B = W_eff (N = d_in contiguous) is MN-major; for dW, A = dY^T and B = X
//     are both MN-major (T is the reduction and the row index of both);
//   * ragged edges: TMA fills out-of-range elements with zeros and the
//     epilogue masks its stores; split-K (grid.z) adds partial tiles with
//     fp32 atomics when there are fewer tiles than SMs;
//   * every mbarrier wait is bounded (sbl_device.cuh) and unwinds with a
//     latched error instead of hanging.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "sbl_device.cuh"
#include "sbl_internal.h"

namespace sbl {
namespace {

constexpr int BM = 128;
constexpr int kThreads = 192;

enum Epi : int { kEpiFwd = 0, kEpiDx = 1, kEpiDw = 2 };

struct GemmArgs {
  int M, N, K;
  int kb_per_split;
  float* out;
  long long ldo;
  int32_t* acc_out;
  const float* amax;
  const float* gamma;
  int accumulate;  // dW: add into `out`
  int atomic_out;  // split-K: atomically add into `out`
  uint32_t* err;
};

template <bool kI8, bool kAMN, bool kBMN, int BN, int STAGES>
struct Cfg {
  static constexpr int BK = kI8 ? 128 : 64;  // elements per stage along K (128 bytes)
  static constexpr int UK = kI8 ? 32 : 16;   // K per tcgen05.mma (32 bytes)
  static constexpr int A_BYTES = BM * 128;
  static constexpr int B_BYTES = BN * 128;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 /*align*/ + 256 /*barriers*/;
  static constexpr uint32_t TMEM_COLS = BN;
  static constexpr uint32_t IDESC = instr_desc(kI8, BM, BN, kAMN, kBMN);
};

template <int EPI>
__device__ __forceinline__ void store_chunk(const GemmArgs& a, int row, int col0, const uint32_t (&r)[32],
                                            float scale) {
  float* orow = a.out + static_cast<long long>(row) * a.ldo;
  float v[32];
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    if constexpr (EPI == kEpiFwd) {
      v[j] = __fmul_rn(__int2float_rn(static_cast<int>(r[j])), scale);
    } else if constexpr (EPI == kEpiDx) {
      v[j] = __fmul_rn(scale, __uint_as_float(r[j]));
    } else {
      v[j] = __uint_as_float(r[j]);
    }
  }
  const bool full = col0 + 32 <= a.N;
  if constexpr (EPI == kEpiDw) {
    if (a.atomic_out) {
      if (full) {
#pragma unroll
        for (int j = 0; j < 32; j += 4)
          atomicAdd(reinterpret_cast<float4*>(orow + col0 + j), make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]));
      } else {
        for (int j = 0; j < 32 && col0 + j < a.N; ++j) atomicAdd(orow + col0 + j, v[j]);
      }
      return;
    }
    if (a.accumulate) {
      if (full) {
#pragma unroll
        for (int j = 0; j < 32; j += 4) {
          float4 o = *reinterpret_cast<const float4*>(orow + col0 + j);
          o.x = __fadd_rn(o.x, v[j]);
          o.y = __fadd_rn(o.y, v[j + 1]);
          o.z = __fadd_rn(o.z, v[j + 2]);
          o.w = __fadd_rn(o.w, v[j + 3]);
          *reinterpret_cast<float4*>(orow + col0 + j) = o;
        }
      } else {
        for (int j = 0; j < 32 && col0 + j < a.N; ++j) orow[col0 + j] = __fadd_rn(orow[col0 + j], v[j]);
      }
      return;
    }
  }
  if (full) {
#pragma unroll
    for (int j = 0; j < 32; j += 4)
      *reinterpret_cast<float4*>(orow + col0 + j) = make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]);
  } else {
    for (int j = 0; j < 32 && col0 + j < a.N; ++j) orow[col0 + j] = v[j];
  }
  if constexpr (EPI == kEpiFwd) {
    if (a.acc_out != nullptr) {
      int32_t* arow = a.acc_out + static_cast<long long>(row) * a.ldo;
      if (full) {
#pragma unroll
        for (int j = 0; j < 32; j += 4)
          *reinterpret_cast<int4*>(arow + col0 + j) = make_int4(static_cast<int>(r[j]), static_cast<int>(r[j + 1]),
                                                                static_cast<int>(r[j + 2]), static_cast<int>(r[j + 3]));
      } else {
        for (int j = 0; j < 32 && col0 + j < a.N; ++j) arow[col0 + j] = static_cast<int>(r[j]);
      }
    }
  }
}

template <bool kI8, bool kAMN, bool kBMN, int BN, int STAGES, int EPI>
__global__ void __launch_bounds__(kThreads, 1)
    tc_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const GemmArgs args) {
  using C = Cfg<kI8, kAMN, kBMN, BN, STAGES>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * C::STAGE_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* accum = empty + STAGES;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accum + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int m0 = blockIdx.y * BM;
  const int n0 = blockIdx.x * BN;
  const int KB = (args.K + C::BK - 1) / C::BK;
  const int kb0 = blockIdx.z * args.kb_per_split;
  const int kb1 = min(KB, kb0 + args.kb_per_split);
  const int nk = kb1 - kb0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(accum, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      int issued = 0;
      for (int i = 0; i < nk; ++i) {
        const int s = i % STAGES;
        const uint32_t round = static_cast<uint32_t>(i / STAGES);
        if (!mbar_wait(&empty[s], (round & 1u) ^ 1u, abort_flag, args.err)) break;
        mbar_arrive_expect_tx(&full[s], C::STAGE_BYTES);
        uint8_t* sa = smem + s * C::STAGE_BYTES;
        uint8_t* sb = sa + C::A_BYTES;
        const int kc = (kb0 + i) * C::BK;
        if constexpr (!kAMN) {
          tma_load_2d(sa, &tmA, &full[s], kc, m0);
        } else {
#pragma unroll
          for (int c = 0; c < BM / 64; ++c) tma_load_2d(sa + c * C::BK * 128, &tmA, &full[s], m0 + 64 * c, kc);
        }
        if constexpr (!kBMN) {
          tma_load_2d(sb, &tmB, &full[s], kc, n0);
        } else {
#pragma unroll
          for (int c = 0; c < BN / 64; ++c) tma_load_2d(sb + c * C::BK * 128, &tmB, &full[s], n0 + 64 * c, kc);
        }
        issued = i + 1;
      }
      if (*abort_flag) {
        // Let the copies already in flight land before the block exits.
        for (int i = (issued > STAGES ? issued - STAGES : 0); i < issued; ++i)
          mbar_wait(&full[i % STAGES], static_cast<uint32_t>(i / STAGES) & 1u, nullptr, args.err);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      for (int i = 0; i < nk; ++i) {
        const int s = i % STAGES;
        const uint32_t round = static_cast<uint32_t>(i / STAGES);
        if (!mbar_wait(&full[s], round & 1u, abort_flag, args.err)) break;
        tc_fence_after();
        const uint32_t sa = smem_u32(smem + s * C::STAGE_BYTES);
        const uint32_t sb = sa + C::A_BYTES;
#pragma unroll
        for (int kk = 0; kk < C::BK / C::UK; ++kk) {
          const uint64_t adesc = kAMN ? smem_desc_sw128(sa + kk * C::UK * 128, C::BK * 128, 1024)
                                      : smem_desc_sw128(sa + kk * 32, 16, 1024);
          const uint64_t bdesc = kBMN ? smem_desc_sw128(sb + kk * C::UK * 128, C::BK * 128, 1024)
                                      : smem_desc_sw128(sb + kk * 32, 16, 1024);
          umma<kI8>(tmem_base, adesc, bdesc, C::IDESC, (i > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(&empty[s]);
      }
      umma_commit(accum);
    }
  } else {
    const bool ok = mbar_wait(accum, 0u, abort_flag, args.err);
    tc_fence_after();
    if (ok && !*abort_flag) {
      const int q = warp & 3;
      const int row = m0 + 32 * q + lane;
      float scale = 0.0f;
      if constexpr (EPI == kEpiFwd) {
        if (row < args.M) scale = __fmul_rn(*args.gamma, __fdiv_rn(args.amax[row], 127.0f));
      } else if constexpr (EPI == kEpiDx) {
        scale = *args.gamma;
      }
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        const int col0 = n0 + 32 * c;
        if (col0 >= args.N) break;  // warp-uniform
        uint32_t r[32];
        tmem_ld_32x32b_x32(tmem_base + (static_cast<uint32_t>(32 * q) << 16) + static_cast<uint32_t>(32 * c), r);
        tmem_ld_wait();
        if (row < args.M) store_chunk<EPI>(args, row, col0, r, scale);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

// ------------------------------------------------------------------ host side
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encoder() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// Row-major [outer, inner] matrix, box [box_outer, box_inner], 128-byte swizzle.
bool make_tmap(CUtensorMap* m, const void* base, bool bf16, uint64_t inner, uint64_t outer, uint64_t row_bytes,
               uint32_t box_inner, uint32_t box_outer) {
  EncodeTiledFn enc = encoder();
  if (enc == nullptr) return false;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = enc(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8, 2,
                         const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <bool kI8, bool kAMN, bool kBMN, int BN, int STAGES, int EPI>
cudaError_t run(const CUtensorMap& ta, const CUtensorMap& tb, const GemmArgs& a, int splits,
                cudaStream_t stream) {
  using C = Cfg<kI8, kAMN, kBMN, BN, STAGES>;
  auto kern = tc_gemm_kernel<kI8, kAMN, kBMN, BN, STAGES, EPI>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  const dim3 grid((a.N + BN - 1) / BN, (a.M + BM - 1) / BM, splits);
  kern<<<grid, kThreads, C::SMEM_BYTES, stream>>>(ta, tb, a);
  return cudaGetLastError();
}

constexpr int kBN = 256;
constexpr int kStages = 4;

}  // namespace

cudaError_t launch_forward(const int8_t* Xq, const float* amax, const int8_t* W_eff, const float* gamma, int T,
                           int d_in, int d_out, float* Y, int32_t* acc, cudaStream_t stream, int num_sms,
                           uint32_t* err) {
  (void)num_sms;
  if (T == 0 || d_out == 0) return cudaSuccess;
  if (d_in == 0) {
    cudaError_t e = cudaMemsetAsync(Y, 0, sizeof(float) * static_cast<size_t>(T) * d_out, stream);
    if (e == cudaSuccess && acc != nullptr)
      e = cudaMemsetAsync(acc, 0, sizeof(int32_t) * static_cast<size_t>(T) * d_out, stream);
    return e;
  }
  CUtensorMap ta, tb;
  if (!make_tmap(&ta, Xq, false, d_in, T, d_in, 128, BM)) return cudaErrorInvalidValue;
  if (!make_tmap(&tb, W_eff, false, d_in, d_out, d_in, 128, kBN)) return cudaErrorInvalidValue;
  GemmArgs a{};
  a.M = T;
  a.N = d_out;
  a.K = d_in;
  a.kb_per_split = (d_in + 127) / 128;
  a.out = Y;
  a.ldo = d_out;
  a.acc_out = acc;
  a.amax = amax;
  a.gamma = gamma;
  a.err = err;
  return run<true, false, false, kBN, kStages, kEpiFwd>(ta, tb, a, 1, stream);
}

cudaError_t launch_backward(const void* dY, const void* X, const void* W_eff_bf16, const float* gamma, int T,
                            int d_in, int d_out, float* dX, float* dW, int accumulate_dW, cudaStream_t stream,
                            int num_sms, uint32_t* err) {
  cudaError_t e = cudaSuccess;
  if (dX != nullptr && T > 0 && d_in > 0) {
    if (d_out == 0) {
      e = cudaMemsetAsync(dX, 0, sizeof(float) * static_cast<size_t>(T) * d_in, stream);
    } else {
      CUtensorMap ta, tb;
      // A = dY [T, d_out], K-major (K = d_out); B = W_eff [d_out, d_in], N-major.
      if (!make_tmap(&ta, dY, true, d_out, T, 2ull * d_out, 64, BM)) return cudaErrorInvalidValue;
      if (!make_tmap(&tb, W_eff_bf16, true, d_in, d_out, 2ull * d_in, 64, 64)) return cudaErrorInvalidValue;
      GemmArgs a{};
      a.M = T;
      a.N = d_in;
      a.K = d_out;
      a.kb_per_split = (d_out + 63) / 64;
      a.out = dX;
      a.ldo = d_in;
      a.gamma = gamma;
      a.err = err;
      e = run<false, false, true, kBN, kStages, kEpiDx>(ta, tb, a, 1, stream);
    }
    if (e != cudaSuccess) return e;
  }
  if (dW != nullptr && d_out > 0 && d_in > 0) {
    if (T == 0) {
      if (!accumulate_dW) e = cudaMemsetAsync(dW, 0, sizeof(float) * static_cast<size_t>(d_out) * d_in, stream);
      return e;
    }
    CUtensorMap ta, tb;
    // A = dY^T: element (m = o, k = t) at dY[t, o] -> M-major; B = X^T: (n = j, k = t) at X[t, j] -> N-major.
    if (!make_tmap(&ta, dY, true, d_out, T, 2ull * d_out, 64, 64)) return cudaErrorInvalidValue;
    if (!make_tmap(&tb, X, true, d_in, T, 2ull * d_in, 64, 64)) return cudaErrorInvalidValue;
    const int KB = (T + 63) / 64;
    const int tiles = ((d_in + kBN - 1) / kBN) * ((d_out + BM - 1) / BM);
    int splits = num_sms / tiles;
    if (splits < 1) splits = 1;
    if (splits > KB) splits = KB;
    const int kbps = (KB + splits - 1) / splits;
    splits = (KB + kbps - 1) / kbps;
    GemmArgs a{};
    a.M = d_out;
    a.N = d_in;
    a.K = T;
    a.kb_per_split = kbps;
    a.out = dW;
    a.ldo = d_in;
    a.accumulate = accumulate_dW;
    a.atomic_out = splits > 1;
    a.err = err;
    if (splits > 1 && !accumulate_dW) {
      e = cudaMemsetAsync(dW, 0, sizeof(float) * static_cast<size_t>(d_out) * d_in, stream);
      if (e != cudaSuccess) return e;
    }
    e = run<false, true, true, kBN, kStages, kEpiDw>(ta, tb, a, splits, stream);
  }
  return e;
}

}  // namespace sbl
