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
#include <algorithm>
#include <atomic>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "packed_decode.cuh"
#include "sbl_device.cuh"
#include "sbl_internal.h"

namespace sbl {
namespace {

constexpr int BM = 128;
constexpr int kThreads = 192;

enum Epi : int { kEpiFwd = 0, kEpiDx = 1, kEpiDw = 2 };

// Programmatic dependent launch: a product may start while the previous
// kernel of its stream finishes.  The prologue (barriers, tensor memory,
// descriptor prefetch, the packed-B selector table) touches only kernel
// parameters and on-chip state; every thread waits for the previous kernel
// before any global load, TMA copy or store.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;"); }

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
  int atomic_i32;  // forward split-K: add the int32 partial sums, as exact fp32 integers, into `out`
  uint32_t* err;
};

template <bool kI8, bool kAMN, bool kBMN, int BN, int STAGES>
struct Cfg {
  static constexpr int BK = kI8 ? 128 : 64;  // elements per stage along K (128 bytes)
  static constexpr int UK = kI8 ? 32 : 16;   // K per tcgen05.mma (32 bytes)
  static constexpr int A_BYTES = BM * 128;
  static constexpr int B_BYTES = BN * 128;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int EPI_WARP_FLOATS = 32 * 33;  // 32 x 32 fp32 transpose tile, padded rows
  static constexpr int EPI_BYTES = 4 * EPI_WARP_FLOATS * 4;
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + EPI_BYTES + 1024 /*align*/ + 256 /*barriers*/;
  static constexpr uint32_t TMEM_COLS = 2 * BN;  // two accumulator buffers
  static constexpr uint32_t IDESC = instr_desc(kI8, BM, BN, kAMN, kBMN);
};

// Work item -> (m block, n block, k split).  Items are ordered in strips of
// GM consecutive m blocks: inside a strip m varies fastest, then n; k splits
// are outermost.  GM = 1 is plain n-fastest order (the concurrent tiles share
// the B tiles and each A row block is read once); GM = Mt makes all m blocks
// of an n block run together so a streamed B operand is read once.  The
// host picks GM from the operands' sizes.
struct Sched {
  int Mt, Nt, splits, total, GM;
  __device__ __forceinline__ void item(int w, int& mb, int& nb, int& sp) const {
    const int per = Mt * Nt;
    sp = w / per;
    int r = w - sp * per;
    const int strip_items = GM * Nt;
    const int strip = r / strip_items;
    r -= strip * strip_items;
    const int gm = min(GM, Mt - strip * GM);  // the last strip may be narrower
    nb = r / gm;
    mb = strip * GM + (r - nb * gm);
  }
};

// Epilogue of one 32 x 32 chunk held one row per lane (r[j] = column j).
// Phase 1 applies the scale in that layout and writes the chunk into a padded
// shared tile; phase 2 reads it back four rows per instruction, so every
// global access of the warp covers four whole 128-byte row segments.
template <int EPI>
__device__ __forceinline__ void epilogue_chunk(const GemmArgs& a, float* tile, int row0, int col0, int lane,
                                               const uint32_t (&r)[32], float scale) {
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    float v;
    if constexpr (EPI == kEpiFwd) {
      v = a.atomic_i32 ? __int2float_rn(static_cast<int>(r[j]))
                       : __fmul_rn(__int2float_rn(static_cast<int>(r[j])), scale);
    } else if constexpr (EPI == kEpiDx) {
      v = __fmul_rn(scale, __uint_as_float(r[j]));
    } else {
      v = __uint_as_float(r[j]);
    }
    tile[lane * 33 + j] = v;
  }
  if constexpr (EPI == kEpiFwd) {
    if (!a.atomic_i32 && a.acc_out != nullptr && row0 + lane < a.M) {
      int32_t* arow = a.acc_out + static_cast<long long>(row0 + lane) * a.ldo + col0;
#pragma unroll
      for (int j = 0; j < 32; j += 4)
        if (col0 + j < a.N)
          *reinterpret_cast<int4*>(arow + j) = make_int4(static_cast<int>(r[j]), static_cast<int>(r[j + 1]),
                                                         static_cast<int>(r[j + 2]), static_cast<int>(r[j + 3]));
    }
  }
  __syncwarp();
  const int cq = (lane & 7) * 4;
#pragma unroll
  for (int it = 0; it < 8; ++it) {
    const int rr = it * 4 + (lane >> 3);
    const int grow = row0 + rr;
    const int gcol = col0 + cq;
    if (grow < a.M && gcol < a.N) {  // N % 8 == 0: a float4 is either all in or all out
      const float* t = tile + rr * 33 + cq;
      float4 v = make_float4(t[0], t[1], t[2], t[3]);
      float* dst = a.out + static_cast<long long>(grow) * a.ldo + gcol;
      if constexpr (EPI == kEpiFwd) {
        if (a.atomic_i32) {
          // one k split's int32 sums as fp32: every partial and total is an
          // integer below 2^24 in magnitude, so each fp32 addition is exact
          // and the order of the atomics does not matter
          atomicAdd(reinterpret_cast<float4*>(dst), v);
          continue;
        }
      }
      if constexpr (EPI == kEpiDw) {
        if (a.atomic_out) {
          atomicAdd(reinterpret_cast<float4*>(dst), v);
          continue;
        }
        if (a.accumulate) {
          const float4 o = *reinterpret_cast<const float4*>(dst);
          v.x = __fadd_rn(o.x, v.x);
          v.y = __fadd_rn(o.y, v.y);
          v.z = __fadd_rn(o.z, v.z);
          v.w = __fadd_rn(o.w, v.w);
        }
      }
      *reinterpret_cast<float4*>(dst) = v;
    }
  }
  __syncwarp();
}

// Persistent kernel: one CTA per SM walks the work items blockIdx.x,
// blockIdx.x + gridDim.x, ...  The shared-memory ring and its phases run on
// across items; the accumulator alternates between two TMEM buffers so the
// epilogue of one item overlaps the tensor-core work of the next.
template <bool kI8, bool kAMN, bool kBMN, int BN, int STAGES, int EPI>
__global__ void __launch_bounds__(kThreads, 1)
    tc_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const GemmArgs args, const Sched sched) {
  using C = Cfg<kI8, kAMN, kBMN, BN, STAGES>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* epi_tiles = reinterpret_cast<float*>(smem + STAGES * C::STAGE_BYTES);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * C::STAGE_BYTES + C::EPI_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;  // [2] accumulator buffer ready for the epilogue
  uint64_t* tempty = tfull + 2;      // [2] accumulator buffer drained by the epilogue
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tempty + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int KB = (args.K + C::BK - 1) / C::BK;

  if (threadIdx.x == 0) pdl_launch_dependents();
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 4);
    }
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
  pdl_wait();

  if (warp == 0) {
    if (lane == 0) {
      int it = 0;  // k-blocks issued by this CTA so far (position in the stage ring)
      bool ok = true;
      for (int w = blockIdx.x; w < sched.total && ok; w += gridDim.x) {
        int mb, nb, sp;
        sched.item(w, mb, nb, sp);
        const int kb0 = sp * args.kb_per_split;
        const int kb1 = min(KB, kb0 + args.kb_per_split);
        const int m0 = mb * BM, n0 = nb * BN;
        for (int kb = kb0; kb < kb1; ++kb) {
          const int s = it % STAGES;
          const uint32_t round = static_cast<uint32_t>(it / STAGES);
          if (!mbar_wait(&empty[s], (round & 1u) ^ 1u, abort_flag, args.err)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[s], C::STAGE_BYTES);
          uint8_t* sa = smem + s * C::STAGE_BYTES;
          uint8_t* sb = sa + C::A_BYTES;
          const int kc = kb * C::BK;
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
          ++it;
        }
      }
      if (!ok) {
        // Let the copies already in flight land before the block exits.
        for (int i = (it > STAGES ? it - STAGES : 0); i < it; ++i)
          mbar_wait(&full[i % STAGES], static_cast<uint32_t>(i / STAGES) & 1u, nullptr, args.err);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      int it = 0, t = 0;
      bool ok = true;
      for (int w = blockIdx.x; w < sched.total && ok; w += gridDim.x, ++t) {
        int mb, nb, sp;
        sched.item(w, mb, nb, sp);
        const int kb0 = sp * args.kb_per_split;
        const int kb1 = min(KB, kb0 + args.kb_per_split);
        const int b = t & 1;
        if (!mbar_wait(&tempty[b], (static_cast<uint32_t>(t >> 1) & 1u) ^ 1u, abort_flag, args.err)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(b * BN);
        for (int kb = kb0; kb < kb1; ++kb) {
          const int s = it % STAGES;
          const uint32_t round = static_cast<uint32_t>(it / STAGES);
          if (!mbar_wait(&full[s], round & 1u, abort_flag, args.err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + s * C::STAGE_BYTES);
          const uint32_t sb = sa + C::A_BYTES;
#pragma unroll
          for (int kk = 0; kk < C::BK / C::UK; ++kk) {
            const uint64_t adesc = kAMN ? smem_desc_sw128(sa + kk * C::UK * 128, C::BK * 128, 1024)
                                        : smem_desc_sw128(sa + kk * 32, 16, 1024);
            const uint64_t bdesc = kBMN ? smem_desc_sw128(sb + kk * C::UK * 128, C::BK * 128, 1024)
                                        : smem_desc_sw128(sb + kk * 32, 16, 1024);
            umma<kI8>(d_tmem, adesc, bdesc, C::IDESC, (kb > kb0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(&empty[s]);
          ++it;
        }
        umma_commit(&tfull[b]);  // fires when this item's MMAs are done (also on abort)
      }
    }
  } else {
    const int q = warp & 3;  // TMEM lane quarter this warp may read
    float* tile = epi_tiles + q * C::EPI_WARP_FLOATS;
    int t = 0;
    for (int w = blockIdx.x; w < sched.total; w += gridDim.x, ++t) {
      int mb, nb, sp;
      sched.item(w, mb, nb, sp);
      const int b = t & 1;
      if (!mbar_wait(&tfull[b], static_cast<uint32_t>(t >> 1) & 1u, abort_flag, args.err)) break;
      tc_fence_after();
      if (*abort_flag) break;
      const int row0 = mb * BM + 32 * q;
      const int row = row0 + lane;
      float scale = 0.0f;
      if constexpr (EPI == kEpiFwd) {
        if (row < args.M) scale = __fmul_rn(*args.gamma, __fdiv_rn(args.amax[row], 127.0f));
      } else if constexpr (EPI == kEpiDx) {
        scale = *args.gamma;
      }
      const uint32_t tbase = tmem_base + (static_cast<uint32_t>(32 * q) << 16) + static_cast<uint32_t>(b * BN);
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        const int col0 = nb * BN + 32 * c;
        if (col0 >= args.N) break;  // warp-uniform
        uint32_t r[32];
        tmem_ld_32x32b_x32(tbase + static_cast<uint32_t>(32 * c), r);
        tmem_ld_wait();
        epilogue_chunk<EPI>(args, tile, row0, col0, lane, r, scale);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[b]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

// ------------------------------------------------------------ CTA-pair kernel
// Same product with a cluster of two CTAs per 256 x 256 tile (tcgen05
// cta_group::2): CTA r of the pair stages rows [128 r, 128 r + 128) of the A
// tile and rows [128 r, 128 r + 128) of the B tile (N half); the even CTA
// issues tcgen05.mma with M = 256, which reads both CTAs' shared memory and
// writes 128 accumulator rows into each CTA's TMEM.  Per SM this halves the
// B bytes staged and read per MMA compared with a 128 x 256 tile on one SM.
//   full[s]   (even CTA only): the even producer arms it with both CTAs' bytes;
//             both producers' TMA loads complete on it.
//   empty[s]  (both CTAs): freed by one multicast tcgen05.commit.
//   tfull[b]  (both CTAs): accumulator buffer b ready (multicast commit).
//   tempty[b] (even CTA only): 4 epilogue warps of each CTA arrive.
template <bool kI8, bool kAMN, bool kBMN, int STAGES, int KP = 0>
struct Cfg2 {
  static constexpr int BN = 256;                 // N of the pair's tile
  static constexpr int BK = kI8 ? 128 : 64;      // elements per stage along K (128 bytes)
  static constexpr int UK = kI8 ? 32 : 16;       // K per tcgen05.mma (32 bytes)
  static constexpr int A_BYTES = 128 * 128;      // this CTA's 128 A rows
  static constexpr int B_BYTES = 128 * 128;      // this CTA's 128 B rows
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int EPI_WARP_FLOATS = 32 * 33;
  static constexpr int EPI_BYTES = 4 * EPI_WARP_FLOATS * 4;
  // Packed B (KP > 0): per-lane replicated decode tables after the barriers.
  static constexpr int LUT_BYTES = KP > 0 ? 256 * 32 * 8 + 256 * 8 : 0;
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + EPI_BYTES + 1024 + 256 + LUT_BYTES;
  static constexpr int THREADS = KP > 0 ? 448 : 192;  // packed: + 8 decoder warps
  static constexpr uint32_t TMEM_COLS = 2 * BN;
  static constexpr uint32_t IDESC = instr_desc(kI8, 256, BN, kAMN, kBMN);
};

// Where the packed weight lives (forward from the packed format).
struct PackedB {
  const uint8_t* codes;  // codes plane, row stride crow
  const uint8_t* index;  // index plane, row stride irow
  long long crow, irow;
  int rows;              // d_out
};

// Decodes half `hf` (chunks 8 hf .. 8 hf + 7, 64 weights) of K block `kb`
// of weight row `row` from the packed planes into row `r` of a 128 x
// 128-byte int8 B tile with the 128-byte swizzle (16-byte unit c of row r
// stored at unit c ^ (r % 8)), the layout a TMA load of W_eff would produce.
// Rows past d_out and chunks past d_in/8 load as zero words; what they decode
// to is never used (their outputs are not stored, and the matching
// activations are zero-filled by TMA).  The chunk decoder is the byte-permute
// one of packed_decode.cuh; the scatter-selector table is replicated per
// lane (the entry of mask m for lane l at byte m * 256 + l * 8).
template <int KP>
struct PackedHalf {
  uint32_t w[(KP + 1) / 2 + 1];  // 8 chunks x 2KP bits = 2KP bytes (+1 word of zeros)
  uint2 m;                       // the 8 slot masks
};

template <int KP>
__device__ __forceinline__ void load_packed_half(PackedHalf<KP>& ph, const PackedB& pb, int row, int kb, int hf,
                                                 int nchunks) {
  uint32_t* w = ph.w;
#pragma unroll
  for (int i = 0; i < (KP + 1) / 2 + 1; ++i) w[i] = 0u;
  uint2 m = make_uint2(0u, 0u);
  const int ch0 = kb * 16 + 8 * hf;
  if (row < pb.rows && ch0 < nchunks) {
    const int valid = (nchunks * 2 * KP + 7) / 8;  // code bytes of a row
    const uint8_t* cr = pb.codes + static_cast<long long>(row) * pb.crow;
    const int off = ch0 * 2 * KP / 8;              // 2KP bytes per 8 chunks
    if constexpr ((KP & 1) == 0) {
#pragma unroll
      for (int i = 0; i < KP / 2; ++i)
        if (off + 4 * i < valid) w[i] = __ldg(reinterpret_cast<const uint32_t*>(cr + off) + i);
    } else {
#pragma unroll
      for (int i = 0; i < KP; ++i)
        if (off + 2 * i < valid)
          w[i >> 1] |= static_cast<uint32_t>(__ldg(reinterpret_cast<const uint16_t*>(cr + off) + i)) << (16 * (i & 1));
    }
    m = __ldg(reinterpret_cast<const uint2*>(pb.index + static_cast<long long>(row) * pb.irow + ch0));
  }
  ph.m = m;
}

template <int KP>
__device__ __forceinline__ void expand_packed_half(const PackedHalf<KP>& ph, int hf, uint8_t* tile, int r,
                                                   const uint8_t* sel_bytes, uint32_t lane8) {
  const uint32_t* w = ph.w;
  const uint2 m = ph.m;
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    uint32_t out[4];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int j = 2 * c + h;  // chunk within the half
      const int bit = 2 * KP * j;
      const int wi = bit >> 5, sh = bit & 31;
      const uint32_t v = sh == 0 ? w[wi] : __funnelshift_r(w[wi], w[wi + 1], sh);
      uint32_t lo, hi;
      ChunkCodes<KP>::decode(v, lo, hi);
      const uint32_t amsel = 0x5504u | (static_cast<uint32_t>(j & 3) << 4);
      const uint2 sel = *reinterpret_cast<const uint2*>(sel_bytes + prmt(j < 4 ? m.x : m.y, lane8, amsel));
      out[2 * h] = prmt(lo, hi, sel.x);
      out[2 * h + 1] = prmt(lo, hi, sel.y);
    }
    const int unit = 4 * hf + c;  // 16-byte unit within the 128-byte row
    *reinterpret_cast<uint4*>(tile + r * 128 + ((unit ^ (r & 7)) << 4)) = make_uint4(out[0], out[1], out[2], out[3]);
  }
}

// Several independent products in one launch (the projections of a layer):
// per problem its two tensor maps, arguments and tile schedule; work items
// are numbered problem after problem (the host orders problems heaviest
// first), and every role of the kernel finds an item's problem the same way.
// G = 1 is the single product.
template <int G>
struct alignas(64) PairGroup {
  CUtensorMap tmA[G];
  CUtensorMap tmB[G];
  GemmArgs args[G];
  Sched sched[G];
  int item_start[G + 1];
  int count, total;
  __device__ __forceinline__ void locate(int w, int& p, int& mb, int& nb, int& sp) const {
    p = 0;
    if constexpr (G > 1) {
      while (p + 1 < count && w >= item_start[p + 1]) ++p;
    }
    sched[p].item(w - item_start[p], mb, nb, sp);
  }
};

template <bool kI8, bool kAMN, bool kBMN, int STAGES, int EPI, int KP = 0, int G = 1>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(KP > 0 ? 448 : kThreads, 1)
    tc_gemm_pair_kernel(const __grid_constant__ PairGroup<G> grp, const PackedB pb) {
  const GemmArgs& args = grp.args[0];  // fields shared by the group (err) and the single product
  using C = Cfg2<kI8, kAMN, kBMN, STAGES, KP>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* epi_tiles = reinterpret_cast<float*>(smem + STAGES * C::STAGE_BYTES);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * C::STAGE_BYTES + C::EPI_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tempty + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  uint8_t* sel_bytes = smem + STAGES * C::STAGE_BYTES + C::EPI_BYTES + 256;  // KP > 0: [256][32] uint2
  uint2* sel_one = reinterpret_cast<uint2*>(sel_bytes + 256 * 32 * 8);        // KP > 0: [256] uint2

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = pair::cluster_rank();
  const bool leader = rank == 0;
  const int pair_id = blockIdx.x >> 1;
  const int n_pairs = gridDim.x >> 1;
  const uint32_t peer_abort = pair::map_to(smem_u32(const_cast<int*>(abort_flag)), rank ^ 1u);

  if (threadIdx.x == 0) pdl_launch_dependents();
  if constexpr (KP > 0) {
    for (int i = threadIdx.x; i < 256; i += blockDim.x) {
      uint32_t s0, s1;
      scatter_selectors(static_cast<uint32_t>(i), KP, s0, s1);
      sel_one[i] = make_uint2(s0, s1);
    }
    __syncthreads();
    uint2* tab = reinterpret_cast<uint2*>(sel_bytes);
    for (int i = threadIdx.x; i < 256 * 32; i += blockDim.x) tab[i] = sel_one[i >> 5];
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      // packed B: the even CTA's producer plus 8 decoder warps of each CTA
      mbar_init(&full[s], KP > 0 ? 17 : 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 8);
    }
    *abort_flag = 0;
    fence_mbar_init();
    for (int i = 0; i < grp.count; ++i) {
      tma_prefetch_desc(&grp.tmA[i]);
      if constexpr (KP == 0) tma_prefetch_desc(&grp.tmB[i]);
    }
  }
  if (warp == 1) {
    pair::tmem_alloc(tmem_slot, C::TMEM_COLS);
    pair::tmem_relinquish();
  }
  tc_fence_before();
  pair::cluster_sync();  // barriers of both CTAs initialised, TMEM allocated, tables built
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait();

  auto give_up = [&]() {
    *abort_flag = 1;
    pair::store_remote_u32(peer_abort, 1u);
  };

  if (warp == 0) {
    if (lane == 0) {
      int it = 0;
      bool ok = true;
      for (int w = pair_id; w < grp.total && ok; w += n_pairs) {
        int pi, mb, nb, sp;
        grp.locate(w, pi, mb, nb, sp);
        const GemmArgs& A = grp.args[pi];
        const CUtensorMap* tmA = &grp.tmA[pi];
        const CUtensorMap* tmB = &grp.tmB[pi];
        const int KB = (A.K + C::BK - 1) / C::BK;
        const int kb0 = sp * A.kb_per_split;
        const int kb1 = min(KB, kb0 + A.kb_per_split);
        const int m0 = mb * 256 + 128 * static_cast<int>(rank);
        const int n0 = nb * C::BN + 128 * static_cast<int>(rank);
        for (int kb = kb0; kb < kb1; ++kb) {
          const int s = it % STAGES;
          const uint32_t round = static_cast<uint32_t>(it / STAGES);
          if (!mbar_wait(&empty[s], (round & 1u) ^ 1u, abort_flag, args.err)) {
            give_up();
            ok = false;
            break;
          }
          if (leader) mbar_arrive_expect_tx(&full[s], KP > 0 ? 2 * C::A_BYTES : 2 * C::STAGE_BYTES);
          const uint32_t fbar = pair::map_to(smem_u32(&full[s]), 0u);
          uint8_t* sa = smem + s * C::STAGE_BYTES;
          uint8_t* sb = sa + C::A_BYTES;
          const int kc = kb * C::BK;
          if constexpr (!kAMN) {
            pair::tma_load_2d(sa, tmA, fbar, kc, m0);
          } else {
            pair::tma_load_2d(sa, tmA, fbar, m0, kc);
            pair::tma_load_2d(sa + C::BK * 128, tmA, fbar, m0 + 64, kc);
          }
          if constexpr (KP == 0) {
            if constexpr (!kBMN) {
              pair::tma_load_2d(sb, tmB, fbar, kc, n0);
            } else {
              pair::tma_load_2d(sb, tmB, fbar, n0, kc);
              pair::tma_load_2d(sb + C::BK * 128, tmB, fbar, n0 + 64, kc);
            }
          }
          ++it;
        }
      }
      if (!ok && leader) {
        for (int i = (it > STAGES ? it - STAGES : 0); i < it; ++i)
          mbar_wait(&full[i % STAGES], static_cast<uint32_t>(i / STAGES) & 1u, nullptr, args.err);
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      int it = 0, t = 0;
      bool ok = true;
      for (int w = pair_id; w < grp.total && ok; w += n_pairs, ++t) {
        int pi, mb, nb, sp;
        grp.locate(w, pi, mb, nb, sp);
        const GemmArgs& A = grp.args[pi];
        const int KB = (A.K + C::BK - 1) / C::BK;
        const int kb0 = sp * A.kb_per_split;
        const int kb1 = min(KB, kb0 + A.kb_per_split);
        const int b = t & 1;
        if (!mbar_wait(&tempty[b], (static_cast<uint32_t>(t >> 1) & 1u) ^ 1u, abort_flag, args.err)) {
          give_up();
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(b * C::BN);
        for (int kb = kb0; kb < kb1; ++kb) {
          const int s = it % STAGES;
          const uint32_t round = static_cast<uint32_t>(it / STAGES);
          if (!mbar_wait(&full[s], round & 1u, abort_flag, args.err)) {
            give_up();
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + s * C::STAGE_BYTES);
          const uint32_t sb = sa + C::A_BYTES;
#pragma unroll
          for (int kk = 0; kk < C::BK / C::UK; ++kk) {
            const uint64_t adesc = kAMN ? smem_desc_sw128(sa + kk * C::UK * 128, C::BK * 128, 1024)
                                        : smem_desc_sw128(sa + kk * 32, 16, 1024);
            const uint64_t bdesc = kBMN ? smem_desc_sw128(sb + kk * C::UK * 128, C::BK * 128, 1024)
                                        : smem_desc_sw128(sb + kk * 32, 16, 1024);
            pair::umma<kI8>(d_tmem, adesc, bdesc, C::IDESC, (kb > kb0 || kk > 0) ? 1u : 0u);
          }
          pair::umma_commit_multicast(&empty[s], 0x3);
          ++it;
        }
        pair::umma_commit_multicast(&tfull[b], 0x3);
      }
    }
  } else if (KP > 0 && warp >= 6) {
    if constexpr (KP > 0) {
      // Decoder warps 6-13: thread (r, hf) expands half hf of row r of this
      // CTA's 128-row B half for every K block, one stage ahead of the MMA
      // like the TMA producer.
      const int dt = (warp - 6) * 32 + lane;
      const int r = dt & 127, hf = dt >> 7;
      const int nchunks = args.K / 8;
      const int KB = (args.K + C::BK - 1) / C::BK;
      const Sched& sched = grp.sched[0];
      // Walk the same (item, k block) sequence as the TMA producer; the
      // packed words of the next k block are loaded (from L2) into registers
      // before waiting for the current stage, hiding the load latency.
      int w = pair_id, kb = 0, kb1 = 0, row = 0;
      auto start_item = [&](int item) {
        int mb, nb, sp;
        sched.item(item, mb, nb, sp);
        kb = sp * args.kb_per_split;
        kb1 = min(KB, kb + args.kb_per_split);
        row = nb * C::BN + 128 * static_cast<int>(rank) + r;
      };
      if (w < grp.total) start_item(w);
      PackedHalf<KP> cur, nxt;
      if (w < grp.total) load_packed_half<KP>(cur, pb, row, kb, hf, nchunks);
      int it = 0;
      while (w < grp.total) {
        // position of the next k block in the sequence
        int nw = w, nkb = kb + 1, nkb1 = kb1, nrow = row;
        if (nkb >= kb1) {
          nw = w + n_pairs;
          if (nw < grp.total) {
            int mb, nb, sp;
            sched.item(nw, mb, nb, sp);
            nkb = sp * args.kb_per_split;
            nkb1 = min(KB, nkb + args.kb_per_split);
            nrow = nb * C::BN + 128 * static_cast<int>(rank) + r;
          }
        }
        if (nw < grp.total) load_packed_half<KP>(nxt, pb, nrow, nkb, hf, nchunks);
        const int s = it % STAGES;
        const uint32_t round = static_cast<uint32_t>(it / STAGES);
        const bool waited = mbar_wait(&empty[s], (round & 1u) ^ 1u, abort_flag, args.err);
        if (!__all_sync(0xFFFFFFFFu, waited)) {  // the whole warp leaves together
          give_up();
          break;
        }
        uint8_t* sb = smem + s * C::STAGE_BYTES + C::A_BYTES;
        expand_packed_half<KP>(cur, hf, sb, r, sel_bytes, static_cast<uint32_t>(lane) * 8u);
        // make the generic-proxy stores visible to the tensor core (async proxy)
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
        if (lane == 0) {
          const uint32_t fb = pair::map_to(smem_u32(&full[s]), 0u);
          asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(fb) : "memory");
        }
        ++it;
        w = nw;
        kb = nkb;
        kb1 = nkb1;
        row = nrow;
        cur = nxt;
      }
    }
  } else {
    const int q = warp & 3;
    float* tile = epi_tiles + q * C::EPI_WARP_FLOATS;
    int t = 0;
    for (int w = pair_id; w < grp.total; w += n_pairs, ++t) {
      int pi, mb, nb, sp;
      grp.locate(w, pi, mb, nb, sp);
      const GemmArgs& A = grp.args[pi];
      const int b = t & 1;
      if (!mbar_wait(&tfull[b], static_cast<uint32_t>(t >> 1) & 1u, abort_flag, args.err)) {
        give_up();
        break;
      }
      tc_fence_after();
      if (*abort_flag) break;
      const int row0 = mb * 256 + 128 * static_cast<int>(rank) + 32 * q;
      const int row = row0 + lane;
      float scale = 0.0f;
      if constexpr (EPI == kEpiFwd) {
        if (row < A.M) scale = __fmul_rn(*A.gamma, __fdiv_rn(A.amax[row], 127.0f));
      } else if constexpr (EPI == kEpiDx) {
        scale = *A.gamma;
      }
      const uint32_t tbase = tmem_base + (static_cast<uint32_t>(32 * q) << 16) + static_cast<uint32_t>(b * C::BN);
#pragma unroll 1
      for (int c = 0; c < C::BN / 32; ++c) {
        const int col0 = nb * C::BN + 32 * c;
        if (col0 >= A.N) break;  // warp-uniform
        uint32_t r[32];
        tmem_ld_32x32b_x32(tbase + static_cast<uint32_t>(32 * c), r);
        tmem_ld_wait();
        epilogue_chunk<EPI>(A, tile, row0, col0, lane, r, scale);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) pair::mbar_arrive_remote(pair::map_to(smem_u32(&tempty[b]), 0u));
    }
  }
  tc_fence_before();
  pair::cluster_sync();  // no MMA, copy or arrive of either CTA is still in flight
  if (warp == 1) {
    tc_fence_after();
    pair::tmem_dealloc(tmem_base, C::TMEM_COLS);
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

}  // namespace

bool make_tmap_u32(CUtensorMap* m, const void* base, unsigned long long inner, unsigned long long rows,
                   unsigned long long row_bytes, unsigned box_inner, unsigned box_rows) {
  EncodeTiledFn enc = encoder();
  if (enc == nullptr) return false;
  const cuuint64_t dims[2] = {inner, rows};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_inner, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_tmap_u8(CUtensorMap* m, const void* base, unsigned long long inner, unsigned long long rows,
                  unsigned long long row_bytes, unsigned box_inner, unsigned box_rows, bool swizzle128) {
  EncodeTiledFn enc = encoder();
  if (enc == nullptr) return false;
  const cuuint64_t dims[2] = {inner, rows};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_inner, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

namespace {

// Launch with programmatic stream serialization (see pdl_wait).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), int grid, int threads, int smem, cudaStream_t stream,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(static_cast<unsigned>(threads));
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<Args&&>(args)...);
}

template <bool kI8, bool kAMN, bool kBMN, int BN, int STAGES, int EPI>
cudaError_t run(const CUtensorMap& ta, const CUtensorMap& tb, const GemmArgs& a, int splits, int num_sms,
                cudaStream_t stream) {
  using C = Cfg<kI8, kAMN, kBMN, BN, STAGES>;
  auto kern = tc_gemm_kernel<kI8, kAMN, kBMN, BN, STAGES, EPI>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  Sched sc;
  sc.Mt = (a.M + BM - 1) / BM;
  sc.Nt = (a.N + BN - 1) / BN;
  sc.splits = splits;
  sc.total = sc.Mt * sc.Nt * splits;
  sc.GM = 1;
  const int grid = sc.total < num_sms ? sc.total : num_sms;
  return launch_pdl(kern, grid, kThreads, C::SMEM_BYTES, stream, ta, tb, a, sc);
}

// Strip height (m blocks) that minimises the estimated DRAM bytes of the
// operands.  The c tiles in flight span mw m blocks and nw n blocks: n
// fastest (gm = 1) gives mw = ceil(c / Nt), nw = min(Nt, c); strips of gm
// give mw = min(gm, c), nw = min(Nt, ceil(c / gm)).  A (a_bytes in total) is
// then read about Nt / nw times and B about Mt / mw times, except that an
// operand small enough to stay in L2 (48 MB) is read once.  Candidates: 1
// and all m blocks.
int pick_strip(int Mt, int Nt, int c, double a_bytes, double b_bytes) {
  constexpr double kL2Resident = 48.0 * 1024 * 1024;
  auto cost = [&](int gm) {
    double mw, nw;
    if (gm == 1) {
      mw = (c + Nt - 1) / Nt;
      nw = Nt < c ? Nt : c;
    } else {
      mw = gm < c ? gm : c;
      const int n = (c + gm - 1) / gm;
      nw = n < Nt ? n : Nt;
    }
    const double a_reads = (a_bytes <= kL2Resident) ? 1.0 : (Nt / nw > 1.0 ? Nt / nw : 1.0);
    const double b_reads = (b_bytes <= kL2Resident) ? 1.0 : (Mt / mw > 1.0 ? Mt / mw : 1.0);
    return a_bytes * a_reads + b_bytes * b_reads;
  };
  return cost(Mt) < cost(1) ? Mt : 1;
}

template <bool kI8, bool kAMN, bool kBMN, int STAGES, int EPI, int KP = 0>
cudaError_t run_pair(const CUtensorMap& ta, const CUtensorMap& tb, const GemmArgs& a, int splits, int num_sms,
                     cudaStream_t stream, double a_bytes, double b_bytes, const PackedB& pb = PackedB{}) {
  using C = Cfg2<kI8, kAMN, kBMN, STAGES, KP>;
  auto kern = tc_gemm_pair_kernel<kI8, kAMN, kBMN, STAGES, EPI, KP, 1>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  Sched sc;
  sc.Mt = (a.M + 255) / 256;
  sc.Nt = (a.N + C::BN - 1) / C::BN;
  sc.splits = splits;
  sc.total = sc.Mt * sc.Nt * splits;
  int pairs = num_sms / 2;
  if (pairs > sc.total) pairs = sc.total;
  sc.GM = pick_strip(sc.Mt, sc.Nt, pairs, a_bytes, b_bytes);
  PairGroup<1> grp{};
  grp.tmA[0] = ta;
  grp.tmB[0] = tb;
  grp.args[0] = a;
  grp.sched[0] = sc;
  grp.item_start[0] = 0;
  grp.item_start[1] = sc.total;
  grp.count = 1;
  grp.total = sc.total;
  return launch_pdl(kern, 2 * pairs, C::THREADS, C::SMEM_BYTES, stream, grp, pb);
}

constexpr int kFwdGroup = 8;  // products of one grouped forward launch at most

constexpr int kBN = 256;
constexpr int kStages = 4;
constexpr int kPairStages = 6;
constexpr int kPackedStages = 4;

}  // namespace

// Which tensor-core kernel the products use: 0 = CTA pairs (default),
// 1 = one CTA per 128 x 256 tile.  Process-wide; set through
// sbl_set_gemm_variant().
std::atomic<int> g_gemm_variant{0};

namespace {

}  // namespace

namespace {
// Forward with split K: the GEMM has added the exact integer sums into Y as
// fp32 values (|acc| <= 128 d_in < 2^24); turn them into y = fp32(acc) *
// fp32(gamma * fp32(amax_t / 127)) in place, with the same operations as the
// GEMM epilogue, and copy the sums to `acc` when it is given.  d_out % 8 ==
// 0, so a 16-byte vector never straddles two rows.
__global__ void __launch_bounds__(256) fwd_split_finalize_kernel(float4* __restrict__ Y, int4* __restrict__ acc,
                                                                 const float* __restrict__ amax,
                                                                 const float* __restrict__ gamma, int d_out,
                                                                 size_t n4) {
  const float gm = *gamma;
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n4;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const int row = static_cast<int>((4 * i) / static_cast<size_t>(d_out));
    const float sc = __fmul_rn(gm, __fdiv_rn(amax[row], 127.0f));
    const float4 f = Y[i];  // exact integers
    if (acc != nullptr)
      acc[i] = make_int4(__float2int_rn(f.x), __float2int_rn(f.y), __float2int_rn(f.z), __float2int_rn(f.w));
    Y[i] = make_float4(__fmul_rn(f.x, sc), __fmul_rn(f.y, sc), __fmul_rn(f.z, sc), __fmul_rn(f.w, sc));
  }
}
}  // namespace

cudaError_t launch_forward(const int8_t* Xq, const float* amax, const int8_t* W_eff, const float* gamma, int T,
                           int d_in, int d_out, float* Y, int32_t* acc, cudaStream_t stream, int num_sms,
                           uint32_t* err) {
  if (T == 0 || d_out == 0) return cudaSuccess;
  if (d_in == 0) {
    cudaError_t e = cudaMemsetAsync(Y, 0, sizeof(float) * static_cast<size_t>(T) * d_out, stream);
    if (e == cudaSuccess && acc != nullptr)
      e = cudaMemsetAsync(acc, 0, sizeof(int32_t) * static_cast<size_t>(T) * d_out, stream);
    return e;
  }
  const bool use_pair = g_gemm_variant == 0;
  CUtensorMap ta, tb;
  if (!make_tmap(&ta, Xq, false, d_in, T, d_in, 128, BM)) return cudaErrorInvalidValue;
  if (!make_tmap(&tb, W_eff, false, d_in, d_out, d_in, 128, use_pair ? 128 : kBN)) return cudaErrorInvalidValue;
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
  if (use_pair) {
    // Few output tiles (a short token batch): split K so every CTA pair has
    // work.  The splits add their exact integer sums into Y, which a second
    // pass scales in place (bit-identical to the unsplit product).
    const int KB = (d_in + 127) / 128;
    const int tiles = ((T + 255) / 256) * ((d_out + 255) / 256);
    const int pairs = num_sms / 2;
    int splits = 1;
    if (tiles < pairs && d_in < (1 << 17)) {  // 128 * d_in < 2^24: exact fp32 partial sums
      splits = pairs / tiles;
      if (splits > KB / 4) splits = KB / 4;  // at least four K blocks per split
      if (splits < 1) splits = 1;
    }
    if (splits > 1) {
      a.kb_per_split = (KB + splits - 1) / splits;
      splits = (KB + a.kb_per_split - 1) / a.kb_per_split;
      a.atomic_i32 = 1;
      const size_t n = static_cast<size_t>(T) * d_out;
      cudaError_t e = cudaMemsetAsync(Y, 0, sizeof(float) * n, stream);
      if (e != cudaSuccess) return e;
      e = run_pair<true, false, false, kPairStages, kEpiFwd>(ta, tb, a, splits, num_sms, stream,
                                                             static_cast<double>(T) * d_in,
                                                             static_cast<double>(d_out) * d_in);
      if (e != cudaSuccess) return e;
      const size_t n4 = n / 4;
      size_t blocks = (n4 + 255) / 256;
      if (blocks > static_cast<size_t>(num_sms) * 8) blocks = static_cast<size_t>(num_sms) * 8;
      fwd_split_finalize_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
          reinterpret_cast<float4*>(Y), reinterpret_cast<int4*>(acc), amax, gamma, d_out, n4);
      return cudaGetLastError();
    }
    return run_pair<true, false, false, kPairStages, kEpiFwd>(ta, tb, a, 1, num_sms, stream,
                                                             static_cast<double>(T) * d_in,
                                                             static_cast<double>(d_out) * d_in);
  }
  return run<true, false, false, kBN, kStages, kEpiFwd>(ta, tb, a, 1, num_sms, stream);
}

cudaError_t launch_forward_group(const FwdProblemDev* probs, int count, cudaStream_t stream, int num_sms,
                                 uint32_t* err) {
  // One launch pays the start-up cost once, which is what short token batches
  // need; products that are large together run one by one instead, where each
  // launch keeps its own operands' reuse in L2 (measured: grouping the seven
  // 3B projections halves the pass at 512 tokens and slows it at 32768).
  long long tiles = 0;
  for (int i = 0; i < count; ++i)
    if (probs[i].T > 0 && probs[i].d_out > 0)
      tiles += static_cast<long long>((probs[i].T + 255) / 256) * ((probs[i].d_out + 255) / 256);
  if (g_gemm_variant != 0 || tiles > 4LL * (num_sms / 2)) {  // one launch per product
    for (int i = 0; i < count; ++i) {
      const FwdProblemDev& q = probs[i];
      const cudaError_t e = launch_forward(q.Xq, q.amax, q.W_eff, q.gamma, q.T, q.d_in, q.d_out, q.Y, q.acc, stream,
                                           num_sms, err);
      if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
  }
  using C = Cfg2<true, false, false, kPairStages, 0>;
  for (int c0 = 0; c0 < count; c0 += kFwdGroup) {
    const int cnt = (count - c0) < kFwdGroup ? (count - c0) : kFwdGroup;
    // longest K first: those items take longest and should start first
    int order[kFwdGroup];
    int n = 0;
    for (int i = 0; i < cnt; ++i) {
      const FwdProblemDev& q = probs[c0 + i];
      if (q.T == 0 || q.d_out == 0) continue;
      if (q.d_in == 0) {  // an empty product: zeros
        cudaError_t e = cudaMemsetAsync(q.Y, 0, sizeof(float) * static_cast<size_t>(q.T) * q.d_out, stream);
        if (e == cudaSuccess && q.acc != nullptr)
          e = cudaMemsetAsync(q.acc, 0, sizeof(int32_t) * static_cast<size_t>(q.T) * q.d_out, stream);
        if (e != cudaSuccess) return e;
        continue;
      }
      order[n++] = c0 + i;
    }
    for (int i = 1; i < n; ++i)
      for (int k = i; k > 0 && probs[order[k]].d_in > probs[order[k - 1]].d_in; --k) {
        const int tmp = order[k];
        order[k] = order[k - 1];
        order[k - 1] = tmp;
      }
    if (n == 0) continue;
    // A product whose K loop is much longer than the group's shortest one is
    // cut into K splits of about that length, so its tiles do not set the
    // launch's length alone.  The splits add their exact integer sums into a
    // zeroed Y (|acc| <= 128 * d_in < 2^24 keeps every fp32 partial exact) and
    // a pass after the launch scales Y in place, as the single-product split.
    int kb_min = 1 << 30;
    for (int i = 0; i < n; ++i) kb_min = std::min(kb_min, (probs[order[i]].d_in + 127) / 128);
    int split_of[kFwdGroup];
    for (int i = 0; i < n; ++i) {
      const FwdProblemDev& q = probs[order[i]];
      const int KB = (q.d_in + 127) / 128;
      int splits = 1;
      if (KB >= 2 * kb_min && q.d_in < (1 << 17)) {
        splits = (KB + kb_min - 1) / kb_min;
        if (splits > KB / 4) splits = KB / 4;  // at least four K blocks per split
        if (splits < 1) splits = 1;
      }
      if (splits > 1) {
        const int kbs = (KB + splits - 1) / splits;
        splits = (KB + kbs - 1) / kbs;
      }
      split_of[i] = splits;
      if (splits > 1) {
        const cudaError_t e = cudaMemsetAsync(q.Y, 0, sizeof(float) * static_cast<size_t>(q.T) * q.d_out, stream);
        if (e != cudaSuccess) return e;
      }
    }
    PairGroup<kFwdGroup> grp{};
    int total = 0;
    for (int i = 0; i < n; ++i) {
      const FwdProblemDev& q = probs[order[i]];
      if (!make_tmap(&grp.tmA[i], q.Xq, false, q.d_in, q.T, q.d_in, 128, BM)) return cudaErrorInvalidValue;
      if (!make_tmap(&grp.tmB[i], q.W_eff, false, q.d_in, q.d_out, q.d_in, 128, 128)) return cudaErrorInvalidValue;
      GemmArgs& a = grp.args[i];
      a = GemmArgs{};
      a.M = q.T;
      a.N = q.d_out;
      a.K = q.d_in;
      const int KB = (q.d_in + 127) / 128;
      a.kb_per_split = (KB + split_of[i] - 1) / split_of[i];
      a.atomic_i32 = split_of[i] > 1 ? 1 : 0;
      a.out = q.Y;
      a.ldo = q.d_out;
      a.acc_out = q.acc;
      a.amax = q.amax;
      a.gamma = q.gamma;
      a.err = err;
      Sched& sc = grp.sched[i];
      sc.Mt = (q.T + 255) / 256;
      sc.Nt = (q.d_out + C::BN - 1) / C::BN;
      sc.splits = split_of[i];
      sc.total = sc.Mt * sc.Nt * sc.splits;
      sc.GM = pick_strip(sc.Mt, sc.Nt, num_sms / 2, static_cast<double>(q.T) * q.d_in,
                         static_cast<double>(q.d_out) * q.d_in);
      grp.item_start[i] = total;
      total += sc.total;
    }
    grp.item_start[n] = total;
    grp.count = n;
    grp.total = total;
    int pairs = num_sms / 2;
    if (pairs > total) pairs = total;
    auto kern = tc_gemm_pair_kernel<true, false, false, kPairStages, kEpiFwd, 0, kFwdGroup>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    e = launch_pdl(kern, 2 * pairs, C::THREADS, C::SMEM_BYTES, stream, grp, PackedB{});
    if (e != cudaSuccess) return e;
    for (int i = 0; i < n; ++i) {
      if (split_of[i] == 1) continue;
      const FwdProblemDev& q = probs[order[i]];
      const size_t n4 = static_cast<size_t>(q.T) * q.d_out / 4;
      size_t blocks = (n4 + 255) / 256;
      if (blocks > static_cast<size_t>(num_sms) * 8) blocks = static_cast<size_t>(num_sms) * 8;
      fwd_split_finalize_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
          reinterpret_cast<float4*>(q.Y), reinterpret_cast<int4*>(q.acc), q.amax, q.gamma, q.d_out, n4);
      e = cudaGetLastError();
      if (e != cudaSuccess) return e;
    }
  }
  return cudaSuccess;
}

cudaError_t launch_backward(const void* dY, const void* X, const void* W_eff_bf16, const float* gamma, int T,
                            int d_in, int d_out, float* dX, float* dW, int accumulate_dW, cudaStream_t stream,
                            int num_sms, uint32_t* err) {
  const bool use_pair = g_gemm_variant == 0;
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
      e = use_pair ? run_pair<false, false, true, kPairStages, kEpiDx>(ta, tb, a, 1, num_sms, stream,
                                                                      2.0 * T * d_out, 2.0 * d_out * d_in)
                   : run<false, false, true, kBN, kStages, kEpiDx>(ta, tb, a, 1, num_sms, stream);
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
    const int tiles = use_pair ? ((d_in + 255) / 256) * ((d_out + 255) / 256)
                               : ((d_in + kBN - 1) / kBN) * ((d_out + BM - 1) / BM);
    int splits = (use_pair ? num_sms / 2 : num_sms) / tiles;
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
    e = use_pair ? run_pair<false, true, true, kPairStages, kEpiDw>(ta, tb, a, splits, num_sms, stream,
                                                                   2.0 * T * d_out, 2.0 * T * d_in)
                 : run<false, true, true, kBN, kStages, kEpiDw>(ta, tb, a, splits, num_sms, stream);
  }
  return e;
}

cudaError_t launch_forward_packed(const int8_t* Xq, const float* amax, const uint8_t* packed, const float* gamma,
                                  int T, int d_in, int d_out, int N, int M, float* Y, int32_t* acc,
                                  cudaStream_t stream, int num_sms, uint32_t* err) {
  if (T == 0 || d_out == 0) return cudaSuccess;
  if (d_in == 0) {
    cudaError_t e = cudaMemsetAsync(Y, 0, sizeof(float) * static_cast<size_t>(T) * d_out, stream);
    if (e == cudaSuccess && acc != nullptr)
      e = cudaMemsetAsync(acc, 0, sizeof(int32_t) * static_cast<size_t>(T) * d_out, stream);
    return e;
  }
  CUtensorMap ta;
  if (!make_tmap(&ta, Xq, false, d_in, T, d_in, 128, BM)) return cudaErrorInvalidValue;
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
  PackedB pb{};
  pb.crow = static_cast<long long>(packed_codes_row_bytes(d_in, N, M));
  pb.irow = static_cast<long long>(packed_index_row_bytes(d_in, M));
  pb.codes = packed;
  pb.index = packed + static_cast<size_t>(d_out) * pb.crow;
  pb.rows = d_out;
  const double ab = static_cast<double>(T) * d_in;
  const double bb = static_cast<double>(d_out) * (pb.crow + pb.irow);
  switch (8 * N / M) {
#define SBL_FWD_PACKED(KK) \
  case KK:                 \
    return run_pair<true, false, false, kPackedStages, kEpiFwd, KK>(ta, ta, a, 1, num_sms, stream, ab, bb, pb);
    SBL_FWD_PACKED(1)
    SBL_FWD_PACKED(2)
    SBL_FWD_PACKED(3)
    SBL_FWD_PACKED(4)
    SBL_FWD_PACKED(5)
    SBL_FWD_PACKED(6)
    SBL_FWD_PACKED(7)
    SBL_FWD_PACKED(8)
#undef SBL_FWD_PACKED
    default:
      return cudaErrorInvalidValue;
  }
}

}  // namespace sbl
