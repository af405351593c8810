// gemv_direct.cu -- (a10) decode GEMV on the packed 2-bit ternary + N:M index
// format (and on the dense 2-bit layout): every warp streams its own rows.
//
// "突破性发现：极低位量化与稀疏化的完美协同", 7.1 推理优化技巧 (the deployed
// weight is a pre-computed 2-bit ternary + index format, read once per
// decode step); Sparse-BitNet summary, 核心方法 and Algorithm 1 step (6)
// (y = s * W_eff x~ with int32 accumulation).
//
// y[b, o] = fp32(fp32(acc[b, o]) * fp32(gamma * fp32(amax_b / 127))) with
// acc = sum_j W_eff[o, j] * Xq[b, j] exactly in int32, batch <= 16.
//
// Work decomposition.  A row block is 16 weight rows of one problem (the
// rows of one m16n8k32 MMA).  A row of at most kSliceStages stages (a stage =
// 128 chunks = 1024 weights) is one slice; a longer row is cut into
// one-stage slices, so a block's slices are small enough to share out evenly
// over its warps whatever d_in is.  Row blocks are dealt to
// the persistent blocks (one per SM) round-robin, longest rows first; the
// block's slices go to its 12 warps round-robin.  Each warp owns a ring of
// kRing stages in shared memory that its lane 0 fills with 2-D TMA copies
// (16 rows x one stage of codes, and of slot masks), kRing stages ahead of
// the warp's own consumption and across its slice boundaries, so a warp's
// weight stream never drains; no warp waits for another warp's data.  A
// warp accumulates a whole slice in MMA registers, then:
//   - a row block of one slice is scaled and stored by that warp;
//   - a row block of several slices adds its int32 partial sums into a
//     shared-memory slot with atomics (exact and order-free); the warp that
//     completes the last slice scales and stores it and frees the slot.
// Per chunk of 8 weights a lane runs the byte-permute decode of
// packed_decode.cuh (table-driven scatter for the N:M format, none for the
// dense layout) and feeds whole chunks into m16n8k32 s8 fragments: the k
// order inside each MMA is permuted so a lane's 8 positions are one chunk
// and its activation fragment is one 8-byte piece of x.
//
// Programmatic dependent launch: the selector table is built and the first
// kRing stages of every warp are requested while the previous kernel
// finishes; activations, scales and outputs are touched only after
// griddepcontrol.wait.  Every wait is bounded (sbl_device.cuh).
#include <cuda.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "packed_decode.cuh"
#include "sbl_device.cuh"
#include "sbl_internal.h"

namespace sbl {
namespace {

constexpr int kDWarps = 12;
constexpr int kDThreads = kDWarps * 32;
constexpr int kRing = 2;            // stages in flight per warp
constexpr int kStageChunks = 128;   // 1024 weights per stage: four 32-chunk k-steps
constexpr int kSliceStages = 256 / kStageChunks;  // 2048 weights per slice at most
constexpr int kMaxLocalRB = 256;    // row blocks one block can own in one launch
constexpr int kSlots = 8;           // shared accumulators of split row blocks
constexpr int kDMaxGroup = 16;
constexpr int kSelEntries = 256;
constexpr int kSelTableBytes = kSelEntries * 32 * 8;  // one uint2 per mask and lane

// A stage holds 16 rows of codes then 16 rows of slot masks.  Each row is
// copied 16 bytes wider than the stage's own bytes (the extra bytes are the
// start of the next stage, or zero fill past the row), so that consecutive
// rows start in different shared-memory banks and the lanes of a warp, one
// row per lane group, read without bank conflicts.
template <int K, bool D2>
struct Ring {
  static constexpr int CODE_ROW = kStageChunks * 2 * K / 8;  // code bytes per row and stage (32K)
  static constexpr int MASK_ROW = D2 ? 0 : kStageChunks;     // one mask byte per chunk
  static constexpr int CODE_PITCH = CODE_ROW + 16;
  static constexpr int MASK_PITCH = D2 ? 0 : MASK_ROW + 16;
  static constexpr int STAGE = 16 * (CODE_PITCH + MASK_PITCH);
  static constexpr int TABLE = D2 ? 0 : kSelTableBytes + kSelEntries * 8;
  // warps per block: as many as fit (the 8:8 format's rings need one fewer)
  static constexpr int WARPS = (TABLE + kDWarps * kRing * STAGE + 128 + 16384 <= 232448) ? kDWarps : kDWarps - 1;
  static constexpr int SMEM = TABLE + WARPS * kRing * STAGE + 128;
};

struct DirectProblem {
  const int8_t* Xq;
  const float* amax;
  const float* gamma;
  float* Y;
  int d_in, d_out;
  int nchunks, stages, slices;  // chunks, stages per row; slices per row block
};

struct alignas(64) DirectGroup {
  CUtensorMap tm_codes[kDMaxGroup];  // codes plane, uint32 [d_out, crow / 4], box 16 x CODE_ROW / 4
  CUtensorMap tm_index[kDMaxGroup];  // index plane, uint32 [d_out, irow / 4], box 16 x 16
  DirectProblem p[kDMaxGroup];       // longest rows first
  int rb_start[kDMaxGroup + 1];      // first row block of each problem
  int count, batch;
};

__device__ __forceinline__ void mma16832(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;"); }

// Code field of chunk j (0..7) of a run of 8 chunks held in w[] (2K bits each).
template <int K>
__device__ __forceinline__ uint32_t field(const uint32_t (&w)[5], int j) {
  const int bit = 2 * K * j;
  const int wi = bit >> 5, sh = bit & 31;
  return sh == 0 ? w[wi] : __funnelshift_r(w[wi], w[wi + 1], sh);
}

// The 2K code bytes of 8 chunks of one row, from shared memory (byte offset
// 2K * (chunk / 8): 4-byte aligned for even K, 2-byte aligned for odd K).
template <int K>
__device__ __forceinline__ void read_codes(uint32_t (&w)[5], const uint8_t* p) {
#pragma unroll
  for (int i = 0; i < 5; ++i) w[i] = 0u;
  if constexpr (K == 8) {
    const uint4 v = *reinterpret_cast<const uint4*>(p);
    w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
  } else if constexpr (K == 4) {
    const uint2 v = *reinterpret_cast<const uint2*>(p);
    w[0] = v.x; w[1] = v.y;
  } else if constexpr ((K & 1) == 0) {
#pragma unroll
    for (int i = 0; i < K / 2; ++i) w[i] = *reinterpret_cast<const uint32_t*>(p + 4 * i);
  } else {
#pragma unroll
    for (int i = 0; i < K; ++i)
      w[i >> 1] |= static_cast<uint32_t>(*reinterpret_cast<const uint16_t*>(p + 2 * i)) << (16 * (i & 1));
  }
}

// Activations of one lane for one k-step (chunks c .. c + 7 of its tokens).
template <int NT>
__device__ __forceinline__ void load_x(uint4 (&xv)[NT][4], const int8_t* const (&xr)[NT], const bool (&tv)[NT],
                                       int c, int nchunks) {
#pragma unroll
  for (int n = 0; n < NT; ++n)
#pragma unroll
    for (int q = 0; q < 4; ++q)
      xv[n][q] = (tv[n] && c + 2 * q < nchunks) ? __ldg(reinterpret_cast<const uint4*>(xr[n] + 8 * (c + 2 * q)))
                                                : make_uint4(0u, 0u, 0u, 0u);
}

// Decode a lane's 8 chunks of rows g and g + 8 (code words wa, wb; slot
// masks ma, mb) and multiply them with its activations.
template <int K, int NT, bool D2>
__device__ __forceinline__ void mul_step(int (&acc)[2][NT][4], const uint32_t (&wa)[5], const uint32_t (&wb)[5],
                                         uint2 ma, uint2 mb, const uint4 (&xv)[NT][4], const uint8_t* sel_bytes,
                                         uint32_t lane8) {
  using CC = ChunkCodes<K>;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    uint32_t a0, a1, a2, a3;
    if constexpr (D2) {
      CC::decode(field<K>(wa, j), a0, a2);
      CC::decode(field<K>(wb, j), a1, a3);
    } else {
      const uint32_t amsel = 0x5504u | (static_cast<uint32_t>(j & 3) << 4);
      uint32_t lo, hi;
      CC::decode(field<K>(wa, j), lo, hi);
      const uint2 sa = *reinterpret_cast<const uint2*>(sel_bytes + prmt(j < 4 ? ma.x : ma.y, lane8, amsel));
      a0 = prmt(lo, hi, sa.x);
      a2 = prmt(lo, hi, sa.y);
      CC::decode(field<K>(wb, j), lo, hi);
      const uint2 sb = *reinterpret_cast<const uint2*>(sel_bytes + prmt(j < 4 ? mb.x : mb.y, lane8, amsel));
      a1 = prmt(lo, hi, sb.x);
      a3 = prmt(lo, hi, sb.y);
    }
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      const uint4 x = xv[n][j >> 1];
      mma16832(acc[j & 1][n], a0, a1, a2, a3, (j & 1) ? x.z : x.x, (j & 1) ? x.w : x.y);
    }
  }
}

__device__ __forceinline__ float out_scale(const DirectProblem& P, int tok) {
  return __fmul_rn(*P.gamma, __fdiv_rn(P.amax[tok], 127.0f));
}

// Where a slice of the block lies: local row block li, problem pi, row block
// rb of that problem, and its stage range [st0, st1) within the rows.
struct SliceInfo {
  int li, pi, rb, st0, st1;
};

template <int K, int NT, bool D2>
__global__ void __launch_bounds__(kDThreads, 1)
    gemv_direct_kernel(const __grid_constant__ DirectGroup grp, uint32_t* err) {
  using R = Ring<K, D2>;
  extern __shared__ __align__(128) uint8_t dsm[];
  uint8_t* sel_bytes = dsm;                                        // [256][32] uint2 (N:M format only)
  uint2* sel_one = reinterpret_cast<uint2*>(dsm + kSelTableBytes);  // [256] uint2
  uint8_t* rings = dsm + R::TABLE + ((128u - ((smem_u32(dsm) + R::TABLE) & 127u)) & 127u);
  __shared__ int s_rb[kMaxLocalRB];       // global row block of each local row block
  __shared__ int s_pi[kMaxLocalRB];       // its problem
  __shared__ int s_ord[kMaxLocalRB];      // ordinal among the split local row blocks (-1: one slice)
  __shared__ int s_pre[kMaxLocalRB + 1];  // first slice of each local row block
  __shared__ int s_acc[kSlots][16][16];
  __shared__ int s_cnt[kSlots];
  __shared__ int s_gen[kSlots];
  __shared__ __align__(8) uint64_t s_full[kDWarps][kRing];
  __shared__ int s_total;

  __shared__ int s_rbs[kDMaxGroup + 1], s_stages[kDMaxGroup], s_slices[kDMaxGroup];
  __shared__ int s_S[kMaxLocalRB];

  if (threadIdx.x == 0) griddep_launch_dependents();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = gridDim.x;
  // Kernel parameters live in constant memory, where a miss costs a trip to
  // L2: copy the few per-problem fields the block needs into shared memory
  // once, in parallel, and build the slice list from there.
  if (threadIdx.x <= grp.count) s_rbs[threadIdx.x] = grp.rb_start[threadIdx.x];
  if (threadIdx.x < grp.count) {
    s_stages[threadIdx.x] = grp.p[threadIdx.x].stages;
    s_slices[threadIdx.x] = grp.p[threadIdx.x].slices;
  }
  if (threadIdx.x < R::WARPS * kRing) mbar_init(&s_full[0][0] + threadIdx.x, 1);
  for (int i = threadIdx.x; i < kSlots * 16 * 16; i += blockDim.x) (&s_acc[0][0][0])[i] = 0;
  if (threadIdx.x < kSlots) {
    s_cnt[threadIdx.x] = 0;
    s_gen[threadIdx.x] = 0;
  }
  if (threadIdx.x == 0) fence_mbar_init();
  __syncthreads();
  const int count = grp.count;
  const int total_rb = s_rbs[count];
  int nloc = total_rb > static_cast<int>(blockIdx.x) ? (total_rb - 1 - static_cast<int>(blockIdx.x)) / G + 1 : 0;
  if (nloc > kMaxLocalRB) nloc = kMaxLocalRB;
  for (int i = threadIdx.x; i < nloc; i += blockDim.x) {  // one local row block per thread
    const int u = static_cast<int>(blockIdx.x) + i * G;
    int pi = 0;
    while (pi + 1 < count && u >= s_rbs[pi + 1]) ++pi;
    s_rb[i] = u;
    s_pi[i] = pi;
    s_S[i] = s_slices[pi];
  }
  __syncthreads();
  if (threadIdx.x == 0) {  // prefix sums over a few shared-memory entries
    int pre = 0, ord = 0;
    for (int i = 0; i < nloc; ++i) {
      const int S = s_S[i];
      s_ord[i] = S > 1 ? ord++ : -1;
      s_pre[i] = pre;
      pre += S;
    }
    s_pre[nloc] = pre;
    s_total = pre;
  }
  __syncthreads();  // slice list and barriers ready

  const int total = s_total;
  auto slice_info = [&](int sl) {
    int lo = 0, hi = nloc;  // last li < nloc with s_pre[li] <= sl
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (s_pre[mid] <= sl) lo = mid;
      else hi = mid;
    }
    SliceInfo s;
    s.li = lo;
    s.pi = s_pi[lo];
    s.rb = s_rb[lo] - s_rbs[s.pi];
    const int j = sl - s_pre[lo];
    const int stages = s_stages[s.pi], S = s_slices[s.pi];
    s.st0 = j * stages / S;
    s.st1 = (j + 1) * stages / S;
    return s;
  };
  uint8_t* ring = rings + warp * kRing * R::STAGE;
  uint64_t* full = s_full[warp];

  // ---- producer cursor (lane 0 only): the warp's next stage to request
  int p_sl = warp, p_st = 0;
  SliceInfo p_si{};
  if (p_sl < total) {
    p_si = slice_info(p_sl);
    p_st = p_si.st0;
  }
  int issued = 0;
  auto issue_next = [&]() {
    if (p_sl >= total) return;
    if (lane == 0) {
      // the slot's previous contents were read by the generic proxy; order
      // those reads before the async-proxy copy that overwrites them
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      const int slot = issued % kRing;
      uint8_t* st = ring + slot * R::STAGE;
      mbar_arrive_expect_tx(&full[slot], R::STAGE);
      tma_load_2d(st, &grp.tm_codes[p_si.pi], &full[slot], p_st * (R::CODE_ROW / 4), p_si.rb * 16);
      if constexpr (!D2)
        tma_load_2d(st + 16 * R::CODE_PITCH, &grp.tm_index[p_si.pi], &full[slot], p_st * (R::MASK_ROW / 4),
                    p_si.rb * 16);
    }
    ++issued;
    if (++p_st >= p_si.st1) {
      p_sl += R::WARPS;
      if (p_sl < total) {
        p_si = slice_info(p_sl);
        p_st = p_si.st0;
      }
    }
  };
  // the weights do not depend on the previous kernel: request them first
  for (int i = 0; i < kRing; ++i) issue_next();

  if constexpr (!D2) {
    for (int i = threadIdx.x; i < kSelEntries; i += blockDim.x) {
      uint32_t s0, s1;
      scatter_selectors(static_cast<uint32_t>(i), K, s0, s1);
      sel_one[i] = make_uint2(s0, s1);
    }
    __syncthreads();
    uint2* tab = reinterpret_cast<uint2*>(sel_bytes);
    for (int i = threadIdx.x; i < kSelEntries * 32; i += blockDim.x) tab[i] = sel_one[i >> 5];
    __syncthreads();
  }
  griddep_wait();  // activations, scales and outputs may belong to the previous kernel

  const int g = lane >> 2, t = lane & 3;
  const uint32_t lane8 = static_cast<uint32_t>(lane) * 8u;
  int consumed = 0;
  bool ok = true;
  for (int sl = warp; sl < total && ok; sl += R::WARPS) {
    const SliceInfo si = slice_info(sl);
    const DirectProblem& P = grp.p[si.pi];
    const int8_t* xr[NT];
    bool tv[NT];
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      const int tok = n * 8 + g;
      tv[n] = tok < grp.batch;
      xr[n] = P.Xq + static_cast<size_t>(tv[n] ? tok : 0) * P.d_in;
    }
    int acc[2][NT][4];
#pragma unroll
    for (int e = 0; e < 2; ++e)
#pragma unroll
      for (int n = 0; n < NT; ++n) acc[e][n][0] = acc[e][n][1] = acc[e][n][2] = acc[e][n][3] = 0;

    for (int st = si.st0; st < si.st1; ++st, ++consumed) {
      const int slot = consumed % kRing;
      const int c0 = st * kStageChunks + 8 * t;  // this lane's first chunk of k-step 0
      uint4 xv[NT][4];
      load_x<NT>(xv, xr, tv, c0, P.nchunks);
      if (!mbar_wait_sleep(&full[slot], static_cast<uint32_t>(consumed / kRing) & 1u, nullptr, err)) {
        ok = false;
        break;
      }
      const uint8_t* sp = ring + slot * R::STAGE;
      const uint8_t* mp = sp + 16 * R::CODE_PITCH;
#pragma unroll
      for (int h = 0; h < kStageChunks / 32; h += 2) {
        // two k-steps' codes and masks of rows g and g + 8 into registers
        uint32_t wa0[5], wb0[5], wa1[5], wb1[5];
        uint2 ma0 = make_uint2(0u, 0u), mb0 = ma0, ma1 = ma0, mb1 = ma0;
        read_codes<K>(wa0, sp + g * R::CODE_PITCH + 2 * K * (t + 4 * h));
        read_codes<K>(wb0, sp + (g + 8) * R::CODE_PITCH + 2 * K * (t + 4 * h));
        read_codes<K>(wa1, sp + g * R::CODE_PITCH + 2 * K * (t + 4 * h + 4));
        read_codes<K>(wb1, sp + (g + 8) * R::CODE_PITCH + 2 * K * (t + 4 * h + 4));
        if constexpr (!D2) {
          ma0 = *reinterpret_cast<const uint2*>(mp + g * R::MASK_PITCH + 32 * h + 8 * t);
          mb0 = *reinterpret_cast<const uint2*>(mp + (g + 8) * R::MASK_PITCH + 32 * h + 8 * t);
          ma1 = *reinterpret_cast<const uint2*>(mp + g * R::MASK_PITCH + 32 * h + 32 + 8 * t);
          mb1 = *reinterpret_cast<const uint2*>(mp + (g + 8) * R::MASK_PITCH + 32 * h + 32 + 8 * t);
        }
        if (h + 2 >= kStageChunks / 32) {
          // every lane has read its last values of the stage: the slot may be
          // refilled (a warp barrier that is also a compiler memory barrier, so
          // no read of the slot is moved below the copy that refills it)
          asm volatile("bar.warp.sync -1;" ::: "memory");
          issue_next();
        }
        if (h > 0) load_x<NT>(xv, xr, tv, c0 + 32 * h, P.nchunks);
        mul_step<K, NT, D2>(acc, wa0, wb0, ma0, mb0, xv, sel_bytes, lane8);
        load_x<NT>(xv, xr, tv, c0 + 32 * h + 32, P.nchunks);
        mul_step<K, NT, D2>(acc, wa1, wb1, ma1, mb1, xv, sel_bytes, lane8);
      }
    }
    if (!ok) break;

    // C fragment of lane (g, t): [n][0..1] = row g, tokens n*8+2t, +1; [n][2..3] = row g + 8
    const int r0 = si.rb * 16 + g, r1 = r0 + 8;
    int v[NT][4];
#pragma unroll
    for (int n = 0; n < NT; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) v[n][e] = acc[0][n][e] + acc[1][n][e];
    const int ord = s_ord[si.li];
    if (ord < 0) {
#pragma unroll
      for (int n = 0; n < NT; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int tok = n * 8 + 2 * t + (e & 1);
          const int row = (e < 2) ? r0 : r1;
          if (tok < grp.batch && row < P.d_out)
            P.Y[static_cast<size_t>(tok) * P.d_out + row] = __fmul_rn(__int2float_rn(v[n][e]), out_scale(P, tok));
        }
      continue;
    }
    // split row block: wait (bounded) until slot q has been freed by the
    // split row block kSlots before this one, then add into it
    const int q = ord % kSlots, gen = ord / kSlots;
    int good = 1;
    if (lane == 0) {
      const volatile int* vg = &s_gen[q];
      if (*vg != gen) {
        const uint64_t t0 = globaltimer_ns();
        while (*vg != gen) {
          __nanosleep(64);
          if (globaltimer_ns() - t0 > kWaitLimitNs) {
            latch_error(err, kErrTimeout);
            good = 0;
            break;
          }
        }
      }
    }
    if (!__shfl_sync(0xFFFFFFFFu, good, 0)) {
      ok = false;
      break;
    }
#pragma unroll
    for (int n = 0; n < NT; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int tok = n * 8 + 2 * t + (e & 1);
        if (tok < grp.batch) atomicAdd(&s_acc[q][g + ((e < 2) ? 0 : 8)][tok], v[n][e]);
      }
    __syncwarp();
    int last = 0;
    if (lane == 0) {
      __threadfence_block();
      last = atomicAdd(&s_cnt[q], 1) == s_slices[si.pi] - 1;
    }
    if (__shfl_sync(0xFFFFFFFFu, last, 0)) {
      __threadfence_block();
      for (int i = lane; i < 16 * grp.batch; i += 32) {
        const int r = i / grp.batch, tok = i - r * grp.batch;
        const int val = atomicExch(&s_acc[q][r][tok], 0);
        const int row = si.rb * 16 + r;
        if (row < P.d_out)
          P.Y[static_cast<size_t>(tok) * P.d_out + row] = __fmul_rn(__int2float_rn(val), out_scale(P, tok));
      }
      __syncwarp();
      if (lane == 0) {
        s_cnt[q] = 0;
        __threadfence_block();
        atomicAdd(&s_gen[q], 1);
      }
    }
  }
  // On an abandoned wait, let the copies this warp still has in flight land
  // (bounded) before the block's shared memory is released.
  if (!ok) {
    for (int i = consumed; i < issued; ++i)
      mbar_wait(&full[i % kRing], static_cast<uint32_t>(i / kRing) & 1u, nullptr, err);
  }
}

template <int K, bool D2>
cudaError_t launch_direct_k(const DirectGroup& grp, int blocks, cudaStream_t stream, uint32_t* err) {
  auto kern = grp.batch <= 8 ? gemv_direct_kernel<K, 1, D2> : gemv_direct_kernel<K, 2, D2>;
  const int smem = Ring<K, D2>::SMEM;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(blocks));
  cfg.blockDim = dim3(Ring<K, D2>::WARPS * 32);
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, grp, err);
}

}  // namespace

cudaError_t launch_gemv_direct(const GemvProblemDev* probs, int count, int batch, int N, int M,
                               cudaStream_t stream, int num_sms, uint32_t* err, bool dense2) {
  if (count <= 0 || count > kDMaxGroup || batch < 1 || batch > 16) return cudaErrorInvalidValue;
  if (dense2) N = M = 8;  // the dense layout is the codes plane of the 8:8 format
  const int K = 8 * N / M;
  const int code_box = (kStageChunks * 2 * K / 8 + 16) / 4;  // uint32 words per row and stage, + 16 B
  const int mask_box = (kStageChunks + 16) / 4;
  DirectGroup grp{};
  int order[kDMaxGroup];  // longest rows first (insertion sort, stable)
  for (int i = 0; i < count; ++i) order[i] = i;
  for (int i = 1; i < count; ++i)
    for (int k = i; k > 0 && probs[order[k]].d_in > probs[order[k - 1]].d_in; --k) {
      const int tmp = order[k];
      order[k] = order[k - 1];
      order[k - 1] = tmp;
    }
  int rbs = 0;
  for (int i = 0; i < count; ++i) {
    const GemvProblemDev& q = probs[order[i]];
    const size_t crow = packed_codes_row_bytes(q.d_in, N, M);
    const size_t irow = packed_index_row_bytes(q.d_in, M);
    if (!make_tmap_u32(&grp.tm_codes[i], q.packed, crow / 4, q.d_out, crow, code_box, 16))
      return cudaErrorInvalidValue;
    if (!dense2 && !make_tmap_u32(&grp.tm_index[i], q.packed + static_cast<size_t>(q.d_out) * crow, irow / 4,
                                  q.d_out, irow, mask_box, 16))
      return cudaErrorInvalidValue;
    DirectProblem& d = grp.p[i];
    d.Xq = q.Xq;
    d.amax = q.amax;
    d.gamma = q.gamma;
    d.Y = q.Y;
    d.d_in = q.d_in;
    d.d_out = q.d_out;
    d.nchunks = q.d_in / 8;
    d.stages = (d.nchunks + kStageChunks - 1) / kStageChunks;
    // rows of up to kSliceStages stages stay whole; longer rows are cut into
    // one-stage slices, so the warps of a block that owns a long row block
    // still end up with nearly equal work
    d.slices = d.stages <= kSliceStages ? 1 : d.stages;
    grp.rb_start[i] = rbs;
    rbs += (q.d_out + 15) / 16;
  }
  grp.rb_start[count] = rbs;
  grp.count = count;
  grp.batch = batch;
  if (rbs == 0) return cudaSuccess;
  int blocks = num_sms;
  if (blocks > rbs) blocks = rbs;
  if ((rbs + blocks - 1) / blocks > kMaxLocalRB) blocks = (rbs + kMaxLocalRB - 1) / kMaxLocalRB;
  switch (K) {
    case 8: return dense2 ? launch_direct_k<8, true>(grp, blocks, stream, err)
                          : launch_direct_k<8, false>(grp, blocks, stream, err);
    case 7: return launch_direct_k<7, false>(grp, blocks, stream, err);
    case 6: return launch_direct_k<6, false>(grp, blocks, stream, err);
    case 5: return launch_direct_k<5, false>(grp, blocks, stream, err);
    case 4: return launch_direct_k<4, false>(grp, blocks, stream, err);
    case 3: return launch_direct_k<3, false>(grp, blocks, stream, err);
    case 2: return launch_direct_k<2, false>(grp, blocks, stream, err);
    case 1: return launch_direct_k<1, false>(grp, blocks, stream, err);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace sbl
