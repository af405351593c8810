// gemv_tma.cu -- (a10) decode GEMV on the dense 2-bit ternary layout, fed by
// per-warp TMA rings.
//
// "突破性发现：极低位量化与稀疏化的完美协同", 7.1 推理优化技巧 (the deployed
// weight is a pre-computed 2-bit ternary format, read once per decode step,
// multiplied with bit operations); Sparse-BitNet summary, 核心方法 and
// Algorithm 1 step (6) (y = s * W_eff x~ with int32 accumulation).
//
// y[b, o] = fp32(fp32(acc[b, o]) * fp32(gamma * fp32(amax_b / 127))) with
// acc = sum_j W_eff[o, j] * Xq[b, j] exactly in int32, batch <= 16.  The
// weight is the dense layout: 2-bit codes of every position, rows padded to
// 16 bytes (the codes plane of the 8:8 packed format, so that format is
// served too).
//
// Decode is pure streaming, one launch per layer, each of which may start
// consuming only once its predecessor has finished.  Measured on B200, what
// keeps HBM busy under that rule is the tensor memory accelerator with the
// copies requested before the wait; one warp-instruction per 16 bytes
// (plain or cp.async loads) stalls near half of HBM.  So:
//
//   * Work unit: a round = 16 rows x 256 weights (32 chunks of 8 per row;
//     each lane owns 8 consecutive chunks of rows perm(g) and perm(g) + 8).
//     The k order inside each m16n8k32 MMA is permuted so that a lane's 8
//     positions are one chunk and its activation fragment one 8-byte piece
//     of x.
//   * Schedule: the rounds of all row blocks of the group (longest rows
//     first) form one sequence; block b owns the row blocks that start in
//     [b, b + 1) * total / grid, and its warps split the block's rounds into
//     equal contiguous ranges (a warp may cross row blocks and a row block
//     may be shared by warps).  Every partial sum is an exact int32 added into
//     the block's accumulator of that row block in shared memory; after one
//     block barrier the block scales and stores its rows.  No workspace.
//   * Streaming: lane 0 of each warp copies the warp's stages (up to 4
//     rounds of one row block, 4 KB) into a ring of kDepth slots with 2-D
//     TMA boxes of 16 rows x 128 bytes and the 128-byte swizzle; the ring
//     is filled before griddepcontrol.wait, so the weights of a layer stream
//     in while the previous layer finishes.  16-byte piece c of row r of box
//     kb sits at kb * 2048 + r * 128 + 16 * (c ^ (r & 7)); a lane reads rows
//     perm(g) and perm(g) + 8 with perm = {0, 4, 1, 5, 2, 6, 3, 7}, so the two
//     rows one quarter warp reads differ in bit 2 and never share a bank.
//   * Blocks are small enough (8 warps, about 100 KB) that the next
//     launch's block fits beside a running one; each block asks for its
//     successor at once (programmatic dependent launch).  Activations,
//     scales and outputs are touched only after the wait, and the output
//     scales are requested right after it, off the end of the block.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "packed_decode.cuh"
#include "sbl_device.cuh"
#include "sbl_internal.h"

namespace sbl {
namespace {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kStageRounds = 4;                   // rounds per stage at most
constexpr int kStage = 16 * kStageRounds * 64;    // 4 KB
constexpr int kMaxLocalRB = 24;                   // row blocks one block may own
constexpr int kMaxGroup = 16;

struct DenseProblem {
  const uint8_t* codes;  // dense 2-bit codes, rows of `crow` bytes
  const int8_t* Xq;
  const float* amax;
  const float* gamma;
  float* Y;
  long long base;  // index of the problem's first round in the group's sequence
  int d_in, d_out, nchunks, rounds, nrb, crow;
};

struct DenseGroup {
  DenseProblem p[kMaxGroup];  // longest rows first
  long long total;            // rounds of the whole group
  int count, batch;
};

struct TmaGroup {
  CUtensorMap tm[kMaxGroup];  // uint8 [d_out, crow], box 128 B x 16 rows, 128-byte swizzle
  DenseGroup g;
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

// Position in the group's sequence of rounds: problem, row block of the
// problem, round within the row block, block-local index of the row block.
struct Cursor {
  int pi, rb, r, lrb;
};

__device__ __forceinline__ void advance(const DenseGroup& grp, Cursor& c) {
  if (c.pi >= grp.count) return;
  if (++c.r < grp.p[c.pi].rounds) return;
  c.r = 0;
  ++c.lrb;
  if (++c.rb < grp.p[c.pi].nrb) return;
  c.rb = 0;
  ++c.pi;
}

// The first row block of the group that starts at or after round q (one past
// the last row block if none), with its starting round in *start.
__device__ __forceinline__ Cursor first_at(const DenseGroup& grp, long long q, long long* start) {
  for (int i = 0; i < grp.count; ++i) {
    const DenseProblem& P = grp.p[i];
    const long long end = P.base + static_cast<long long>(P.nrb) * P.rounds;
    if (q < end) {
      const long long rb = q <= P.base ? 0 : (q - P.base + P.rounds - 1) / P.rounds;
      if (rb < P.nrb) {
        *start = P.base + rb * P.rounds;
        return Cursor{i, static_cast<int>(rb), 0, 0};
      }
    }
  }
  *start = grp.total;
  return Cursor{grp.count, 0, 0, 0};
}

// A warp's walk over its rounds in stages: cursor and rounds left in its range.
struct StageWalk {
  Cursor c;
  int left;
};

// Rounds of the stage at w: at most kStageRounds, within the row block and
// within the warp's range.
__device__ __forceinline__ int stage_len(const DenseGroup& grp, const StageWalk& w) {
  return min(kStageRounds, min(grp.p[w.c.pi].rounds - w.c.r, w.left));
}

__device__ __forceinline__ void stage_next(const DenseGroup& grp, StageWalk& w, int n) {
  w.left -= n;
  w.c.r += n;
  if (w.c.r >= grp.p[w.c.pi].rounds) {
    w.c.r = grp.p[w.c.pi].rounds - 1;
    advance(grp, w.c);
  }
}

// Code field of chunk j (0..7) of a lane's 16 bytes (16 bits per chunk).
__device__ __forceinline__ uint32_t field(const uint4& v, int j) {
  const uint32_t w = (j >> 1) == 0 ? v.x : (j >> 1) == 1 ? v.y : (j >> 1) == 2 ? v.z : v.w;
  return (j & 1) ? (w >> 16) : w;
}

// The block's row blocks in order (problem and row block of each local index).
struct LocalRBs {
  int pi[kMaxLocalRB];
  int rb[kMaxLocalRB];
  int n;
};

template <int NT, int DEPTH>
__global__ void __launch_bounds__(kThreads, 2)
    gemv_tma_kernel(const __grid_constant__ TmaGroup params, uint32_t* err) {
  extern __shared__ __align__(1024) uint8_t smem[];
  __shared__ __align__(16) DenseGroup grp;
  __shared__ __align__(8) uint64_t full[kWarps][DEPTH];
  __shared__ LocalRBs lrbs;
  __shared__ float scale[kMaxGroup * 16];
  uint8_t* rings = smem + ((1024u - (smem_u32(smem) & 1023u)) & 1023u);
  int* accum = reinterpret_cast<int*>(rings + kWarps * DEPTH * kStage);  // [kMaxLocalRB][16][8 NT]

  if (threadIdx.x == 0) griddep_launch_dependents();
  // Kernel parameters live in constant memory, cold at every launch, where
  // each miss is a trip to L2: copy the schedule's fields into shared memory
  // once, all threads in parallel (the tensor maps stay where they are).
  {
    static_assert(sizeof(DenseGroup) % 8 == 0, "parameter block copied in 8-byte words");
    const uint2* src = reinterpret_cast<const uint2*>(&params.g);
    uint2* dst = reinterpret_cast<uint2*>(&grp);
    for (int i = threadIdx.x; i < static_cast<int>(sizeof(DenseGroup) / 8); i += kThreads) dst[i] = src[i];
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  if (threadIdx.x < kWarps * DEPTH) mbar_init(&full[0][0] + threadIdx.x, 1);
  if (threadIdx.x == 0) fence_mbar_init();
  __syncthreads();

  const long long G = gridDim.x, b = blockIdx.x;
  long long s0, s1;
  const Cursor c0 = first_at(grp, b * grp.total / G, &s0);
  first_at(grp, (b + 1) * grp.total / G, &s1);
  const long long span = s1 - s0;
  const long long q0 = s0 + warp * span / kWarps, q1 = s0 + (warp + 1) * span / kWarps;
  Cursor cur = c0;  // walk from the block's first row block to round q0
  for (long long skip = q0 - s0; skip > 0 && cur.pi < grp.count;) {
    const int rem = grp.p[cur.pi].rounds - cur.r;
    if (skip < rem) {
      cur.r += static_cast<int>(skip);
      break;
    }
    skip -= rem;
    cur.r = grp.p[cur.pi].rounds - 1;
    advance(grp, cur);
  }
  uint8_t* ring = rings + warp * DEPTH * kStage;

  // Lane 0 copies the warp's stages in order.  A stage of an odd number of
  // rounds copies one round more than it uses (its last box is two rounds
  // wide); boxes past the row or past d_out read zeros.
  StageWalk pw{cur, static_cast<int>(q1 - q0)};
  int issued = 0;
  auto issue_next = [&]() {
    if (pw.left <= 0) return;
    const int n = stage_len(grp, pw);
    if (lane == 0) {
      const int slot = issued % DEPTH;
      uint8_t* dst = ring + slot * kStage;
      const int boxes = (n + 1) >> 1;
      // earlier generic reads of the slot come before the async-proxy copy
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      mbar_arrive_expect_tx(&full[warp][slot], boxes * 2048);
      for (int kb = 0; kb < boxes; ++kb)
        tma_load_2d(dst + kb * 2048, &params.tm[pw.c.pi], &full[warp][slot], (pw.c.r + 2 * kb) * 64, pw.c.rb * 16);
    }
    ++issued;
    stage_next(grp, pw, n);
  };
  // the weights do not depend on the previous kernel: fill the ring first
  for (int i = 0; i < DEPTH; ++i) issue_next();
  if (threadIdx.x == 0) {  // the block's row blocks, for the stores at the end
    Cursor c = c0;
    long long s = s0;
    int l = 0;
    for (; s < s1 && l < kMaxLocalRB; ++l) {
      lrbs.pi[l] = c.pi;
      lrbs.rb[l] = c.rb;
      s += grp.p[c.pi].rounds;
      c.r = grp.p[c.pi].rounds - 1;
      advance(grp, c);
    }
    lrbs.n = l;
  }
  for (int i = threadIdx.x; i < kMaxLocalRB * 16 * 8 * NT; i += kThreads) accum[i] = 0;
  __syncthreads();
  griddep_wait();  // activations, scales and outputs may belong to the previous kernel

  // output scales of every problem and token, requested now and written to
  // shared memory at the end
  const int batch = grp.batch;
  float my_scale = 0.0f;
  if (threadIdx.x < grp.count * batch) {
    const int pi = threadIdx.x / batch, tok = threadIdx.x - pi * batch;
    my_scale = __fmul_rn(*grp.p[pi].gamma, __fdiv_rn(grp.p[pi].amax[tok], 127.0f));
  }

  const int ra = ((g & 1) << 2) | (g >> 1);               // rows ra and ra + 8 of each stage
  const int off0 = ra * 128 + 16 * (t ^ (ra & 7));        // pieces of rounds 0, 2 (+ 2048)
  const int off1 = ra * 128 + 16 * ((4 + t) ^ (ra & 7));  // pieces of rounds 1, 3 (+ 2048)
  bool tv[NT];                                            // tokens g (+ 8) exist
#pragma unroll
  for (int m = 0; m < NT; ++m) tv[m] = m * 8 + g < batch;
  int acc[2][NT][4];
#pragma unroll
  for (int e = 0; e < 2; ++e)
#pragma unroll
    for (int m = 0; m < NT; ++m) acc[e][m][0] = acc[e][m][1] = acc[e][m][2] = acc[e][m][3] = 0;

  // Activations of a stage: x of tokens g (+ 8) at the lane's first chunk of
  // the stage's first round; round rho is 256 * rho bytes further.  Chunks
  // past the row read as zero (nchunks is even).
  struct XStage {
    const uint4* p[NT];
    int chunk0, nchunks;
  };
  auto x_stage = [&](const StageWalk& w, XStage& xs) {
    const DenseProblem& P = grp.p[w.c.pi];
    xs.chunk0 = 32 * w.c.r + 8 * t;
    xs.nchunks = P.nchunks;
#pragma unroll
    for (int m = 0; m < NT; ++m)
      xs.p[m] = reinterpret_cast<const uint4*>(P.Xq + static_cast<size_t>(tv[m] ? m * 8 + g : 0) * P.d_in +
                                               8 * xs.chunk0);
  };
  auto x_load = [&](uint4 (&xv)[NT][4], const XStage& xs, int rho) {
    const int c = xs.chunk0 + 32 * rho;
#pragma unroll
    for (int m = 0; m < NT; ++m) {
      if (tv[m] && c + 8 <= xs.nchunks) {
#pragma unroll
        for (int q = 0; q < 4; ++q) xv[m][q] = __ldg(xs.p[m] + 16 * rho + q);
      } else {
#pragma unroll
        for (int q = 0; q < 4; ++q)
          xv[m][q] = (tv[m] && c + 2 * q < xs.nchunks) ? __ldg(xs.p[m] + 16 * rho + q) : make_uint4(0u, 0u, 0u, 0u);
      }
    }
  };

  using CC = ChunkCodes<8>;
  StageWalk cw{cur, static_cast<int>(q1 - q0)};
  uint4 xb[2][NT][4];  // activations, double-buffered by round parity
  XStage xs_cur{}, xs_next{};
  int n = 0;
  if (cw.left > 0) {
    x_stage(cw, xs_cur);
    n = stage_len(grp, cw);
    x_load(xb[0], xs_cur, 0);
  }
  bool ok = true;
  int consumed = 0;
  while (cw.left > 0 && ok) {
    const int slot = consumed % DEPTH;
    const bool rb_ends = cw.c.r + n == grp.p[cw.c.pi].rounds;
    const int lrb = cw.c.lrb;
    StageWalk nw = cw;  // the next stage, for the activations of its first round
    stage_next(grp, nw, n);
    const bool has_next = nw.left > 0;
    int n_next = 0;
    if (has_next) {
      x_stage(nw, xs_next);
      n_next = stage_len(grp, nw);
    }
    if (!mbar_wait(&full[warp][slot], static_cast<uint32_t>(consumed / DEPTH) & 1u, nullptr, err)) {
      ok = false;
      break;
    }
    const uint8_t* st = ring + slot * kStage;
#pragma unroll
    for (int rho = 0; rho < kStageRounds; ++rho) {
      if (rho < n) {
        const int o = (rho >> 1) * 2048 + ((rho & 1) ? off1 : off0);
        const uint4 wa = *reinterpret_cast<const uint4*>(st + o);
        const uint4 wb = *reinterpret_cast<const uint4*>(st + o + 8 * 128);
        // activations of the next round, one round ahead, into the other buffer
        if (rho + 1 < n) {
          x_load(xb[(rho + 1) & 1], xs_cur, rho + 1);
        } else if (has_next) {
          x_load(xb[(rho + 1) & 1], xs_next, 0);
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          uint32_t a0, a1, a2, a3;
          CC::decode(field(wa, j), a0, a2);
          CC::decode(field(wb, j), a1, a3);
#pragma unroll
          for (int m = 0; m < NT; ++m) {
            const uint4 x = xb[rho & 1][m][j >> 1];
            mma16832(acc[j & 1][m], a0, a1, a2, a3, (j & 1) ? x.z : x.x, (j & 1) ? x.w : x.y);
          }
        }
      }
    }
    // the next stage's first round sits in buffer n & 1; it must be in buffer 0
    if (n & 1) {
#pragma unroll
      for (int m = 0; m < NT; ++m)
#pragma unroll
        for (int q = 0; q < 4; ++q) xb[0][m][q] = xb[1][m][q];
    }
    // every lane is done with the slot: refill it
    __syncwarp();
    ++consumed;
    issue_next();
    if (rb_ends || !has_next) {
      // the warp's part of this row block is done: add it into the block's accumulator
      if (lrb < kMaxLocalRB) {
        int* a = accum + lrb * (16 * 8 * NT);
#pragma unroll
        for (int m = 0; m < NT; ++m) {
          atomicAdd(a + ra * (8 * NT) + m * 8 + 2 * t, acc[0][m][0] + acc[1][m][0]);
          atomicAdd(a + ra * (8 * NT) + m * 8 + 2 * t + 1, acc[0][m][1] + acc[1][m][1]);
          atomicAdd(a + (ra + 8) * (8 * NT) + m * 8 + 2 * t, acc[0][m][2] + acc[1][m][2]);
          atomicAdd(a + (ra + 8) * (8 * NT) + m * 8 + 2 * t + 1, acc[0][m][3] + acc[1][m][3]);
        }
      }
#pragma unroll
      for (int e = 0; e < 2; ++e)
#pragma unroll
        for (int m = 0; m < NT; ++m) acc[e][m][0] = acc[e][m][1] = acc[e][m][2] = acc[e][m][3] = 0;
    }
    cw = nw;
    xs_cur = xs_next;
    n = n_next;
  }
  if (!ok) {  // let this warp's copies in flight land (bounded) before the block's memory is released
    for (int i = consumed; i < issued; ++i)
      mbar_wait(&full[warp][i % DEPTH], static_cast<uint32_t>(i / DEPTH) & 1u, nullptr, err);
  }
  if (threadIdx.x < grp.count * batch) scale[threadIdx.x] = my_scale;
  __syncthreads();

  // scale and store the block's rows: one flat loop over (row block, token, row)
  const int per = 16 * batch;
  for (int i = threadIdx.x; i < lrbs.n * per; i += kThreads) {
    const int l = i / per, rem = i - l * per;
    const int tok = rem >> 4, r16 = rem & 15;
    const int pi = lrbs.pi[l];
    const DenseProblem& P = grp.p[pi];
    const int row = lrbs.rb[l] * 16 + r16;
    if (row < P.d_out)
      P.Y[static_cast<size_t>(tok) * P.d_out + row] =
          __fmul_rn(__int2float_rn(accum[l * (16 * 8 * NT) + r16 * (8 * NT) + tok]), scale[pi * batch + tok]);
  }
}

template <int NT, int DEPTH>
cudaError_t launch_nt(const TmaGroup& grp, int blocks, cudaStream_t stream, uint32_t* err) {
  auto kern = gemv_tma_kernel<NT, DEPTH>;
  const int smem = 1024 + kWarps * DEPTH * kStage + kMaxLocalRB * 16 * 8 * NT * 4;
  const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(blocks));
  cfg.blockDim = dim3(kThreads);
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

cudaError_t launch_gemv_dense_tma(const GemvProblemDev* probs, int count, int batch, cudaStream_t stream,
                                  int num_sms, uint32_t* err) {
  if (count <= 0 || count > kMaxGroup || batch < 1 || batch > 16) return cudaErrorInvalidValue;
  TmaGroup tg{};
  DenseGroup& grp = tg.g;
  int order[kMaxGroup];  // longest rows first (insertion sort, stable)
  for (int i = 0; i < count; ++i) order[i] = i;
  for (int i = 1; i < count; ++i)
    for (int k = i; k > 0 && probs[order[k]].d_in > probs[order[k - 1]].d_in; --k) {
      const int tmp = order[k];
      order[k] = order[k - 1];
      order[k - 1] = tmp;
    }
  long long total = 0;
  int min_rounds = 1 << 30;
  int n = 0;  // problems with work; empty ones are left out of the sequence
  for (int i = 0; i < count; ++i) {
    const GemvProblemDev& q = probs[order[i]];
    if (q.d_out <= 0 || q.d_in <= 0) continue;
    DenseProblem& d = grp.p[n];
    d.crow = static_cast<int>(dense2_row_bytes(q.d_in));
    d.codes = q.packed;
    d.Xq = q.Xq;
    d.amax = q.amax;
    d.gamma = q.gamma;
    d.Y = q.Y;
    d.d_in = q.d_in;
    d.d_out = q.d_out;
    d.nchunks = q.d_in / 8;
    d.rounds = (d.nchunks + 31) / 32;
    d.nrb = (q.d_out + 15) / 16;
    d.base = total;
    total += static_cast<long long>(d.nrb) * d.rounds;
    if (d.rounds < min_rounds) min_rounds = d.rounds;
    if (!make_tmap_u8(&tg.tm[n], d.codes, static_cast<unsigned long long>(d.crow),
                      static_cast<unsigned long long>(d.d_out), static_cast<unsigned long long>(d.crow), 128, 16,
                      true))
      return cudaErrorInvalidValue;
    ++n;
  }
  grp.total = total;
  grp.count = n;
  grp.batch = batch;
  if (total == 0) return cudaSuccess;
  // One block per SM, or more when a block's share would span more row
  // blocks than its accumulator holds.  A block owns the row blocks that
  // start inside an interval of at most ceil(total / grid) rounds, so at most
  // ceil(total / grid) / min_rounds + 1 of them: keep that <= kMaxLocalRB.
  long long blocks = num_sms;
  const long long cap = static_cast<long long>(kMaxLocalRB - 2) * min_rounds;
  const long long need = (total + cap - 1) / cap;
  if (need > blocks) blocks = need;
  if (blocks > total) blocks = total;
  // two blocks per SM (the next launch's beside the running one): a ring of
  // 3 stages per warp at batch <= 8, 2 at batch <= 16 (larger accumulators)
  return batch > 8 ? launch_nt<2, 2>(tg, static_cast<int>(blocks), stream, err)
                   : launch_nt<1, 3>(tg, static_cast<int>(blocks), stream, err);
}

}  // namespace sbl
