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
//     of x.  A stage is always 4 rounds of one row block (16 rows x 1024
//     weights, 4 KB); the last stage of a row reads zeros past its end, so
//     the inner loop has no length test and no partial stages.
//   * Schedule: the stages of all row blocks of the group (longest rows
//     first) form one sequence; block b owns the row blocks that start in
//     [b, b + 1) * total / grid, and its warps split the block's stages into
//     equal contiguous ranges (a warp may cross row blocks and a row block
//     may be shared by warps).  A warp walks its range with the current
//     problem's fields in registers.  Every partial sum is an exact int32
//     added into the block's accumulator of that row block in shared memory;
//     after one block barrier the block scales and stores its rows.  No
//     workspace.
//   * Streaming: lane 0 of each warp copies the warp's stages into a ring
//     of DEPTH slots with two 2-D TMA boxes of 16 rows x 128 bytes each and
//     the 128-byte swizzle; the ring is filled before griddepcontrol.wait,
//     so the weights of a layer stream in while the previous layer finishes.
//     16-byte piece c of row r of box kb sits at kb * 2048 + r * 128 +
//     16 * (c ^ (r & 7)); a lane reads rows perm(g) and perm(g) + 8 with
//     perm = {0, 4, 1, 5, 2, 6, 3, 7}, so the two rows one quarter warp reads
//     differ in bit 2 and never share a bank.
//   * Blocks are small enough (8 warps, half an SM's shared memory) that the next
//     launch's block fits beside a running one; each block asks for its
//     successor at once (programmatic dependent launch).  Activations,
//     scales and outputs are touched only after the wait, and the output
//     scales are requested right after it, off the end of the block.
#include <cuda.h>
#include <cuda_runtime.h>
#include <atomic>
#include <cstdint>

#include "packed_decode.cuh"
#include "sbl_device.cuh"
#include "sbl_internal.h"

namespace sbl {
namespace {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kRounds = 4;                    // rounds per stage, always
constexpr int kStage = 16 * kRounds * 64;     // 4 KB: 16 rows x 1024 weights
constexpr int kMaxLocalRB = 24;               // row blocks one block may own
constexpr int kMaxGroup = 16;

struct DenseProblem {
  const uint8_t* codes;  // dense 2-bit codes, rows of `crow` bytes
  const int8_t* Xq;
  const float* amax;
  const float* gamma;
  float* Y;
  long long base;  // index of the problem's first stage in the group's sequence
  int d_in, d_out, nchunks, spr, nrb, crow;  // spr: stages per row block
};

struct DenseGroup {
  DenseProblem p[kMaxGroup];  // longest rows first
  long long total;            // stages of the whole group
  int count, batch;
  int xbytes;                 // shared memory for activations (a multiple of 16)
  int pad_;
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

// 1-D bulk copy global -> shared of `bytes` bytes, completion on an mbarrier.
// Both addresses must be 16-byte aligned and `bytes` a multiple of 16.
__device__ __forceinline__ void bulk_load_1d(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(dst)),
               "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;"); }

// The first row block of the group that starts at or after stage q (one past
// the last row block if none): its problem and row block, its first stage in
// *start.
__device__ __forceinline__ int2 first_at(const DenseGroup& grp, long long q, long long* start) {
  for (int i = 0; i < grp.count; ++i) {
    const DenseProblem& P = grp.p[i];
    const long long end = P.base + static_cast<long long>(P.nrb) * P.spr;
    if (q < end) {
      const long long rb = q <= P.base ? 0 : (q - P.base + P.spr - 1) / P.spr;
      if (rb < P.nrb) {
        *start = P.base + rb * P.spr;
        return make_int2(i, static_cast<int>(rb));
      }
    }
  }
  *start = grp.total;
  return make_int2(grp.count, 0);
}

// A walk over a warp's stages, with the fields of the current problem kept in
// registers (they change only when the walk enters the next problem).
template <int NT>
struct Walk {
  int pi, rb, kc, lrb;   // problem, row block, stage within the row block, block-local row block
  int spr, nrb, nchunks;
  bool xsh;              // the activations are in shared memory
  const int8_t* xr[NT];  // activation rows of tokens g and g + 8 (row 0 for tokens past the batch)
};

// xoff[pi] >= 0: the activations of problem pi sit at xs + xoff[pi] in
// shared memory, else they are read from global memory.
template <int NT>
__device__ __forceinline__ void walk_load(const DenseGroup& grp, Walk<NT>& w, int g, const int* xoff,
                                          const int8_t* xs) {
  if (w.pi >= grp.count) return;
  const DenseProblem& P = grp.p[w.pi];
  w.spr = P.spr;
  w.nrb = P.nrb;
  w.nchunks = P.nchunks;
  const int xo = xoff[w.pi];
  w.xsh = xo >= 0;
  const int8_t* x0 = w.xsh ? xs + xo : P.Xq;
#pragma unroll
  for (int m = 0; m < NT; ++m) w.xr[m] = x0 + static_cast<size_t>(m * 8 + g < grp.batch ? m * 8 + g : 0) * P.d_in;
}

template <int NT>
__device__ __forceinline__ void walk_next(const DenseGroup& grp, Walk<NT>& w, int g, const int* xoff,
                                          const int8_t* xs) {
  if (++w.kc < w.spr) return;
  w.kc = 0;
  ++w.lrb;
  if (++w.rb < w.nrb) return;
  w.rb = 0;
  ++w.pi;
  walk_load(grp, w, g, xoff, xs);
}

// Activations of a lane's 8 chunks from chunk c on, of tokens g (+ 8), from
// shared (SH) or global memory.  Chunks past the row read as zero (nchunks
// is even, so a 16-byte piece is either inside the row or past it).
template <int NT, bool SH>
__device__ __forceinline__ void x_fetch(uint4 (&xv)[NT][4], const Walk<NT>& w, int c, const bool (&tv)[NT]) {
#pragma unroll
  for (int m = 0; m < NT; ++m) {
    const uint4* p = reinterpret_cast<const uint4*>(w.xr[m] + 8 * c);
    if (tv[m] && c + 8 <= w.nchunks) {
#pragma unroll
      for (int q = 0; q < 4; ++q) xv[m][q] = SH ? p[q] : __ldg(p + q);
    } else {
#pragma unroll
      for (int q = 0; q < 4; ++q)
        xv[m][q] = (tv[m] && c + 2 * q < w.nchunks) ? (SH ? p[q] : __ldg(p + q)) : make_uint4(0u, 0u, 0u, 0u);
    }
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
  __shared__ int xoff[kMaxGroup];      // offset of each problem's activations in xs, or -1
  __shared__ int xown[kMaxGroup];      // this problem's copy fills its region (not shared with an earlier one)
  __shared__ int xtotal;               // bytes of activations copied into xs
  __shared__ __align__(8) uint64_t xbar;
  uint8_t* rings = smem + ((1024u - (smem_u32(smem) & 1023u)) & 1023u);
  // [kMaxLocalRB][16 rows][batch tokens] exact partial sums, then the activations
  int* accum = reinterpret_cast<int*>(rings + kWarps * DEPTH * kStage);

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
  if (threadIdx.x == 0) {
    mbar_init(&xbar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  const int batch = grp.batch;
  int8_t* xs = reinterpret_cast<int8_t*>(accum + kMaxLocalRB * 16 * batch);

  // The block owns the row blocks that start in [b, b + 1) * total / grid;
  // its warps split those stages into equal contiguous ranges.
  const long long G = gridDim.x, b = blockIdx.x;
  long long s0, s1;
  const int2 c0 = first_at(grp, b * grp.total / G, &s0);
  first_at(grp, (b + 1) * grp.total / G, &s1);
  const long long span = s1 - s0;
  const long long q0 = s0 + warp * span / kWarps, q1 = s0 + (warp + 1) * span / kWarps;
  const int nst = static_cast<int>(q1 - q0);  // this warp's stages
  Walk<NT> start;
  start.pi = c0.x;
  start.rb = c0.y;
  start.kc = 0;
  start.lrb = 0;
  for (long long skip = q0 - s0; skip > 0 && start.pi < grp.count;) {  // move to stage q0
    const DenseProblem& P = grp.p[start.pi];
    const long long rem = static_cast<long long>(P.nrb - start.rb) * P.spr;  // stages left in the problem
    if (skip < rem) {
      const int rbs = static_cast<int>(skip / P.spr);
      start.rb += rbs;
      start.lrb += rbs;
      start.kc = static_cast<int>(skip - static_cast<long long>(rbs) * P.spr);
      break;
    }
    skip -= rem;
    start.lrb += P.nrb - start.rb;
    ++start.pi;
    start.rb = 0;
  }
  start.spr = start.nrb = start.nchunks = 0;
  start.xsh = false;
  walk_load(grp, start, g, xoff, xs);  // schedule fields; the activation rows are set after the barrier
  uint8_t* ring = rings + warp * DEPTH * kStage;

  // Lane 0 copies the warp's stages in order, two boxes of 16 rows x 2
  // rounds each; boxes past the row or past d_out read zeros.
  Walk<NT> pw = start;
  int issued = 0;
  auto issue_next = [&]() {
    if (issued >= nst) return;
    if (lane == 0) {
      const int slot = issued % DEPTH;
      uint8_t* dst = ring + slot * kStage;
      // earlier generic reads of the slot come before the async-proxy copy
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      mbar_arrive_expect_tx(&full[warp][slot], kStage);
      tma_load_2d(dst, &params.tm[pw.pi], &full[warp][slot], pw.kc * (kRounds * 64), pw.rb * 16);
      tma_load_2d(dst + kStage / 2, &params.tm[pw.pi], &full[warp][slot], pw.kc * (kRounds * 64) + 128,
                  pw.rb * 16);
    }
    ++issued;
    walk_next(grp, pw, g, xoff, xs);
  };
  // the weights do not depend on the previous kernel: fill the ring first
  for (int i = 0; i < DEPTH; ++i) issue_next();
  if (threadIdx.x == 0) {  // the block's row blocks, for the stores at the end
    int pi = c0.x, rb = c0.y, l = 0;
    for (long long s = s0; s < s1 && l < kMaxLocalRB && pi < grp.count; ++l) {
      lrbs.pi[l] = pi;
      lrbs.rb[l] = rb;
      s += grp.p[pi].spr;
      if (++rb == grp.p[pi].nrb) {
        rb = 0;
        ++pi;
      }
    }
    lrbs.n = l;
    // Activations of the block's problems go to shared memory while they
    // fit, in order; problems that read the same activations share a copy.
    long long used = 0;
    for (int i = 0; i < kMaxGroup; ++i) xoff[i] = -1, xown[i] = 0;
    if (l > 0) {
      for (int q = lrbs.pi[0]; q <= lrbs.pi[l - 1]; ++q) {
        const DenseProblem& P = grp.p[q];
        for (int e = lrbs.pi[0]; e < q; ++e)
          if (xoff[e] >= 0 && grp.p[e].Xq == P.Xq && grp.p[e].d_in == P.d_in) xoff[q] = xoff[e];
        const long long bytes = static_cast<long long>(batch) * P.d_in;
        if (xoff[q] < 0 && used + bytes <= grp.xbytes) {
          xoff[q] = static_cast<int>(used);
          xown[q] = 1;
          used += bytes;
        }
      }
    }
    xtotal = static_cast<int>(used);  // at most grp.xbytes
  }
  for (int i = threadIdx.x; i < kMaxLocalRB * 16 * batch; i += kThreads) accum[i] = 0;
  __syncthreads();
  griddep_wait();  // activations, scales and outputs may belong to the previous kernel
  if (threadIdx.x == 0 && xtotal > 0) {  // one bulk copy per staged activation tensor
    mbar_arrive_expect_tx(&xbar, static_cast<uint32_t>(xtotal));
    for (int q = 0; q < grp.count; ++q)
      if (xown[q]) bulk_load_1d(xs + xoff[q], grp.p[q].Xq, static_cast<uint32_t>(batch * grp.p[q].d_in), &xbar);
  }

  // gamma and amax of every problem and token, requested now and combined
  // into the output scales at the end, so that no warp waits for them here
  float my_gamma = 0.0f, my_amax = 0.0f;
  if (threadIdx.x < grp.count * batch) {
    const int pi = threadIdx.x / batch, tok = threadIdx.x - pi * batch;
    my_gamma = *grp.p[pi].gamma;
    my_amax = grp.p[pi].amax[tok];
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

  // Activations of round rho of the stage at w (the lane's 8 chunks of that round).
  auto x_load = [&](uint4 (&xv)[NT][4], const Walk<NT>& w, int rho) {
    const int c = w.kc * (kRounds * 32) + 32 * rho + 8 * t;
    if (w.xsh) {
      x_fetch<NT, true>(xv, w, c, tv);
    } else {
      x_fetch<NT, false>(xv, w, c, tv);
    }
  };

  using CC = ChunkCodes<8>;
  Walk<NT> cw = start;
  walk_load(grp, cw, g, xoff, xs);
  uint4 xb[2][NT][4];  // activations, double-buffered by round parity
  bool ok = true;
  if (nst > 0) {
    if (xtotal > 0) ok = mbar_wait(&xbar, 0u, nullptr, err);
    if (ok) x_load(xb[0], cw, 0);
  }
  int s = 0;
  for (; s < nst && ok; ++s) {
    const int slot = s % DEPTH;
    const bool last = s + 1 == nst;
    const bool rb_ends = last || cw.kc + 1 == cw.spr;
    const int lrb = cw.lrb;
    Walk<NT> nw = cw;  // the next stage, for the activations of its first round
    walk_next(grp, nw, g, xoff, xs);
    if (!mbar_wait(&full[warp][slot], static_cast<uint32_t>(s / DEPTH) & 1u, nullptr, err)) {
      ok = false;
      break;
    }
    const uint8_t* st = ring + slot * kStage;
#pragma unroll
    for (int rho = 0; rho < kRounds; ++rho) {
      const int o = (rho >> 1) * 2048 + ((rho & 1) ? off1 : off0);
      const uint4 wa = *reinterpret_cast<const uint4*>(st + o);
      const uint4 wb = *reinterpret_cast<const uint4*>(st + o + 8 * 128);
      // activations of the next round, one round ahead, into the other buffer
      if (rho + 1 < kRounds) {
        x_load(xb[(rho + 1) & 1], cw, rho + 1);
      } else if (!last) {
        x_load(xb[0], nw, 0);
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
    // every lane is done with the slot: refill it
    __syncwarp();
    issue_next();
    if (rb_ends) {
      // the warp's part of this row block is done: add it into the block's accumulator
      if (lrb < kMaxLocalRB) {
        int* a = accum + lrb * (16 * batch);
#pragma unroll
        for (int m = 0; m < NT; ++m) {
          const int tok = m * 8 + 2 * t;  // tokens tok and tok + 1 of rows ra and ra + 8
          if (tok < batch) {
            atomicAdd(a + ra * batch + tok, acc[0][m][0] + acc[1][m][0]);
            atomicAdd(a + (ra + 8) * batch + tok, acc[0][m][2] + acc[1][m][2]);
          }
          if (tok + 1 < batch) {
            atomicAdd(a + ra * batch + tok + 1, acc[0][m][1] + acc[1][m][1]);
            atomicAdd(a + (ra + 8) * batch + tok + 1, acc[0][m][3] + acc[1][m][3]);
          }
        }
      }
#pragma unroll
      for (int e = 0; e < 2; ++e)
#pragma unroll
        for (int m = 0; m < NT; ++m) acc[e][m][0] = acc[e][m][1] = acc[e][m][2] = acc[e][m][3] = 0;
    }
    cw = nw;
  }
  if (!ok) {  // let this warp's copies in flight land (bounded) before the block's memory is released
    for (int i = s; i < issued; ++i)
      mbar_wait(&full[warp][i % DEPTH], static_cast<uint32_t>(i / DEPTH) & 1u, nullptr, err);
  }
  if (threadIdx.x == 0 && xtotal > 0) mbar_wait(&xbar, 0u, nullptr, err);  // no copy in flight at exit
  if (threadIdx.x < grp.count * batch) scale[threadIdx.x] = __fmul_rn(my_gamma, __fdiv_rn(my_amax, 127.0f));
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
          __fmul_rn(__int2float_rn(accum[(l * 16 + r16) * batch + tok]), scale[pi * batch + tok]);
  }
}

template <int NT, int DEPTH>
cudaError_t launch_nt(TmaGroup& tg, int blocks, cudaStream_t stream, uint32_t* err) {
  auto kern = gemv_tma_kernel<NT, DEPTH>;
  // Dynamic shared memory: the rings, the accumulator, and whatever is left
  // under half an SM's shared memory (two blocks per SM) for activations.
  static std::atomic<int> static_smem{-1};
  if (static_smem.load(std::memory_order_relaxed) < 0) {
    cudaFuncAttributes fa{};
    const cudaError_t e = cudaFuncGetAttributes(&fa, kern);
    if (e != cudaSuccess) return e;
    static_smem.store(static_cast<int>(fa.sharedSizeBytes), std::memory_order_relaxed);
  }
  int dev = 0, per_sm = 0, reserved = 0, optin = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&per_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  if (e != cudaSuccess) return e;
  const int st = static_smem.load(std::memory_order_relaxed);
  int dyn_max = per_sm / 2 - reserved - st;
  if (dyn_max > optin - st) dyn_max = optin - st;
  const int base = 1024 + kWarps * DEPTH * kStage + kMaxLocalRB * 16 * tg.g.batch * 4;
  if (dyn_max < base) dyn_max = base;  // one block per SM then, and no staged activations
  tg.g.xbytes = (dyn_max - base) / 16 * 16;
  const int smem = base + tg.g.xbytes;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, dyn_max);
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
  return cudaLaunchKernelEx(&cfg, kern, tg, err);
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
  int min_spr = 1 << 30;
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
    d.spr = (d.nchunks + kRounds * 32 - 1) / (kRounds * 32);
    d.nrb = (q.d_out + 15) / 16;
    d.base = total;
    total += static_cast<long long>(d.nrb) * d.spr;
    if (d.spr < min_spr) min_spr = d.spr;
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
  // start inside an interval of at most ceil(total / grid) stages, so at most
  // ceil(total / grid) / min_spr + 1 of them: keep that <= kMaxLocalRB.
  long long blocks = num_sms;
  const long long cap = static_cast<long long>(kMaxLocalRB - 2) * min_spr;
  const long long need = (total + cap - 1) / cap;
  if (need > blocks) blocks = need;
  if (blocks > total) blocks = total;
  // two blocks per SM (the next launch's beside the running one): a ring of
  // 3 stages per warp at batch 1, whose activation vectors fit beside it; 2
  // stages above, which leaves room to stage the larger activations of
  // batches up to 8 (measured at batch 8: 5% faster than 3 stages) and fits
  // the accumulators and fragments of batches up to 16
  if (batch > 8) return launch_nt<2, 2>(tg, static_cast<int>(blocks), stream, err);
  return batch > 1 ? launch_nt<1, 2>(tg, static_cast<int>(blocks), stream, err)
                   : launch_nt<1, 3>(tg, static_cast<int>(blocks), stream, err);
}

}  // namespace sbl
