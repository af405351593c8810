// pack_gemv.cu -- (a9) packed inference format and (a10) decode GEMV on sm_100a.
//
// Format (per weight row, two planes each padded to 16 bytes; all code rows
// first, then all index rows):
//   codes plane: per chunk of 8 positions (one group at M = 8, two at M = 4;
//     K = 8N/M slots s_0 < ... < s_(K-1), H = ceil(K/2)) a field of 2K bits
//     at bit 2K * chunk of a little-endian bit stream; the code of s_q
//     (q < H) sits at field bits 4q..4q+1, the code of s_(H+q) at 4q+2..4q+3;
//     codes +1 = 00, -1 = 01, 0 = 10 (packed_decode.cuh decodes them);
//   index plane: the M-bit slot mask of every group, little-endian bit stream.
//   Slots = the group's nonzero positions plus, if fewer than N, its lowest
//   zero positions.
// "突破性发现：极低位量化与稀疏化的完美协同", 7.1 推理优化技巧 (pre-computed,
// cached sparse format; bit operations for ternary products); Sparse-BitNet
// summary, 核心方法 (quant-then-mask makes the deployed weights N:M).
//
// Both kernels work on "chunks" of 8 consecutive positions of a row: one
// group when M = 8, two groups when M = 4.  A chunk has K = 8N/M slots,
// 2K code bits and 8 index bits (one index byte).
//
// Decode GEMV: gemv_packed_kernel here is the block-wide tile-ring kernel,
// selected with sbl_set_gemv_variant(1); the default kernel, with a ring per
// warp, is in gemv_direct.cu.  One launch serves a group of independent
// problems (e.g. the seven projections of a layer).
#include <atomic>
#include <cuda.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "packed_decode.cuh"
#include "sbl_device.cuh"
#include "sbl_internal.h"

namespace sbl {

size_t packed_codes_row_bytes(int d_in, int N, int M) {
  const size_t bits = static_cast<size_t>(d_in / M) * N * 2;
  return ((bits + 7) / 8 + 15) / 16 * 16;
}
size_t packed_index_row_bytes(int d_in, int M) {
  const size_t bits = static_cast<size_t>(d_in / M) * M;
  return ((bits + 7) / 8 + 15) / 16 * 16;
}

namespace {

constexpr int kPackChunksPerThread = 8;

__global__ void pack_kernel(const int8_t* __restrict__ W, int d_out, int d_in, int N, int M, uint8_t* __restrict__ packed,
                            size_t crow, size_t irow, uint32_t* err) {
  const int nchunks = d_in / 8;
  const int tpr = (nchunks + kPackChunksPerThread - 1) / kPackChunksPerThread;  // threads per row
  const long long gt = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x;
  if (gt >= static_cast<long long>(d_out) * tpr) return;
  const int row = static_cast<int>(gt / tpr);
  const int c0 = static_cast<int>(gt % tpr) * kPackChunksPerThread;
  const int c1 = min(nchunks, c0 + kPackChunksPerThread);
  const int gpc = 8 / M;             // groups per chunk
  const int cbits = 2 * N * gpc;     // code bits per chunk
  uint8_t* codes = packed + static_cast<size_t>(row) * crow;
  uint8_t* index = packed + static_cast<size_t>(d_out) * crow + static_cast<size_t>(row) * irow;
  const int8_t* wr = W + static_cast<size_t>(row) * d_in;

  unsigned __int128 cbuf = 0;  // code bits of this thread's chunks (<= 8 * 16 bits)
  const int K = gpc * N;        // slots per chunk
  const int H = (K + 1) / 2;
  bool bad = false;
  for (int ch = c0; ch < c1; ++ch) {
    int slot = 0;  // slot index within the chunk
    const uint2 v = *reinterpret_cast<const uint2*>(wr + 8 * ch);
    const uint32_t b[2] = {v.x, v.y};
    uint32_t mask8 = 0;
    for (int g = 0; g < gpc; ++g) {
      uint32_t nz = 0;
      for (int p = 0; p < M; ++p) {
        const int pos = g * M + p;
        const int8_t q = static_cast<int8_t>((b[pos >> 2] >> (8 * (pos & 3))) & 0xFFu);
        if (q != 0) nz |= 1u << p;
      }
      int nnz = __popc(nz);
      if (nnz > N) {
        bad = true;
        nnz = N;
      }
      uint32_t slots = nz;
      int need = N - __popc(nz);
      for (int p = 0; p < M && need > 0; ++p) {
        if (!((slots >> p) & 1u)) {
          slots |= 1u << p;
          --need;
        }
      }
      if (__popc(nz) > N) {  // keep the format well-formed: first N slots only
        uint32_t s = 0;
        int k = 0;
        for (int p = 0; p < M && k < N; ++p)
          if ((nz >> p) & 1u) {
            s |= 1u << p;
            ++k;
          }
        slots = s;
      }
      mask8 |= slots << (g * M);
      for (int p = 0; p < M; ++p) {
        if (!((slots >> p) & 1u)) continue;
        const int pos = g * M + p;
        const int8_t q = static_cast<int8_t>((b[pos >> 2] >> (8 * (pos & 3))) & 0xFFu);
        const uint32_t code = q > 0 ? 0u : (q < 0 ? 1u : 2u);  // +1 00, -1 01, 0 10
        const int fbit = slot < H ? 4 * slot : 4 * (slot - H) + 2;
        cbuf |= static_cast<unsigned __int128>(code) << ((ch - c0) * 2 * K + fbit);
        ++slot;
      }
    }
    index[ch] = static_cast<uint8_t>(mask8);
  }
  // code bits of chunk c0 start at bit c0 * cbits, a multiple of 8 (c0 % 8 == 0).
  const size_t byte0 = static_cast<size_t>(c0) * cbits / 8;
  const int nbytes = ((c1 - c0) * 2 * K + 7) / 8;
  for (int k = 0; k < nbytes; ++k) codes[byte0 + k] = static_cast<uint8_t>(cbuf >> (8 * k));
  if (bad) latch_error(err, kErrDeviceCheck);
}

// ------------------------------------------------------------------- GEMV
// Decode GEMV on int8 tensor cores (mma.sync m16n8k32, s8 x s8 -> s32).
//
// A work unit is 16 (or 8) weight rows of one problem over its whole K; a
// block's 8 consumer warps split every K tile of 256 chunks, 32 chunks each,
// and add their int32 partial sums through shared memory at the end of the
// unit.  The order of the K sum is free, so the 32 k positions of each mma
// are chosen to suit the format: lane (g, t) (g = lane / 4, t = lane % 4)
// owns the 8 consecutive chunks 8t .. 8t+7 of its warp's 32, i.e. one
// aligned run of 2K code bytes and 8 index bytes per row; mma j of the tile
// takes chunk 8t + j from every t.  A chunk decodes to 8 int8 weights:
// positions 0-3 go to k = 4t..4t+3 (A registers a0 / a1 for rows g / g+8)
// and positions 4-7 to k = 16+4t..16+4t+3 (a2 / a3); the B fragment of token
// n = g is then the 8 activations of the same chunk (b0 = positions 0-3,
// b1 = 4-7).  Decoding one chunk (packed_decode.cuh) is two byte permutes
// against constants (slot codes -> int8 values), one permute that builds
// the selector-table address from the slot-mask byte, one 8-byte table load
// and two permutes that move the slot values to their positions.
//
// Problems whose K is at least twice the shortest K of the launch use 8-row
// units (rows g only; a1 = a3 = 0), and units are numbered heaviest problem
// first, so that the persistent blocks' static round-robin over units stays
// balanced.  At the end of a unit each consumer warp adds its int32 partial
// sums into a double-buffered shared accumulator (shared-memory atomics,
// exact and order-free) and moves on; an epilogue warp scales the finished
// sums by fp32(gamma * fp32(amax_b / 127)) and stores them, so no consumer
// ever waits on an output store.  The kernel is launched with programmatic
// dependent launch: the selector table is built and the weight tiles start
// streaming while the previous kernel on the stream finishes; activations,
// scales and outputs are touched only after griddepcontrol.wait.
constexpr int kGemvMaxGroup = 16;

struct alignas(64) GemvGroup {
  CUtensorMap tm_codes[kGemvMaxGroup];  // codes plane as uint32 [d_out, crow / 4], box rows = unit rows
  CUtensorMap tm_index[kGemvMaxGroup];  // index plane as uint32 [d_out, irow / 4], box rows = unit rows
  GemvProblemDev p[kGemvMaxGroup];
  int unit_start[kGemvMaxGroup + 1];    // first work unit of each problem
  int count, batch;
};

__device__ __forceinline__ void mma_s8_16x8x32(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Code field of chunk j (0..7) of a run of 8 chunks held in words w[] (2K bits each).
template <int K>
__device__ __forceinline__ uint32_t chunk_field(const uint32_t (&w)[5], int j) {
  const int bit = 2 * K * j;
  const int wi = bit >> 5, sh = bit & 31;
  return sh == 0 ? w[wi] : __funnelshift_r(w[wi], w[wi + 1], sh);
}

// Scatter-selector table, replicated once per lane: the entry of slot mask
// m for lane l is the uint2 at byte m * 256 + l * 8, so lane l always reads
// banks 2l, 2l+1 and a warp's 32 lookups never conflict.
constexpr int kSelEntries = 256;
constexpr int kSelTableBytes = kSelEntries * 32 * 8;

// Tile of one stage: up to 16 weight rows x 256 chunks (2048 weights) of K.
// Codes: rows x 64K bytes, index: rows x 256 bytes, both loaded by 2-D TMA
// (uint32 elements, no swizzle) into one stage of a shared-memory ring.
constexpr int kTileChunks = 256;
constexpr int kGemvThreads = 320;  // 8 consumer warps + 1 producer warp + 1 epilogue warp

// D2: the dense 2-bit layout (K = 8 slots = the 8 positions, no index plane,
// no selector table, no scatter).
template <int K, bool D2 = false>
struct GemvTile {
  static constexpr int CODE_ROW = kTileChunks * 2 * K / 8;  // bytes per row
  static constexpr int INDEX_ROW = D2 ? 0 : kTileChunks;     // bytes per row
  static constexpr int BYTES = 16 * (CODE_ROW + INDEX_ROW);
  static constexpr int TABLE = D2 ? 0 : kSelTableBytes + kSelEntries * 8;
  // as many stages as still fit two blocks per SM
  static constexpr int STAGES = D2 ? 8 : (K <= 6 ? 4 : 3);
  static constexpr int SMEM = STAGES * BYTES + TABLE + 128;
};

__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;"); }

// One K tile of one consumer warp: decode this lane's 8 chunks of row g
// (and g + 8 when TWO) from the stage and multiply them into acc.
template <int K, int NT, bool TWO, bool D2>
__device__ __forceinline__ void gemv_tile(int (&acc)[2][NT][4], const uint8_t* st, const uint8_t* sel_bytes,
                                          const uint4 (&xv)[NT][4], int warp, int g, int t, uint32_t lane8) {
  using Tl = GemvTile<K, D2>;
  using CC = ChunkCodes<K>;
  const int coff = (warp * 32 + 8 * t) * 2 * K / 8;
  uint32_t wa[5] = {0u, 0u, 0u, 0u, 0u}, wb[5] = {0u, 0u, 0u, 0u, 0u};
  if constexpr ((K & 1) == 0) {
#pragma unroll
    for (int i = 0; i < K / 2; ++i) {
      wa[i] = *reinterpret_cast<const uint32_t*>(st + g * Tl::CODE_ROW + coff + 4 * i);
      if constexpr (TWO) wb[i] = *reinterpret_cast<const uint32_t*>(st + (g + 8) * Tl::CODE_ROW + coff + 4 * i);
    }
  } else {
#pragma unroll
    for (int i = 0; i < K; ++i) {
      wa[i >> 1] |= static_cast<uint32_t>(*reinterpret_cast<const uint16_t*>(st + g * Tl::CODE_ROW + coff + 2 * i))
                    << (16 * (i & 1));
      if constexpr (TWO)
        wb[i >> 1] |= static_cast<uint32_t>(
                          *reinterpret_cast<const uint16_t*>(st + (g + 8) * Tl::CODE_ROW + coff + 2 * i))
                      << (16 * (i & 1));
    }
  }
  if constexpr (D2) {
    // dense 2-bit: the decoded lo / hi words are positions 0-3 / 4-7 already
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      uint32_t a0, a1 = 0u, a2, a3 = 0u;
      CC::decode(chunk_field<K>(wa, j), a0, a2);
      if constexpr (TWO) CC::decode(chunk_field<K>(wb, j), a1, a3);
#pragma unroll
      for (int n = 0; n < NT; ++n) {
        const uint4 x = xv[n][j >> 1];
        mma_s8_16x8x32(acc[j & 1][n], a0, a1, a2, a3, (j & 1) ? x.z : x.x, (j & 1) ? x.w : x.y);
      }
    }
    return;
  }
  const uint8_t* ib = st + 16 * Tl::CODE_ROW;
  const uint2 ma = *reinterpret_cast<const uint2*>(ib + g * Tl::INDEX_ROW + warp * 32 + 8 * t);
  uint2 mb = make_uint2(0u, 0u);
  if constexpr (TWO) mb = *reinterpret_cast<const uint2*>(ib + (g + 8) * Tl::INDEX_ROW + warp * 32 + 8 * t);
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    // mask byte j -> byte 1 of the table offset, lane * 8 in byte 0
    const uint32_t amsel = 0x5504u | (static_cast<uint32_t>(j & 3) << 4);
    uint32_t lo, hi;
    CC::decode(chunk_field<K>(wa, j), lo, hi);
    const uint2 sa = *reinterpret_cast<const uint2*>(sel_bytes + prmt(j < 4 ? ma.x : ma.y, lane8, amsel));
    const uint32_t a0 = prmt(lo, hi, sa.x), a2 = prmt(lo, hi, sa.y);
    uint32_t a1 = 0u, a3 = 0u;
    if constexpr (TWO) {
      CC::decode(chunk_field<K>(wb, j), lo, hi);
      const uint2 sb = *reinterpret_cast<const uint2*>(sel_bytes + prmt(j < 4 ? mb.x : mb.y, lane8, amsel));
      a1 = prmt(lo, hi, sb.x);
      a3 = prmt(lo, hi, sb.y);
    }
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      const uint4 x = xv[n][j >> 1];
      mma_s8_16x8x32(acc[j & 1][n], a0, a1, a2, a3, (j & 1) ? x.z : x.x, (j & 1) ? x.w : x.y);
    }
  }
}

// Persistent: each block walks the work units with stride gridDim.x and,
// within a unit, its K tiles.  Warp 8 (one thread) issues the TMA loads
// Tl::STAGES tiles ahead; warps 0-7 decode and multiply; warp 9 finishes
// the units (scale and store).
template <int K, int NT, bool D2>
__global__ void __launch_bounds__(kGemvThreads, 2)
    gemv_packed_kernel(const __grid_constant__ GemvGroup grp, uint32_t* err) {
  using Tl = GemvTile<K, D2>;
  using CC = ChunkCodes<K>;
  // Every shared pointer below is derived from gsm_raw by pointer arithmetic
  // (no integer casts), so the compiler keeps them in the shared window and
  // emits shared-memory loads with 32-bit addresses.
  extern __shared__ __align__(128) uint8_t gsm_raw[];
  uint8_t* sel_bytes = gsm_raw;                                                 // [256][32] uint2
  uint2* sel_one = reinterpret_cast<uint2*>(gsm_raw + kSelTableBytes);          // [256] uint2
  const uint32_t ring_off = Tl::TABLE;
  uint8_t* ring = gsm_raw + ring_off + ((128u - ((smem_u32(gsm_raw) + ring_off) & 127u)) & 127u);
  __shared__ int s_acc[2][16][16];                  // unit sums [buffer][row][token]
  __shared__ float s_scale[kGemvMaxGroup][16];      // gamma * amax_tok / 127 per problem
  __shared__ __align__(8) uint64_t s_full[Tl::STAGES], s_empty[Tl::STAGES];
  __shared__ __align__(8) uint64_t s_accf[2], s_acce[2];
  __shared__ int s_abort;

  if (threadIdx.x == 0) griddep_launch_dependents();
  if (threadIdx.x == 0) {
    for (int i = 0; i < Tl::STAGES; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_empty[i], 8);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s_accf[b], 8);
      mbar_init(&s_acce[b], 1);
    }
    s_abort = 0;
    fence_mbar_init();
  }
  __syncthreads();  // barriers initialised

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp != 8) {
    // Warps 0-7 and 9 build the selector table and clear the accumulators
    // while the producer (warp 8) already streams the first tiles; named
    // barrier 1 joins only these 288 threads.
    const int tid = warp == 9 ? 256 + lane : static_cast<int>(threadIdx.x);
    if constexpr (!D2) {
      for (int i = tid; i < kSelEntries; i += 288) {
        uint32_t s0, s1;
        scatter_selectors(static_cast<uint32_t>(i), K, s0, s1);
        sel_one[i] = make_uint2(s0, s1);
      }
    }
    for (int i = tid; i < 2 * 16 * 16; i += 288) (&s_acc[0][0][0])[i] = 0;
    asm volatile("bar.sync 1, 288;" ::: "memory");
    if constexpr (!D2) {
      uint2* tab = reinterpret_cast<uint2*>(sel_bytes);
      for (int i = tid; i < kSelEntries * 32; i += 288) tab[i] = sel_one[i >> 5];
    }
    asm volatile("bar.sync 1, 288;" ::: "memory");
  }
  const int total = grp.unit_start[grp.count];
  auto problem_of = [&](int unit) {
    int pi = 0;
    while (pi + 1 < grp.count && unit >= grp.unit_start[pi + 1]) ++pi;
    return pi;
  };

  if (warp == 8) {
    // ---------------- producer (packed weights only: safe before griddepcontrol.wait)
    if (lane == 0) {
      int it = 0;
      bool ok = true;
      for (int unit = blockIdx.x; unit < total && ok; unit += gridDim.x) {
        const int pi = problem_of(unit);
        const int rows = grp.p[pi].rows;
        const int row0 = (unit - grp.unit_start[pi]) * rows;
        const int nkt = (grp.p[pi].d_in / 8 + kTileChunks - 1) / kTileChunks;
        for (int kt = 0; kt < nkt; ++kt, ++it) {
          const int s = it % Tl::STAGES;
          if (!mbar_wait_sleep(&s_empty[s], (static_cast<uint32_t>(it / Tl::STAGES) & 1u) ^ 1u, &s_abort, err)) {
            ok = false;
            break;
          }
          uint8_t* st = ring + s * Tl::BYTES;
          // the consumers' generic-proxy reads of this stage come before the
          // async-proxy copy that overwrites it
          asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
          mbar_arrive_expect_tx(&s_full[s], rows * (Tl::CODE_ROW + Tl::INDEX_ROW));
          tma_load_2d(st, &grp.tm_codes[pi], &s_full[s], kt * (Tl::CODE_ROW / 4), row0);
          if constexpr (!D2)
            tma_load_2d(st + 16 * Tl::CODE_ROW, &grp.tm_index[pi], &s_full[s], kt * (Tl::INDEX_ROW / 4), row0);
        }
      }
      if (!ok) {
        for (int i = (it > Tl::STAGES ? it - Tl::STAGES : 0); i < it; ++i)
          mbar_wait(&s_full[i % Tl::STAGES], static_cast<uint32_t>(i / Tl::STAGES) & 1u, nullptr, err);
      }
    }
    return;
  }

  griddep_wait();  // activations, scales and outputs may come from / go to the previous kernel

  if (warp == 9) {
    // ---------------- epilogue: scale and store the sums of every unit
    for (int i = lane; i < grp.count * 16; i += 32) {
      const int pi = i >> 4, tok = i & 15;
      s_scale[pi][tok] =
          tok < grp.batch ? __fmul_rn(*grp.p[pi].gamma, __fdiv_rn(grp.p[pi].amax[tok], 127.0f)) : 0.0f;
    }
    __syncwarp();
    int u = 0;
    for (int unit = blockIdx.x; unit < total; unit += gridDim.x, ++u) {
      const int b = u & 1;
      if (!mbar_wait_sleep(&s_accf[b], static_cast<uint32_t>(u >> 1) & 1u, &s_abort, err)) break;
      const int pi = problem_of(unit);
      const GemvProblemDev& P = grp.p[pi];
      const int rows = P.rows;
      const int row0 = (unit - grp.unit_start[pi]) * rows;
      for (int i = lane; i < rows * grp.batch; i += 32) {
        const int r = i / grp.batch, tok = i - r * grp.batch;
        const int v = s_acc[b][r][tok];
        s_acc[b][r][tok] = 0;
        if (row0 + r < P.d_out)
          P.Y[static_cast<size_t>(tok) * P.d_out + row0 + r] = __fmul_rn(__int2float_rn(v), s_scale[pi][tok]);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_acce[b]);
    }
    return;
  }

  // ---------------- consumers (warps 0-7)
  const int g = lane >> 2, t = lane & 3;
  const uint32_t lane8 = static_cast<uint32_t>(lane) * 8u;
  int it = 0, u = 0;
  for (int unit = blockIdx.x; unit < total; unit += gridDim.x, ++u) {
    const int pi = problem_of(unit);
    const GemvProblemDev& P = grp.p[pi];
    const bool two = P.rows == 16;  // rows g and g + 8, else rows g only
    const int d_in = P.d_in;
    const int nchunks = d_in / 8;
    const int nkt = (nchunks + kTileChunks - 1) / kTileChunks;

    int acc[2][NT][4];
#pragma unroll
    for (int e = 0; e < 2; ++e)
#pragma unroll
      for (int n = 0; n < NT; ++n) acc[e][n][0] = acc[e][n][1] = acc[e][n][2] = acc[e][n][3] = 0;

    const uint8_t* xr[NT];
    bool tv[NT];
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      const int tok = n * 8 + g;
      tv[n] = tok < grp.batch;
      xr[n] = reinterpret_cast<const uint8_t*>(P.Xq) + static_cast<size_t>(tv[n] ? tok : 0) * d_in;
    }
    bool ok = true;
    for (int kt = 0; kt < nkt; ++kt, ++it) {
      const int s = it % Tl::STAGES;
      // activations of this lane's 8 chunks (64 bytes per token), issued before the wait
      const int chl = kt * kTileChunks + warp * 32 + 8 * t;
      uint4 xv[NT][4];
#pragma unroll
      for (int n = 0; n < NT; ++n)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          xv[n][q] = make_uint4(0u, 0u, 0u, 0u);
          if (tv[n] && chl + 2 * q < nchunks)
            xv[n][q] = __ldg(reinterpret_cast<const uint4*>(xr[n] + static_cast<size_t>(chl + 2 * q) * 8));
        }
      if (!mbar_wait_sleep(&s_full[s], static_cast<uint32_t>(it / Tl::STAGES) & 1u, &s_abort, err)) {
        ok = false;
        break;
      }
      const uint8_t* st = ring + s * Tl::BYTES;
      if (two)
        gemv_tile<K, NT, true, D2>(acc, st, sel_bytes, xv, warp, g, t, lane8);
      else
        gemv_tile<K, NT, false, D2>(acc, st, sel_bytes, xv, warp, g, t, lane8);
      // Free the stage only now: every value read from it has been used by the
      // decode above, so no load of this warp can still be pending when the
      // next TMA copy overwrites the stage.
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_empty[s]);
    }
    if (!ok) break;
    // hand the unit's partial sums to the epilogue warp
    const int b = u & 1;
    if (!mbar_wait_sleep(&s_acce[b], (static_cast<uint32_t>(u >> 1) & 1u) ^ 1u, &s_abort, err)) break;
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      atomicAdd(&s_acc[b][g][n * 8 + 2 * t], acc[0][n][0] + acc[1][n][0]);
      atomicAdd(&s_acc[b][g][n * 8 + 2 * t + 1], acc[0][n][1] + acc[1][n][1]);
      if (two) {
        atomicAdd(&s_acc[b][g + 8][n * 8 + 2 * t], acc[0][n][2] + acc[1][n][2]);
        atomicAdd(&s_acc[b][g + 8][n * 8 + 2 * t + 1], acc[0][n][3] + acc[1][n][3]);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&s_accf[b]);
  }
}

template <int K, bool D2 = false>
cudaError_t launch_gemv_k(const GemvGroup& grp, int units, int num_sms, cudaStream_t stream, uint32_t* err) {
  auto kern = grp.batch <= 8 ? gemv_packed_kernel<K, 1, D2> : gemv_packed_kernel<K, 2, D2>;
  const int smem = GemvTile<K, D2>::SMEM;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kGemvThreads, smem);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) per_sm = 1;
  int blocks = num_sms * per_sm;  // persistent
  if (blocks > units) blocks = units;
  // Programmatic dependent launch: this grid may start while the previous
  // kernel of the stream finishes (see the kernel's griddepcontrol.wait).
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(blocks));
  cfg.blockDim = dim3(kGemvThreads);
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, grp, err);
}

// ----------------------------------------------------------------- unpack
// Packed format -> int8 W_eff [d_out, d_in] (the operand of the dense int8
// forward), for prefill: decoding a weight once and running the dense
// tensor-core product is cheaper than decoding it again for every token
// tile.  One thread per run of 8 chunks (64 weights) of a row: its 2K code
// bytes and 8 mask bytes are read with plain loads, each chunk is decoded by
// packed_decode.cuh (selector table in shared memory, one copy), and the 64
// bytes are stored with four 16-byte stores.  HBM bound.
template <int K>
__global__ void __launch_bounds__(256) unpack_kernel(const uint8_t* __restrict__ packed, int d_out, int d_in,
                                                     size_t crow, size_t irow, int8_t* __restrict__ W) {
  __shared__ uint2 s_sel[256];
  for (int i = threadIdx.x; i < 256; i += blockDim.x) {
    uint32_t s0, s1;
    scatter_selectors(static_cast<uint32_t>(i), K, s0, s1);
    s_sel[i] = make_uint2(s0, s1);
  }
  __syncthreads();
  const int nch = d_in / 8;
  const int runs_per_row = (nch + 7) / 8;
  const long long total = static_cast<long long>(d_out) * runs_per_row;
  const uint8_t* index = packed + static_cast<size_t>(d_out) * crow;
  for (long long it = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; it < total;
       it += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int row = static_cast<int>(it / runs_per_row);
    const int c0 = static_cast<int>(it - static_cast<long long>(row) * runs_per_row) * 8;
    const int nc = min(8, nch - c0);
    // code bits of chunks c0 .. c0 + nc - 1 (2K bits each, starting at a byte boundary: c0 % 8 == 0)
    uint32_t w[5] = {0u, 0u, 0u, 0u, 0u};
    uint8_t m[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    const uint8_t* cr = packed + static_cast<size_t>(row) * crow + static_cast<size_t>(c0) * 2 * K / 8;
    const uint8_t* mr = index + static_cast<size_t>(row) * irow + c0;
    if ((K & 1) == 0 && nc == 8) {
      // a full run: 2K code bytes at a 4-byte aligned offset, 8 mask bytes at an 8-byte aligned one
#pragma unroll
      for (int i = 0; i < K / 2; ++i) w[i] = __ldg(reinterpret_cast<const uint32_t*>(cr) + i);
      const uint2 mm = __ldg(reinterpret_cast<const uint2*>(mr));
#pragma unroll
      for (int j = 0; j < 8; ++j) m[j] = static_cast<uint8_t>(((j < 4 ? mm.x : mm.y) >> (8 * (j & 3))) & 0xFFu);
    } else {
      const int cbytes = (nc * 2 * K + 7) / 8;
      for (int b = 0; b < cbytes; ++b) w[b >> 2] |= static_cast<uint32_t>(cr[b]) << (8 * (b & 3));
      for (int j = 0; j < nc; ++j) m[j] = mr[j];
    }
    int8_t* out = W + static_cast<size_t>(row) * d_in + static_cast<size_t>(c0) * 8;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (j >= nc) break;
      const int bit = 2 * K * j;
      const int wi = bit >> 5, sh = bit & 31;
      const uint32_t v = sh == 0 ? w[wi] : __funnelshift_r(w[wi], w[wi + 1], sh);
      uint32_t lo, hi;
      ChunkCodes<K>::decode(v, lo, hi);
      const uint2 sel = s_sel[m[j]];
      *reinterpret_cast<uint2*>(out + 8 * j) = make_uint2(prmt(lo, hi, sel.x), prmt(lo, hi, sel.y));
    }
  }
}

// W_eff int8 -> dense 2-bit codes: one thread per 16 output bytes (8 chunks,
// 64 weights) of a row; bytes past d_in / 4 (row padding) are written 0.
__global__ void __launch_bounds__(256) pack_dense2_kernel(const int8_t* __restrict__ W, int d_out, int d_in,
                                                          long long row_bytes, uint8_t* __restrict__ out) {
  const long long per_row = row_bytes / 16;
  const long long total = static_cast<long long>(d_out) * per_row;
  const int nch = d_in / 8;
  for (long long it = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; it < total;
       it += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int row = static_cast<int>(it / per_row);
    const int c0 = static_cast<int>(it - static_cast<long long>(row) * per_row) * 8;
    uint32_t f[4] = {0u, 0u, 0u, 0u};
    for (int j = 0; j < 8 && c0 + j < nch; ++j) {
      const uint2 v = __ldg(reinterpret_cast<const uint2*>(W + static_cast<size_t>(row) * d_in) + c0 + j);
      uint32_t field = 0u;
#pragma unroll
      for (int p = 0; p < 8; ++p) {
        const int8_t q = static_cast<int8_t>(((p < 4 ? v.x : v.y) >> (8 * (p & 3))) & 0xFFu);
        const uint32_t code = q > 0 ? 0u : (q < 0 ? 1u : 2u);  // +1 00, -1 01, 0 10
        field |= code << (p < 4 ? 4 * p : 4 * (p - 4) + 2);
      }
      f[j >> 1] |= field << (16 * (j & 1));
    }
    *reinterpret_cast<uint4*>(out + static_cast<size_t>(row) * row_bytes + static_cast<size_t>(c0) * 2) =
        make_uint4(f[0], f[1], f[2], f[3]);
  }
}

}  // namespace

cudaError_t launch_pack(const int8_t* W_eff, int d_out, int d_in, int N, int M, uint8_t* packed,
                        cudaStream_t stream, uint32_t* err) {
  const size_t crow = packed_codes_row_bytes(d_in, N, M);
  const size_t irow = packed_index_row_bytes(d_in, M);
  cudaError_t e = cudaMemsetAsync(packed, 0, static_cast<size_t>(d_out) * (crow + irow), stream);
  if (e != cudaSuccess) return e;
  const int nchunks = d_in / 8;
  const long long threads =
      static_cast<long long>(d_out) * ((nchunks + kPackChunksPerThread - 1) / kPackChunksPerThread);
  if (threads == 0) return cudaSuccess;
  const unsigned blocks = static_cast<unsigned>((threads + 255) / 256);
  pack_kernel<<<blocks, 256, 0, stream>>>(W_eff, d_out, d_in, N, M, packed, crow, irow, err);
  return cudaGetLastError();
}

std::atomic<int> g_gemv_variant{0};

cudaError_t launch_gemv_group(const GemvProblemDev* probs, int count, int batch, int N, int M,
                              cudaStream_t stream, int num_sms, uint32_t* err, bool dense2) {
  if (batch == 0 || count == 0) return cudaSuccess;
  const int variant = g_gemv_variant.load(std::memory_order_relaxed);
  if (variant == 0 || variant == 2) {
    for (int c0 = 0; c0 < count; c0 += kGemvMaxGroup) {
      const int cnt = (count - c0) < kGemvMaxGroup ? (count - c0) : kGemvMaxGroup;
      // the dense layout (and the 8:8 format, whose codes plane it is) through
      // the TMA-fed kernel; the N:M formats through the per-warp ring kernel
      const bool dense = dense2 || N == M;
      const cudaError_t e = (variant == 0 && dense)
                                ? launch_gemv_dense_tma(probs + c0, cnt, batch, stream, num_sms, err)
                                : launch_gemv_direct(probs + c0, cnt, batch, N, M, stream, num_sms, err, dense2);
      if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
  }
  if (dense2) N = M = 8;    // the dense layout is the codes plane of the 8:8 format
  const int K = 8 * N / M;  // slots per 8 positions
  const int code_tile_words = kTileChunks * 2 * K / 32;
  const int index_tile_words = kTileChunks / 4;
  for (int c0 = 0; c0 < count; c0 += kGemvMaxGroup) {
    GemvGroup grp{};
    grp.count = (count - c0) < kGemvMaxGroup ? (count - c0) : kGemvMaxGroup;
    grp.batch = batch;
    // Unit rows: 8 for problems whose K is at least twice the shortest K of
    // the launch, else 16; units are numbered heaviest (rows x K) first.
    int min_chunks = 1 << 30;
    for (int i = 0; i < grp.count; ++i) min_chunks = min(min_chunks, probs[c0 + i].d_in / 8);
    int order[kGemvMaxGroup];
    long long work[kGemvMaxGroup];
    for (int i = 0; i < grp.count; ++i) {
      const int nch = probs[c0 + i].d_in / 8;
      const int rows = nch >= 2 * min_chunks ? 8 : 16;
      work[i] = static_cast<long long>(rows) * nch;
      order[i] = i;
    }
    for (int i = 1; i < grp.count; ++i)  // insertion sort, heaviest first, stable
      for (int j = i; j > 0 && work[order[j]] > work[order[j - 1]]; --j) {
        const int tmp = order[j];
        order[j] = order[j - 1];
        order[j - 1] = tmp;
      }
    int units = 0;
    for (int i = 0; i < grp.count; ++i) {
      GemvProblemDev p = probs[c0 + order[i]];
      p.crow = packed_codes_row_bytes(p.d_in, N, M);
      p.irow = packed_index_row_bytes(p.d_in, M);
      p.rows = p.d_in / 8 >= 2 * min_chunks ? 8 : 16;
      grp.p[i] = p;
      grp.unit_start[i] = units;
      units += (p.d_out + p.rows - 1) / p.rows;
      if (!make_tmap_u32(&grp.tm_codes[i], p.packed, p.crow / 4, p.d_out, p.crow, code_tile_words, p.rows))
        return cudaErrorInvalidValue;
      if (!dense2 && !make_tmap_u32(&grp.tm_index[i], p.packed + static_cast<size_t>(p.d_out) * p.crow, p.irow / 4,
                                    p.d_out, p.irow, index_tile_words, p.rows))
        return cudaErrorInvalidValue;
    }
    grp.unit_start[grp.count] = units;
    if (units == 0) continue;
    cudaError_t e;
    if (dense2) {
      e = launch_gemv_k<8, true>(grp, units, num_sms, stream, err);
      if (e != cudaSuccess) return e;
      continue;
    }
    switch (K) {
      case 1: e = launch_gemv_k<1>(grp, units, num_sms, stream, err); break;
      case 2: e = launch_gemv_k<2>(grp, units, num_sms, stream, err); break;
      case 3: e = launch_gemv_k<3>(grp, units, num_sms, stream, err); break;
      case 4: e = launch_gemv_k<4>(grp, units, num_sms, stream, err); break;
      case 5: e = launch_gemv_k<5>(grp, units, num_sms, stream, err); break;
      case 6: e = launch_gemv_k<6>(grp, units, num_sms, stream, err); break;
      case 7: e = launch_gemv_k<7>(grp, units, num_sms, stream, err); break;
      default: e = launch_gemv_k<8>(grp, units, num_sms, stream, err); break;
    }
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

cudaError_t launch_unpack(const uint8_t* packed, int d_out, int d_in, int N, int M, int8_t* W_eff,
                          cudaStream_t stream, int num_sms) {
  if (d_out == 0 || d_in == 0) return cudaSuccess;
  const size_t crow = packed_codes_row_bytes(d_in, N, M);
  const size_t irow = packed_index_row_bytes(d_in, M);
  const long long runs = static_cast<long long>(d_out) * ((d_in / 8 + 7) / 8);
  long long blocks = (runs + 255) / 256;
  const long long cap = static_cast<long long>(num_sms) * 8;
  if (blocks > cap) blocks = cap;
  const unsigned nb = static_cast<unsigned>(blocks);
  switch (8 * N / M) {
    case 1: unpack_kernel<1><<<nb, 256, 0, stream>>>(packed, d_out, d_in, crow, irow, W_eff); break;
    case 2: unpack_kernel<2><<<nb, 256, 0, stream>>>(packed, d_out, d_in, crow, irow, W_eff); break;
    case 3: unpack_kernel<3><<<nb, 256, 0, stream>>>(packed, d_out, d_in, crow, irow, W_eff); break;
    case 4: unpack_kernel<4><<<nb, 256, 0, stream>>>(packed, d_out, d_in, crow, irow, W_eff); break;
    case 5: unpack_kernel<5><<<nb, 256, 0, stream>>>(packed, d_out, d_in, crow, irow, W_eff); break;
    case 6: unpack_kernel<6><<<nb, 256, 0, stream>>>(packed, d_out, d_in, crow, irow, W_eff); break;
    case 7: unpack_kernel<7><<<nb, 256, 0, stream>>>(packed, d_out, d_in, crow, irow, W_eff); break;
    default: unpack_kernel<8><<<nb, 256, 0, stream>>>(packed, d_out, d_in, crow, irow, W_eff); break;
  }
  return cudaGetLastError();
}

size_t dense2_row_bytes(int d_in) { return (static_cast<size_t>(d_in) / 4 + 15) / 16 * 16; }

cudaError_t launch_pack_dense2(const int8_t* W_eff, int d_out, int d_in, uint8_t* out, cudaStream_t stream,
                               int num_sms) {
  if (d_out == 0 || d_in == 0) return cudaSuccess;
  const long long rb = static_cast<long long>(dense2_row_bytes(d_in));
  const long long total = static_cast<long long>(d_out) * (rb / 16);
  long long blocks = (total + 255) / 256;
  const long long cap = static_cast<long long>(num_sms) * 8;
  if (blocks > cap) blocks = cap;
  pack_dense2_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(W_eff, d_out, d_in, rb, out);
  return cudaGetLastError();
}

cudaError_t launch_gemv_packed(const int8_t* Xq, const float* amax, int batch, const uint8_t* packed,
                               const float* gamma, int d_in, int d_out, int N, int M, float* Y,
                               cudaStream_t stream, int num_sms, uint32_t* err) {
  if (batch == 0 || d_out == 0) return cudaSuccess;
  GemvProblemDev p{};
  p.packed = packed;
  p.Xq = Xq;
  p.amax = amax;
  p.gamma = gamma;
  p.Y = Y;
  p.d_in = d_in;
  p.d_out = d_out;
  return launch_gemv_group(&p, 1, batch, N, M, stream, num_sms, err, false);
}

}  // namespace sbl
