// pack_gemv.cu -- (a9) packed inference format and (a10) decode GEMV on sm_100a.
//
// Format (per weight row, two planes each padded to 16 bytes; all code rows
// first, then all index rows):
//   codes plane: the N slot codes of every group of M in ascending position
//     order, 2 bits each (00 = 0, 01 = +1, 11 = -1), little-endian bit stream;
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
// Decode GEMV: see gemv_packed_kernel.  One launch can serve a group of
// independent problems (e.g. the seven projections of a layer).
#include <cuda.h>
#include <cuda_runtime.h>
#include <cstdint>

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
  int cnt = 0;
  bool bad = false;
  for (int ch = c0; ch < c1; ++ch) {
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
        const uint32_t code = q > 0 ? 1u : (q < 0 ? 3u : 0u);
        cbuf |= static_cast<unsigned __int128>(code) << cnt;
        cnt += 2;
      }
    }
    index[ch] = static_cast<uint8_t>(mask8);
  }
  // code bits of chunk c0 start at bit c0 * cbits, a multiple of 8 (c0 % 8 == 0).
  const size_t byte0 = static_cast<size_t>(c0) * cbits / 8;
  const int nbytes = (cnt + 7) / 8;
  for (int k = 0; k < nbytes; ++k) codes[byte0 + k] = static_cast<uint8_t>(cbuf >> (8 * k));
  if (bad) latch_error(err, kErrDeviceCheck);
}

// ------------------------------------------------------------------- GEMV
// Decode GEMV on int8 tensor cores (mma.sync m16n8k32, s8 x s8 -> s32).
//
// A warp computes 16 weight rows x all tokens (up to 16) over a K slice.  The
// order of the K sum is free, so the 32 k positions of each mma are chosen
// to suit the format: within a block of 32 chunks (256 weights of a row),
// lane (g, t) (g = lane / 4, t = lane % 4) owns the 8 consecutive chunks
// 8t .. 8t+7, i.e. one aligned run of 2K code bytes and 8 index bytes per
// row; mma number j of the block takes chunk 8t + j from every t.  A chunk
// decodes to 8 int8 weights: positions 0-3 go to k = 4t..4t+3 (A registers
// a0 / a1 for rows g / g+8) and positions 4-7 to k = 16+4t..16+4t+3 (a2 /
// a3).  The B fragment of token n = g is then the 8 int8 activations of the
// same chunk (b0 = positions 0-3, b1 = 4-7): one 8-byte load.  Decoding a
// chunk: its 2K code bits (K = 8N/M slots), two table lookups (4 codes ->
// 4 int8 each) and two __byte_perm with selectors looked up from the 8-bit
// slot mask.  Warps of a block that share 16 rows split K and add their
// int32 partial sums through shared memory; the result is scaled by
// fp32(gamma * fp32(amax_b / 127)) per token.
constexpr int kGemvMaxGroup = 16;

struct alignas(64) GemvGroup {
  CUtensorMap tm_codes[kGemvMaxGroup];  // codes plane as uint32 [d_out, crow / 4]
  CUtensorMap tm_index[kGemvMaxGroup];  // index plane as uint32 [d_out, irow / 4]
  GemvProblemDev p[kGemvMaxGroup];
  int block_start[kGemvMaxGroup + 1];   // first work item (16-row group) of each problem
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

// Code bits of chunk j (0..7) of a run of 8 chunks held in words w[] (2K bits each).
template <int K>
__device__ __forceinline__ uint32_t chunk_codes(const uint32_t (&w)[5], int j) {
  const int bit = 2 * K * j;
  const int wi = bit >> 5, sh = bit & 31;
  const uint32_t v = __funnelshift_r(w[wi], w[wi + 1], sh);
  return (2 * K == 32) ? v : (v & ((1u << (2 * K)) - 1u));
}

// Lookup tables, replicated once per lane: entry e of copy l sits at word
// e * 32 + l, so lane l always reads bank l and lookups with 32 different
// indices never conflict.
//   code table (64 entries): 3 codes (6 bits) -> 3 int8 values (bytes 0-2);
//   selector table (256 entries): slot mask -> two __byte_perm selectors
//     (low 16 bits: positions 0-3, high 16 bits: positions 4-7) that move
//     slot value i to the position of the i-th set bit and a zero byte
//     (byte 7 of the value pair, always 0) elsewhere.
constexpr int kCodeEntries = 64;
constexpr int kSelEntries = 256;

__device__ __forceinline__ uint32_t code_byte(uint32_t code) {
  return code == 1u ? 0x01u : (code == 3u ? 0xFFu : 0u);
}

// Tile of one work item: 16 weight rows x 256 chunks (2048 weights) of K.
// Codes: 16 rows x 64K bytes, index: 16 rows x 256 bytes, both loaded by 2-D
// TMA (uint32 elements, no swizzle) into one stage of a shared-memory ring.
constexpr int kGemvStages = 4;
constexpr int kTileChunks = 256;
constexpr int kGemvThreads = 288;  // 8 consumer warps + 1 producer warp

template <int K>
struct GemvTile {
  static constexpr int CODE_ROW = kTileChunks * 2 * K / 8;  // bytes per row
  static constexpr int INDEX_ROW = kTileChunks;              // bytes per row
  static constexpr int BYTES = 16 * (CODE_ROW + INDEX_ROW);
};

// Persistent: each block walks the work items (16 rows of one problem) with
// stride gridDim.x and, within an item, its K tiles.  Warp 8 (one thread)
// issues the TMA loads kGemvStages tiles ahead; warps 0-7 each decode 32
// chunks (a 32 x 16 weight slab) of every tile into mma.sync fragments
// (k order as described above), keep the int32 sums of the item in
// registers, and after its last K tile add their partial sums through
// shared memory and write the scaled outputs.
template <int K, int NT>
__global__ void __launch_bounds__(kGemvThreads, 2)
    gemv_packed_kernel(const __grid_constant__ GemvGroup grp, uint32_t* err) {
  using Tl = GemvTile<K>;
  extern __shared__ __align__(128) uint8_t gsm_raw[];
  uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(gsm_raw) + 127) & ~uintptr_t(127));
  uint32_t* s_code = reinterpret_cast<uint32_t*>(ring + kGemvStages * Tl::BYTES);  // [64][32]
  uint32_t* s_sel = s_code + kCodeEntries * 32;                                      // [256][32]
  __shared__ int s_part[8][16][16];
  __shared__ __align__(8) uint64_t s_full[kGemvStages], s_empty[kGemvStages];
  __shared__ int s_abort;

  for (int i = threadIdx.x; i < kCodeEntries * 32; i += blockDim.x) {
    const uint32_t c = static_cast<uint32_t>(i) >> 5;
    s_code[i] = code_byte(c & 3u) | (code_byte((c >> 2) & 3u) << 8) | (code_byte((c >> 4) & 3u) << 16);
  }
  for (int i = threadIdx.x; i < kSelEntries * 32; i += blockDim.x) {
    const uint32_t c = static_cast<uint32_t>(i) >> 5;
    uint32_t sel = 0;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const uint32_t nib = ((c >> q) & 1u) ? static_cast<uint32_t>(__popc(c & ((1u << q) - 1u))) : 7u;
      sel |= nib << (4 * q);
    }
    s_sel[i] = sel;
  }
  if (threadIdx.x == 0) {
    for (int i = 0; i < kGemvStages; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_empty[i], 8);
    }
    s_abort = 0;
    fence_mbar_init();
  }
  __syncthreads();

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int total = grp.block_start[grp.count];
  auto problem_of = [&](int unit) {
    int pi = 0;
    while (pi + 1 < grp.count && unit >= grp.block_start[pi + 1]) ++pi;
    return pi;
  };

  if (warp == 8) {
    // ---------------- producer
    if (lane == 0) {
      int it = 0;
      bool ok = true;
      for (int unit = blockIdx.x; unit < total && ok; unit += gridDim.x) {
        const int pi = problem_of(unit);
        const int row0 = (unit - grp.block_start[pi]) * 16;
        const int nkt = (grp.p[pi].d_in / 8 + kTileChunks - 1) / kTileChunks;
        for (int kt = 0; kt < nkt; ++kt, ++it) {
          const int s = it % kGemvStages;
          if (!mbar_wait(&s_empty[s], (static_cast<uint32_t>(it / kGemvStages) & 1u) ^ 1u, &s_abort, err)) {
            ok = false;
            break;
          }
          uint8_t* st = ring + s * Tl::BYTES;
          mbar_arrive_expect_tx(&s_full[s], Tl::BYTES);
          tma_load_2d(st, &grp.tm_codes[pi], &s_full[s], kt * (Tl::CODE_ROW / 4), row0);
          tma_load_2d(st + 16 * Tl::CODE_ROW, &grp.tm_index[pi], &s_full[s], kt * (Tl::INDEX_ROW / 4), row0);
        }
      }
      if (!ok) {
        for (int i = (it > kGemvStages ? it - kGemvStages : 0); i < it; ++i)
          mbar_wait(&s_full[i % kGemvStages], static_cast<uint32_t>(i / kGemvStages) & 1u, nullptr, err);
      }
    }
    return;  // the producer warp takes no part in the consumers' named barrier
  }

  // ---------------- consumers (warps 0-7)
  const int g = lane >> 2, t = lane & 3;
  int it = 0;
  for (int unit = blockIdx.x; unit < total; unit += gridDim.x) {
    const int pi = problem_of(unit);
    const GemvProblemDev& P = grp.p[pi];
    const int row0 = (unit - grp.block_start[pi]) * 16;
    const int d_in = P.d_in, d_out = P.d_out;
    const int nchunks = d_in / 8;
    const int nkt = (nchunks + kTileChunks - 1) / kTileChunks;

    int acc[2][NT][4];
#pragma unroll
    for (int e = 0; e < 2; ++e)
#pragma unroll
      for (int n = 0; n < NT; ++n) acc[e][n][0] = acc[e][n][1] = acc[e][n][2] = acc[e][n][3] = 0;

    const uint2* xr[NT];
    bool tv[NT];
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      const int tok = n * 8 + g;
      tv[n] = tok < grp.batch;
      xr[n] = reinterpret_cast<const uint2*>(P.Xq + static_cast<size_t>(tv[n] ? tok : 0) * d_in);
    }
    bool ok = true;
    for (int kt = 0; kt < nkt; ++kt, ++it) {
      const int s = it % kGemvStages;
      if (!mbar_wait(&s_full[s], static_cast<uint32_t>(it / kGemvStages) & 1u, &s_abort, err)) {
        ok = false;
        break;
      }
      const uint8_t* st = ring + s * Tl::BYTES;
      const int ch0 = kt * kTileChunks + warp * 32 + 8 * t;  // this lane's first chunk (global index)
      // code words and index bytes of rows g and g + 8 for chunks ch0 .. ch0 + 7
      const int coff = (warp * 32 + 8 * t) * 2 * K / 8;
      uint32_t wa[5] = {0u, 0u, 0u, 0u, 0u}, wb[5] = {0u, 0u, 0u, 0u, 0u};
      if constexpr ((K & 1) == 0) {
#pragma unroll
        for (int i = 0; i < K / 2; ++i) {
          wa[i] = *reinterpret_cast<const uint32_t*>(st + g * Tl::CODE_ROW + coff + 4 * i);
          wb[i] = *reinterpret_cast<const uint32_t*>(st + (g + 8) * Tl::CODE_ROW + coff + 4 * i);
        }
      } else {
#pragma unroll
        for (int i = 0; i < K; ++i) {
          wa[i >> 1] |= static_cast<uint32_t>(*reinterpret_cast<const uint16_t*>(st + g * Tl::CODE_ROW + coff + 2 * i))
                        << (16 * (i & 1));
          wb[i >> 1] |= static_cast<uint32_t>(
                             *reinterpret_cast<const uint16_t*>(st + (g + 8) * Tl::CODE_ROW + coff + 2 * i))
                         << (16 * (i & 1));
        }
      }
      const uint8_t* ib = st + 16 * Tl::CODE_ROW;
      const uint2 ma = *reinterpret_cast<const uint2*>(ib + g * Tl::INDEX_ROW + warp * 32 + 8 * t);
      const uint2 mb = *reinterpret_cast<const uint2*>(ib + (g + 8) * Tl::INDEX_ROW + warp * 32 + 8 * t);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const uint32_t ca = chunk_codes<K>(wa, j), cb = chunk_codes<K>(wb, j);
        const uint32_t mA = ((j < 4 ? ma.x : ma.y) >> (8 * (j & 3))) & 0xFFu;
        const uint32_t mB = ((j < 4 ? mb.x : mb.y) >> (8 * (j & 3))) & 0xFFu;
        // slot values v0..v(K-1) as bytes of (lo, hi); byte 7 stays 0 (K <= 7)
        uint32_t alo, ahi, blo, bhi;
        {
          const uint32_t a0 = s_code[((ca & 63u) << 5) + lane];
          const uint32_t b0v = s_code[((cb & 63u) << 5) + lane];
          if constexpr (K <= 3) {
            alo = a0; ahi = 0u; blo = b0v; bhi = 0u;
          } else {
            const uint32_t a1 = s_code[(((ca >> 6) & 63u) << 5) + lane];
            const uint32_t b1v = s_code[(((cb >> 6) & 63u) << 5) + lane];
            alo = a0 | (a1 << 24);
            blo = b0v | (b1v << 24);
            ahi = a1 >> 8;
            bhi = b1v >> 8;
            if constexpr (K > 6) {
              const uint32_t a2 = s_code[(((ca >> 12) & 63u) << 5) + lane];
              const uint32_t b2 = s_code[(((cb >> 12) & 63u) << 5) + lane];
              ahi |= a2 << 16;
              bhi |= b2 << 16;
            }
          }
        }
        const uint32_t selA = s_sel[(mA << 5) + lane], selB = s_sel[(mB << 5) + lane];
        const uint32_t a_lo = __byte_perm(alo, ahi, selA & 0xFFFFu), a_hi = __byte_perm(alo, ahi, selA >> 16);
        const uint32_t b_lo = __byte_perm(blo, bhi, selB & 0xFFFFu), b_hi = __byte_perm(blo, bhi, selB >> 16);
#pragma unroll
        for (int n = 0; n < NT; ++n) {
          const uint2 x = (tv[n] && ch0 + j < nchunks) ? __ldg(xr[n] + ch0 + j) : make_uint2(0u, 0u);
          mma_s8_16x8x32(acc[j & 1][n], a_lo, b_lo, a_hi, b_hi, x.x, x.y);
        }
      }
      // Free the stage only now: every value read from it has been used by the
      // decode above, so no load of this warp can still be pending when the
      // next TMA copy overwrites the stage.
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_empty[s]);
    }
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      s_part[warp][g][n * 8 + 2 * t] = acc[0][n][0] + acc[1][n][0];
      s_part[warp][g][n * 8 + 2 * t + 1] = acc[0][n][1] + acc[1][n][1];
      s_part[warp][g + 8][n * 8 + 2 * t] = acc[0][n][2] + acc[1][n][2];
      s_part[warp][g + 8][n * 8 + 2 * t + 1] = acc[0][n][3] + acc[1][n][3];
    }
    // Barrier of the 8 consumer warps that also agrees on giving up: every
    // consumer reaches it, so a timed-out wait in one warp cannot strand the
    // others at a barrier.
    uint32_t any_fail;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\tbar.red.or.pred q, 1, 256, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(any_fail)
        : "r"(ok ? 0u : 1u)
        : "memory");
    if (any_fail) break;
    if (threadIdx.x < 16 * grp.batch) {
      const int r = threadIdx.x / grp.batch, tok = threadIdx.x - r * grp.batch;
      const int row = row0 + r;
      if (row < d_out) {
        int sum = 0;
#pragma unroll
        for (int w = 0; w < 8; ++w) sum += s_part[w][r][tok];
        const float sc = __fmul_rn(*P.gamma, __fdiv_rn(P.amax[tok], 127.0f));
        P.Y[static_cast<size_t>(tok) * d_out + row] = __fmul_rn(__int2float_rn(sum), sc);
      }
    }
    asm volatile("bar.sync 1, 256;" ::: "memory");
  }
}

template <int K>
cudaError_t launch_gemv_k(const GemvGroup& grp, int units, int num_sms, cudaStream_t stream, uint32_t* err) {
  auto kern = grp.batch <= 8 ? gemv_packed_kernel<K, 1> : gemv_packed_kernel<K, 2>;
  const int smem = kGemvStages * GemvTile<K>::BYTES + (kCodeEntries + kSelEntries) * 32 * 4 + 128;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kGemvThreads, smem);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) per_sm = 1;
  int blocks = num_sms * per_sm;  // persistent
  if (blocks > units) blocks = units;
  kern<<<blocks, kGemvThreads, smem, stream>>>(grp, err);
  return cudaGetLastError();
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

cudaError_t launch_gemv_group(const GemvProblemDev* probs, int count, int batch, int N, int M,
                              cudaStream_t stream, int num_sms, uint32_t* err) {
  if (batch == 0 || count == 0) return cudaSuccess;
  const int K = 8 * N / M;  // slots per 8 positions
  const int code_tile_words = kTileChunks * 2 * K / 32;
  const int index_tile_words = kTileChunks / 4;
  for (int c0 = 0; c0 < count; c0 += kGemvMaxGroup) {
    GemvGroup grp{};
    grp.count = (count - c0) < kGemvMaxGroup ? (count - c0) : kGemvMaxGroup;
    grp.batch = batch;
    int units = 0;
    for (int i = 0; i < grp.count; ++i) {
      GemvProblemDev p = probs[c0 + i];
      p.crow = packed_codes_row_bytes(p.d_in, N, M);
      p.irow = packed_index_row_bytes(p.d_in, M);
      grp.p[i] = p;
      grp.block_start[i] = units;
      units += (p.d_out + 15) / 16;
      if (!make_tmap_u32(&grp.tm_codes[i], p.packed, p.crow / 4, p.d_out, p.crow, code_tile_words, 16) ||
          !make_tmap_u32(&grp.tm_index[i], p.packed + static_cast<size_t>(p.d_out) * p.crow, p.irow / 4, p.d_out,
                         p.irow, index_tile_words, 16))
        return cudaErrorInvalidValue;
    }
    grp.block_start[grp.count] = units;
    if (units == 0) continue;
    cudaError_t e;
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
  return launch_gemv_group(&p, 1, batch, N, M, stream, num_sms, err);
}

}  // namespace sbl
