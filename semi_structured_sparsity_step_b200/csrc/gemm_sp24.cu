// gemm_sp24.cu -- (a8) the forward product of a 2:4 Sparse-BitLinear layer on
// the sparse int8 tensor core of sm_100a (tcgen05.mma.sp, kind::i8).
//
// Sparse-BitNet summary ("Sparse-BitNet：1.58-bit 大模型天然兼容半结构化稀疏"),
// 前置知识 / 半结构化 N:M 稀疏: 2:4 (two kept in every four) is the pattern the
// sparse tensor cores accelerate; 核心方法: the mask is applied after
// quantisation, so the deployed ternary weight already has that structure.
// The product is the one of Algorithm 1 step (6), bit for bit the same as the
// dense forward: acc[t,o] = sum_j Xq[t,j] W_eff[o,j] (int32), then
// Y = fp32(acc) * fp32(gamma * fp32(amax_t / 127)).
//
// Compressed weight (sbl_compress24 writes it from W_eff):
//   values plane    [d_out, vrow] int8, vrow = ceil16(d_in / 2): for every
//                   group of four weights its two slot values, ascending;
//   selector plane  from the first 1024-byte boundary after the values: the
//                   4-bit selector i0 | i1 << 2 of every group, tiled in
//                   blocks of 128 rows x 256 weights (4096 bytes, block
//                   (mb, kb) at (mb * KB + kb) * 4096), each block two halves
//                   of 128 rows x 16 bytes (128 weights per row), row r of a
//                   half at 16 r, low nibble = even group.  Rows are padded
//                   to 256 and weights to 256 with the selector of slots
//                   (0, 1) and zero values.
// Slots are a group's nonzero positions plus its lowest zero positions.
//
// Kernel: CTA pairs (cluster of 2, cta_group::2).  The sparse operand must be
// A, so the pair computes a transposed tile D[o, t] = sum_k W[o,k] Xq[t,k]
// of 256 weight rows x 224 tokens; CTA r stages weight rows [128 r, 128 r +
// 128) and token rows [112 r, 112 r + 112) of the tile.  Per stage (256
// weights of K): A = 128 rows x 128 bytes of kept values (128-byte swizzle),
// B = 112 rows x 256 bytes as two 128-byte swizzled column tiles, and the
// 4096-byte selector block, all by TMA.  The MMA thread of the even CTA
// copies the selectors into TMEM (tcgen05.cp, 128 lanes x 4 columns per
// half, into the 8 selector columns of that ring stage; each instruction
// covers 64 weights = 2 columns) and issues four
// M = 256, N = 224, K = 64 sparse MMAs.  Two 224-column accumulators in TMEM
// let the epilogue of one tile overlap the next.  The epilogue reads each
// 32 x 32 chunk with one weight row per lane and turns it around in a padded
// shared tile, so that every 16-byte store of a warp lands in one of four
// whole 128-byte segments of Y rows (the epilogue, not the tensor core, is
// what bounds this kernel: the MMA thread waited half its time for a free
// accumulator with one 4-byte store per lane and token).
#include <cuda.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "sbl_device.cuh"
#include "sbl_internal.h"

namespace sbl {
namespace {

constexpr int kSpBN = 224;                  // tokens per pair tile (MMA N)
constexpr int kSpHalfN = kSpBN / 2;         // token rows staged per CTA
constexpr int kSpBK = 256;                  // weights of K per stage
constexpr int kSpStages = 4;
constexpr int kSpABytes = 128 * 128;        // kept values: 128 rows x 128 bytes
constexpr int kSpBTile = kSpHalfN * 128;    // one 128-byte column tile of B
constexpr int kSpBBytes = 2 * kSpBTile;
constexpr int kSpEBytes = 4096;             // selector block
constexpr int kSpStageBytes = kSpABytes + kSpBBytes + kSpEBytes;
constexpr int kSpEpiStride = 36;            // floats per row of an epilogue warp's 32 x 32 transpose tile
constexpr int kSpEpiBytes = 4 * 32 * kSpEpiStride * 4;
constexpr int kSpSmem = kSpStages * kSpStageBytes + 256 + kSpEpiBytes + 1024;
constexpr int kSpThreads = 192;
constexpr uint32_t kSpTmemCols = 512;
constexpr uint32_t kSpECol = 2 * kSpBN;     // selector columns after the two accumulators, 8 per ring stage
constexpr uint32_t kSpIdesc = instr_desc(true, 256, kSpBN, false, false) | (1u << 2);  // bit 2: sparse A

static_assert(kSpStageBytes % 1024 == 0, "stage bases stay 1024-byte aligned");
static_assert((kSpABytes + kSpBTile) % 1024 == 0, "second B tile is 1024-byte aligned");
static_assert(kSpECol + 8 * kSpStages <= kSpTmemCols, "every stage's selectors fit after the accumulators");

struct Sp24Args {
  int T, d_in, d_out;
  int KB;            // stages per tile
  int Mt, total;     // weight-row pair tiles, work items
  float* Y;
  int32_t* acc;
  const float* amax;
  const float* gamma;
  uint32_t* err;
};

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kSpThreads, 1)
    sp24_forward_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                        const __grid_constant__ CUtensorMap tmE, const Sp24Args args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kSpStages * kSpStageBytes);
  uint64_t* empty = full + kSpStages;
  uint64_t* tfull = empty + kSpStages;
  uint64_t* tempty = tfull + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tempty + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  uint32_t* epi_tiles = reinterpret_cast<uint32_t*>(smem + kSpStages * kSpStageBytes + 256);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = pair::cluster_rank();
  const bool leader = rank == 0;
  const int pair_id = blockIdx.x >> 1;
  const int n_pairs = gridDim.x >> 1;
  const int KB = args.KB;
  const uint32_t peer_abort = pair::map_to(smem_u32(const_cast<int*>(abort_flag)), rank ^ 1u);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kSpStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 8);
    }
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    tma_prefetch_desc(&tmE);
  }
  if (warp == 1) {
    pair::tmem_alloc(tmem_slot, kSpTmemCols);
    pair::tmem_relinquish();
  }
  tc_fence_before();
  pair::cluster_sync();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  auto give_up = [&]() {
    *abort_flag = 1;
    pair::store_remote_u32(peer_abort, 1u);
  };

  // Work item w: weight-row tile mb = w % Mt (fastest), token tile nb = w / Mt,
  // so the pairs running together share token tiles and Xq streams once.
  if (warp == 0) {
    if (lane == 0) {
      int it = 0;
      bool ok = true;
      for (int w = pair_id; w < args.total && ok; w += n_pairs) {
        const int mb = w % args.Mt, nb = w / args.Mt;
        const int m0 = mb * 256 + 128 * static_cast<int>(rank);   // weight row
        const int n0 = nb * kSpBN + kSpHalfN * static_cast<int>(rank);  // token row
        const int eblk = (2 * mb + static_cast<int>(rank)) * KB;  // selector block of (m0 / 128, 0)
        for (int kb = 0; kb < KB; ++kb) {
          const int s = it % kSpStages;
          const uint32_t round = static_cast<uint32_t>(it / kSpStages);
          if (!mbar_wait(&empty[s], (round & 1u) ^ 1u, abort_flag, args.err)) {
            give_up();
            ok = false;
            break;
          }
          if (leader) mbar_arrive_expect_tx(&full[s], 2 * kSpStageBytes);
          const uint32_t fbar = pair::map_to(smem_u32(&full[s]), 0u);
          uint8_t* sa = smem + s * kSpStageBytes;
          uint8_t* sb = sa + kSpABytes;
          uint8_t* se = sb + kSpBBytes;
          pair::tma_load_2d(sa, &tmA, fbar, kb * (kSpBK / 2), m0);
          pair::tma_load_2d(sb, &tmB, fbar, kb * kSpBK, n0);
          pair::tma_load_2d(sb + kSpBTile, &tmB, fbar, kb * kSpBK + 128, n0);
          pair::tma_load_2d(se, &tmE, fbar, 0, (eblk + kb) * 32);
          ++it;
        }
      }
      if (!ok && leader) {
        for (int i = (it > kSpStages ? it - kSpStages : 0); i < it; ++i)
          mbar_wait(&full[i % kSpStages], static_cast<uint32_t>(i / kSpStages) & 1u, nullptr, args.err);
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      int it = 0, t = 0;
      bool ok = true;
      for (int w = pair_id; w < args.total && ok; w += n_pairs, ++t) {
        const int b = t & 1;
        if (!mbar_wait(&tempty[b], (static_cast<uint32_t>(t >> 1) & 1u) ^ 1u, abort_flag, args.err)) {
          give_up();
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(b * kSpBN);
        for (int kb = 0; kb < KB; ++kb) {
          const int s = it % kSpStages;
          const uint32_t round = static_cast<uint32_t>(it / kSpStages);
          if (!mbar_wait(&full[s], round & 1u, abort_flag, args.err)) {
            give_up();
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + s * kSpStageBytes);
          const uint32_t sb = sa + kSpABytes;
          const uint32_t se = sb + kSpBBytes;
          // each ring stage has its own selector columns, so copying the next
          // stage's selectors never waits for this stage's products to read theirs
          const uint32_t e_tmem = tmem_base + kSpECol + 8u * static_cast<uint32_t>(s);
          pair::tmem_cp_128x128b(e_tmem, smem_desc_rows16(se, 128));
          pair::tmem_cp_128x128b(e_tmem + 4, smem_desc_rows16(se + 2048, 128));
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t adesc = smem_desc_sw128(sa + kk * 32, 16, 1024);
            const uint64_t bdesc = smem_desc_sw128(sb + (kk >> 1) * kSpBTile + (kk & 1) * 64, 16, 1024);
            pair::umma_sp_i8(d_tmem, adesc, bdesc, kSpIdesc, e_tmem + 2 * kk, (kb > 0 || kk > 0) ? 1u : 0u);
          }
          pair::umma_commit_multicast(&empty[s], 0x3);
          ++it;
        }
        pair::umma_commit_multicast(&tfull[b], 0x3);
      }
    }
  } else {
    const int q = warp & 3;  // TMEM lane quarter this warp may read
    const float g = *args.gamma;
    int t = 0;
    for (int w = pair_id; w < args.total; w += n_pairs, ++t) {
      const int mb = w % args.Mt, nb = w / args.Mt;
      const int b = t & 1;
      // the tile's token scales, loaded while its MMAs still run: lane l holds
      // the scale of token nb * kSpBN + 32 c + l in scl[c]
      float scl[kSpBN / 32];
#pragma unroll
      for (int c = 0; c < kSpBN / 32; ++c) {
        const int tl = nb * kSpBN + 32 * c + lane;
        scl[c] = tl < args.T ? __ldg(args.amax + tl) : 0.0f;
      }
#pragma unroll
      for (int c = 0; c < kSpBN / 32; ++c) scl[c] = __fmul_rn(g, __fdiv_rn(scl[c], 127.0f));
      if (!mbar_wait(&tfull[b], static_cast<uint32_t>(t >> 1) & 1u, abort_flag, args.err)) {
        give_up();
        break;
      }
      tc_fence_after();
      if (*abort_flag) break;
      // Each 32 x 32 chunk (lane = weight row, register j = token) goes through
      // a padded shared tile so that the stores run along Y's rows: lane l then
      // holds rows o0 + 4 (l % 8) .. + 3 of token 4 it + l / 8, one 16-byte
      // store per lane and four whole 128-byte row segments per instruction.
      const int o0 = mb * 256 + 128 * static_cast<int>(rank) + 32 * q;  // the warp's first weight row
      const uint32_t tbase = tmem_base + (static_cast<uint32_t>(32 * q) << 16) + static_cast<uint32_t>(b * kSpBN);
      uint32_t* et = epi_tiles + (warp - 2) * (32 * kSpEpiStride);
      const int c4 = 4 * (lane & 7), tr = lane >> 3;
      const bool cols_ok = o0 + c4 < args.d_out;  // d_out % 8 == 0: four rows are all in or all out
#pragma unroll
      for (int c = 0; c < kSpBN / 32; ++c) {
        const int t0 = nb * kSpBN + 32 * c;
        if (t0 >= args.T) break;  // warp-uniform
        uint32_t r[32];
        tmem_ld_32x32b_x32(tbase + static_cast<uint32_t>(32 * c), r);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 32; ++j) et[j * kSpEpiStride + lane] = r[j];
        __syncwarp();
        const float sl = scl[c];
#pragma unroll
        for (int it = 0; it < 8; ++it) {
          const int tl = 4 * it + tr;  // token within the chunk
          const float sc = __shfl_sync(0xFFFFFFFFu, sl, tl);
          const uint4 v = *reinterpret_cast<const uint4*>(et + tl * kSpEpiStride + c4);
          if (cols_ok && t0 + tl < args.T) {
            const long long off = static_cast<long long>(t0 + tl) * args.d_out + o0 + c4;
            *reinterpret_cast<float4*>(args.Y + off) =
                make_float4(__fmul_rn(__int2float_rn(static_cast<int>(v.x)), sc),
                            __fmul_rn(__int2float_rn(static_cast<int>(v.y)), sc),
                            __fmul_rn(__int2float_rn(static_cast<int>(v.z)), sc),
                            __fmul_rn(__int2float_rn(static_cast<int>(v.w)), sc));
            if (args.acc != nullptr) *reinterpret_cast<uint4*>(args.acc + off) = v;
          }
        }
        __syncwarp();
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
    pair::tmem_dealloc(tmem_base, kSpTmemCols);
  }
}

// One thread per 16 weights of one row (rows padded to the selector plane's
// 256, weights to its 256): picks the two slots of each group of four, writes
// their values (8 bytes) and the four selectors (2 bytes).  A group with more
// than two nonzeros latches kErrDeviceCheck (its first two nonzeros are kept).
// Block 0 also zeroes the gap (< 1024 bytes) between the two planes.
__global__ void compress24_kernel(const int8_t* __restrict__ W, int d_out, int d_in, uint8_t* __restrict__ vals,
                                  long long vrow, uint8_t* __restrict__ meta, int KB, long long rows_padded,
                                  uint32_t* err) {
  if (blockIdx.x == 0) {
    uint8_t* gap = vals + static_cast<long long>(d_out) * vrow;
    const int gap_bytes = static_cast<int>(meta - gap);
    for (int i = threadIdx.x; i < gap_bytes; i += blockDim.x) gap[i] = 0;
  }
  const long long chunks_per_row = static_cast<long long>(KB) * 16;
  const long long total = rows_padded * chunks_per_row;
  for (long long idx = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; idx < total;
       idx += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int R = static_cast<int>(idx / chunks_per_row);
    const int c = static_cast<int>(idx - static_cast<long long>(R) * chunks_per_row);
    const int k0 = 16 * c;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (R < d_out && k0 < d_in) v = __ldg(reinterpret_cast<const uint4*>(W + static_cast<long long>(R) * d_in + k0));
    const uint32_t words[4] = {v.x, v.y, v.z, v.w};
    uint32_t out[2] = {0u, 0u};
    uint32_t sel = 0u;
    bool bad = false;
#pragma unroll
    for (int gi = 0; gi < 4; ++gi) {
      const uint32_t wd = words[gi];
      uint32_t nz = 0u;
#pragma unroll
      for (int p = 0; p < 4; ++p) nz |= (((wd >> (8 * p)) & 0xFFu) != 0u ? 1u : 0u) << p;
      bad |= __popc(nz) > 2;
      // nonzero positions first, then zero positions, lowest index first
      uint32_t pick = 0u;
      int n = 0;
#pragma unroll
      for (int p = 0; p < 4; ++p)
        if (((nz >> p) & 1u) && n < 2) {
          pick |= 1u << p;
          ++n;
        }
#pragma unroll
      for (int p = 0; p < 4; ++p)
        if (!((nz >> p) & 1u) && n < 2) {
          pick |= 1u << p;
          ++n;
        }
      const uint32_t i0 = static_cast<uint32_t>(__ffs(static_cast<int>(pick)) - 1);
      const uint32_t i1 = 31u - static_cast<uint32_t>(__clz(static_cast<int>(pick)));
      const uint32_t v0 = (wd >> (8 * i0)) & 0xFFu, v1 = (wd >> (8 * i1)) & 0xFFu;
      out[gi >> 1] |= (v0 | (v1 << 8)) << (16 * (gi & 1));
      sel |= (i0 | (i1 << 2)) << (4 * gi);
    }
    if (bad) latch_error(err, kErrDeviceCheck);
    if (R < d_out && 8LL * c < vrow)
      *reinterpret_cast<uint2*>(vals + static_cast<long long>(R) * vrow + 8 * c) = make_uint2(out[0], out[1]);
    const int mb = R >> 7, r = R & 127;
    const int kb = c >> 4, half = (c >> 3) & 1;
    const long long off = ((static_cast<long long>(mb) * KB + kb) * 2 + half) * 2048 + r * 16 + 2 * (c & 7);
    *reinterpret_cast<uint16_t*>(meta + off) = static_cast<uint16_t>(sel);
  }
}

}  // namespace

size_t sparse24_values_row_bytes(int d_in) { return (static_cast<size_t>(d_in) / 2 + 15) / 16 * 16; }

size_t sparse24_meta_offset(int d_out, int d_in) {
  return (static_cast<size_t>(d_out) * sparse24_values_row_bytes(d_in) + 1023) / 1024 * 1024;
}

static size_t sparse24_kb(int d_in) { return (static_cast<size_t>(d_in) + kSpBK - 1) / kSpBK; }
static size_t sparse24_row_blocks(int d_out) { return 2 * ((static_cast<size_t>(d_out) + 255) / 256); }

size_t sparse24_bytes(int d_out, int d_in) {
  return sparse24_meta_offset(d_out, d_in) + sparse24_row_blocks(d_out) * sparse24_kb(d_in) * kSpEBytes;
}

cudaError_t launch_compress24(const int8_t* W_eff, int d_out, int d_in, uint8_t* out, cudaStream_t stream,
                              int num_sms, uint32_t* err) {
  if (d_out == 0) return cudaSuccess;
  const int KB = static_cast<int>(sparse24_kb(d_in));
  if (KB == 0) return cudaSuccess;
  const long long rows_padded = static_cast<long long>(sparse24_row_blocks(d_out)) * 128;
  const long long total = rows_padded * KB * 16;
  long long blocks = (total + 255) / 256;
  const long long cap = static_cast<long long>(num_sms) * 16;
  if (blocks > cap) blocks = cap;
  compress24_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
      W_eff, d_out, d_in, out, static_cast<long long>(sparse24_values_row_bytes(d_in)),
      out + sparse24_meta_offset(d_out, d_in), KB, rows_padded, err);
  return cudaGetLastError();
}

cudaError_t launch_forward_sparse24(const int8_t* Xq, const float* amax, const uint8_t* w24, const float* gamma,
                                   int T, int d_in, int d_out, float* Y, int32_t* acc, cudaStream_t stream,
                                   int num_sms, uint32_t* err) {
  if (T == 0 || d_out == 0) return cudaSuccess;
  if (d_in == 0) {
    cudaError_t e = cudaMemsetAsync(Y, 0, sizeof(float) * static_cast<size_t>(T) * d_out, stream);
    if (e == cudaSuccess && acc != nullptr)
      e = cudaMemsetAsync(acc, 0, sizeof(int32_t) * static_cast<size_t>(T) * d_out, stream);
    return e;
  }
  const int KB = static_cast<int>(sparse24_kb(d_in));
  const size_t vrow = sparse24_values_row_bytes(d_in);
  const uint8_t* meta = w24 + sparse24_meta_offset(d_out, d_in);
  const unsigned long long e_rows = static_cast<unsigned long long>(sparse24_row_blocks(d_out)) * KB * 32;
  CUtensorMap ta, tb, te;
  if (!make_tmap_u8(&ta, w24, static_cast<unsigned long long>(d_in) / 2, d_out, vrow, 128, 128, true) ||
      !make_tmap_u8(&tb, Xq, d_in, T, d_in, 128, kSpHalfN, true) ||
      !make_tmap_u8(&te, meta, 128, e_rows, 128, 128, 32, false))
    return cudaErrorInvalidValue;
  Sp24Args a{};
  a.T = T;
  a.d_in = d_in;
  a.d_out = d_out;
  a.KB = KB;
  a.Mt = (d_out + 255) / 256;
  const int Nt = (T + kSpBN - 1) / kSpBN;
  a.total = a.Mt * Nt;
  a.Y = Y;
  a.acc = acc;
  a.amax = amax;
  a.gamma = gamma;
  a.err = err;
  cudaError_t e = cudaFuncSetAttribute(sp24_forward_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSpSmem);
  if (e != cudaSuccess) return e;
  int pairs = num_sms / 2;
  if (pairs > a.total) pairs = a.total;
  sp24_forward_kernel<<<2 * pairs, kSpThreads, kSpSmem, stream>>>(ta, tb, te, a);
  return cudaGetLastError();
}

}  // namespace sbl
