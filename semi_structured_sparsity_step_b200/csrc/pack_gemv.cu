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
// Decode GEMV: one warp per output row; lane l takes a contiguous run of
// chunks, reads its code bits through a 64-bit bit reader (aligned 32-bit
// loads) and its index bytes, and expands each chunk to 8 int8 weights with
// two shared-memory tables: codes (4 codes per byte) -> 4 int8 values, and
// slot mask -> __byte_perm selectors that move value i to the position of the
// i-th slot and a zero byte elsewhere.  Products are __dp4a over the int8
// activations of up to 16 tokens; the warp reduces and lane 0 applies
// y = fp32(acc) * fp32(gamma * fp32(amax_b / 127)).
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
struct BitReader {
  const uint32_t* words;
  uint64_t buf;
  int avail;
  int wi;
  __device__ __forceinline__ BitReader(const uint8_t* plane16, size_t bit0) {
    words = reinterpret_cast<const uint32_t*>(plane16);
    wi = static_cast<int>(bit0 >> 5);
    const int sh = static_cast<int>(bit0 & 31);
    buf = __ldg(words + wi) >> sh;
    avail = 32 - sh;
    ++wi;
  }
  __device__ __forceinline__ uint32_t get(int nbits) {  // nbits <= 32
    if (avail < nbits) {
      buf |= static_cast<uint64_t>(__ldg(words + wi)) << avail;
      ++wi;
      avail += 32;
    }
    const uint32_t v = static_cast<uint32_t>(buf) & ((nbits == 32) ? 0xFFFFFFFFu : ((1u << nbits) - 1u));
    buf >>= nbits;
    avail -= nbits;
    return v;
  }
};

template <int BMAX>
__global__ void __launch_bounds__(256) gemv_packed_kernel(const int8_t* __restrict__ Xq, const float* __restrict__ amax,
                                                          int batch, const uint8_t* __restrict__ packed,
                                                          const float* __restrict__ gamma, int d_in, int d_out,
                                                          int kslots, size_t crow, size_t irow,
                                                          float* __restrict__ Y) {
  __shared__ uint32_t s_val[256];  // 4 codes -> 4 int8
  __shared__ uint32_t s_sel[256];  // slot mask -> two byte_perm selectors
  {
    const uint32_t c = threadIdx.x;
    uint32_t v = 0;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const uint32_t code = (c >> (2 * k)) & 3u;
      const uint32_t byte = code == 1u ? 0x01u : (code == 3u ? 0xFFu : 0u);
      v |= byte << (8 * k);
    }
    s_val[c] = v;
    uint32_t sel = 0;
#pragma unroll
    for (int p = 0; p < 8; ++p) {
      const uint32_t nib = ((c >> p) & 1u) ? static_cast<uint32_t>(__popc(c & ((1u << p) - 1u))) : 7u;
      sel |= nib << (4 * p);
    }
    s_sel[c] = sel;
  }
  __syncthreads();

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int row = blockIdx.x * 8 + warp;
  if (row >= d_out) return;
  const int nchunks = d_in / 8;
  const int per = (nchunks + 31) / 32;
  const int ch0 = lane * per;
  const int ch1 = min(nchunks, ch0 + per);
  const int cbits = 2 * kslots;

  int acc[BMAX];
#pragma unroll
  for (int b = 0; b < BMAX; ++b) acc[b] = 0;

  if (ch0 < ch1) {
    const uint8_t* codes = packed + static_cast<size_t>(row) * crow;
    const uint8_t* index = packed + static_cast<size_t>(d_out) * crow + static_cast<size_t>(row) * irow;
    BitReader cr(codes, static_cast<size_t>(ch0) * cbits);
    for (int ch = ch0; ch < ch1; ++ch) {
      const uint32_t c = cr.get(cbits);
      const uint32_t m = __ldg(index + ch);
      const uint32_t w0 = s_val[c & 0xFFu];
      const uint32_t w1 = s_val[(c >> 8) & 0xFFu];
      const uint32_t sel = s_sel[m];
      const int lo = static_cast<int>(__byte_perm(w0, w1, sel & 0xFFFFu));
      const int hi = static_cast<int>(__byte_perm(w0, w1, sel >> 16));
#pragma unroll
      for (int b = 0; b < BMAX; ++b) {
        if (b < batch) {
          const uint2 x = __ldg(reinterpret_cast<const uint2*>(Xq + static_cast<size_t>(b) * d_in + 8 * ch));
          acc[b] = __dp4a(lo, static_cast<int>(x.x), acc[b]);
          acc[b] = __dp4a(hi, static_cast<int>(x.y), acc[b]);
        }
      }
    }
  }
#pragma unroll
  for (int b = 0; b < BMAX; ++b) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc[b] += __shfl_xor_sync(0xFFFFFFFFu, acc[b], o);
  }
  if (lane == 0) {
    const float g = *gamma;
#pragma unroll
    for (int b = 0; b < BMAX; ++b) {
      if (b < batch) {
        const float sc = __fmul_rn(g, __fdiv_rn(amax[b], 127.0f));
        Y[static_cast<size_t>(b) * d_out + row] = __fmul_rn(__int2float_rn(acc[b]), sc);
      }
    }
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

cudaError_t launch_gemv_packed(const int8_t* Xq, const float* amax, int batch, const uint8_t* packed,
                               const float* gamma, int d_in, int d_out, int N, int M, float* Y,
                               cudaStream_t stream, int num_sms) {
  (void)num_sms;
  if (batch == 0 || d_out == 0) return cudaSuccess;
  const size_t crow = packed_codes_row_bytes(d_in, N, M);
  const size_t irow = packed_index_row_bytes(d_in, M);
  const int kslots = 8 * N / M;
  const unsigned blocks = static_cast<unsigned>((d_out + 7) / 8);
#define SBL_GEMV_CASE(BM_)                                                                                   \
  gemv_packed_kernel<BM_><<<blocks, 256, 0, stream>>>(Xq, amax, batch, packed, gamma, d_in, d_out, kslots, crow, \
                                                      irow, Y)
  if (batch <= 1) SBL_GEMV_CASE(1);
  else if (batch <= 2) SBL_GEMV_CASE(2);
  else if (batch <= 4) SBL_GEMV_CASE(4);
  else if (batch <= 8) SBL_GEMV_CASE(8);
  else SBL_GEMV_CASE(16);
#undef SBL_GEMV_CASE
  return cudaGetLastError();
}

}  // namespace sbl
