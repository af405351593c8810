// packed_decode.cuh -- decoding one chunk of the packed 2-bit ternary + N:M
// index format into int8 weights with byte permutes (prmt).
//
// "突破性发现：极低位量化与稀疏化的完美协同", 7.1 推理优化技巧 (bit operations
// on a pre-computed ternary format).  Format of a chunk (8 consecutive
// positions of a row; K = 8N/M slots s_0 < ... < s_(K-1), H = ceil(K/2)):
//   code field of 2K bits: code of s_q (q < H) at bits 4q..4q+1, code of
//   s_(H+q) at bits 4q+2..4q+3; codes +1 = 00, -1 = 01, 0 = 10;
//   slot mask: 8 bits, bit p set when position p is a slot.
//
// Decoding takes three byte permutes per 4 output weights' worth of work:
//   lo = prmt(C, C, sel_lo): nibble q of sel_lo is the code of s_q in bits
//        0-1 (bit 2 is don't-care, bit 3 cleared), so byte q of lo is
//        C[code] with C = {+1, -1, 0, -1};
//   hi = prmt(A, B, sel_hi): nibble q holds the code of s_(H+q) in bits 2-3
//        (bits 0-1 are don't-care because A and B repeat one byte).  Bit 2
//        (negative) picks B = 0xFF over A = 0x01, and bit 3 (zero) switches
//        prmt to sign replication, which turns A's 0x01 into 0x00;
//   out = prmt(lo, hi, scatter selector of the mask): slot i of the chunk
//        goes to its position, dropped positions take a byte known to be 0.
// Unused nibbles of sel_lo are forced to a zero code, so the field may be
// read with the next chunk's bits above it.  When H < 4 the forced byte 3 of
// lo is the zero the dropped positions take, and hi needs no masking at all
// (its unused bytes are never selected); only K = 7 (H = 4 with a dropped
// position) forces hi's byte 3 to zero and uses it instead.
#pragma once

#include <cstdint>

namespace sbl {

// prmt.b32 in its default mode, including the sign-replicate bit (bit 3 of
// each selector nibble), which __byte_perm does not document.
__device__ __forceinline__ uint32_t prmt(uint32_t x, uint32_t y, uint32_t s) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(x), "r"(y), "r"(s));
  return r;
}

template <int K>
struct ChunkCodes {
  static_assert(K >= 1 && K <= 8, "1 <= K <= 8 slots per chunk");
  static constexpr int H = (K + 1) / 2;  // slots decoded into `lo`
  static constexpr int NH = K - H;       // slots decoded into `hi`
  static constexpr uint32_t nib(int q, uint32_t v) { return v << (4 * q); }
  static constexpr uint32_t lo_keep() {
    uint32_t m = 0;
    for (int q = 0; q < H; ++q) m |= nib(q, 0x7u);
    return m;
  }
  static constexpr uint32_t lo_set() {  // unused nibbles -> index 2 (a zero byte of C)
    uint32_t m = 0;
    for (int q = H; q < 4; ++q) m |= nib(q, 0x2u);
    return m;
  }
  static constexpr uint32_t hi_keep() {  // unused nibbles keep only bits 0-1
    uint32_t m = 0xFFFF0000u;
    for (int q = 0; q < 4; ++q) m |= nib(q, q < NH ? 0xFu : 0x3u);
    return m;
  }
  static constexpr uint32_t hi_set() {  // unused nibbles -> sign of A (0x00)
    uint32_t m = 0;
    for (int q = NH; q < 4; ++q) m |= nib(q, 0x8u);
    return m;
  }
  static constexpr uint32_t kC = 0xFF00FF01u;  // byte per lo code: 00 +1, 01 -1, 10 0, 11 -1
  static constexpr uint32_t kA = 0x01010101u;
  static constexpr uint32_t kB = 0xFFFFFFFFu;

  static constexpr bool kHiRaw = H < 4 || K == 8;  // hi needs no masking

  // v: the chunk's code field in bits 0..2K-1 (bits above are ignored).
  __device__ __forceinline__ static void decode(uint32_t v, uint32_t& lo, uint32_t& hi) {
    lo = prmt(kC, kC, (v & lo_keep()) | lo_set());
    hi = kHiRaw ? prmt(kA, kB, v) : prmt(kA, kB, (v & hi_keep()) | hi_set());
  }
};

// Scatter selectors of a slot mask: word 0 for positions 0-3, word 1 for
// positions 4-7.  Slot of rank r goes from byte r of lo (r < H) or byte
// 4 + r - H of hi; other positions (and ranks >= K of a malformed mask)
// take the zero byte: byte 3 of lo when H < 4, else byte 7 of hi.
__host__ __device__ inline void scatter_selectors(uint32_t mask, int K, uint32_t& s0, uint32_t& s1) {
  const int H = (K + 1) / 2;
  const uint32_t zero_byte = H < 4 ? 3u : 7u;
  uint32_t s[2] = {0u, 0u};
  int r = 0;
  for (int p = 0; p < 8; ++p) {
    uint32_t nibv = zero_byte;
    if ((mask >> p) & 1u) {
      if (r < K) nibv = static_cast<uint32_t>(r < H ? r : 4 + r - H);
      ++r;
    }
    s[p >> 2] |= nibv << (4 * (p & 3));
  }
  s0 = s[0];
  s1 = s[1];
}

}  // namespace sbl
