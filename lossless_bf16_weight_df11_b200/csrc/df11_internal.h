// df11_internal.h -- layouts shared by the host code and the kernels of the
// DF11 library (not part of the public ABI).
#pragma once

#include <stdint.h>

namespace df11i {

// Decode tables of one codebook, built on the host by df11_build_tables and
// copied to shared memory by every decoding CTA.
//
// lut: indexed by the next kLutBits stream bits.  Each entry describes the
// whole codes (at most three) that fit in those bits, decoded greedily:
//   bits  0..23  the decoded exponent values, first code in bits 0..7,
//                zero beyond the last code
//   bits 24..25  number of codes (1..3)
//   bit  26      set when the first code is longer than kLutBits bits (or
//                invalid); then the count is zero, bits 28..31 hold kLutBits,
//                and the code must be decoded by the length search below
//   bits 28..31  bits consumed by those codes (1..kLutBits)
// (The fields sit where the decoder can read them with a multiply-high:
// bits consumed = e >> 28, count = (e & 0x03000000) >> 24.)
// limit/base/sym: canonical decoding of a long code from a 32-bit
// left-justified window: its length L is the smallest with
// window < limit[L], its value sym[(window >> (32-L)) + base[L]].
constexpr int kLutBits = 12;
constexpr int kLutSize = 1 << kLutBits;

struct alignas(16) DecodeTables {
  uint32_t lut[kLutSize];
  uint64_t limit[33];
  uint32_t base[33];
  uint8_t codelen[256];
  uint8_t sym[256];
  uint32_t max_len;
  uint32_t min_len;
  uint32_t n_symbols;
  uint32_t lut_bits;
};

static_assert(sizeof(DecodeTables) % 16 == 0, "tables are copied in 16-byte units");

constexpr uint32_t kLutLongFlag = 1u << 26;
constexpr uint32_t kLutCountMask = 3u << 24;
#ifdef __CUDACC__
#define DF11I_HD __host__ __device__
#else
#define DF11I_HD
#endif
DF11I_HD inline constexpr uint32_t lut_entry(uint32_t syms, uint32_t count, uint32_t used) {
  return syms | (count << 24) | (used << 28);
}

// Encoder tile: 256 threads x 16 values.
constexpr int kEncThreads = 256;
constexpr int kEncPerThread = 16;
constexpr int kEncTile = kEncThreads * kEncPerThread;

}  // namespace df11i
