// df11_internal.h -- layouts shared by the host code and the kernels of the
// DF11 library (not part of the public ABI).
#pragma once

#include <stdint.h>

namespace df11i {

// Decode tables of one codebook, built on the host by df11_build_tables (or on
// the device by the codebook kernel) and copied to shared memory by every
// decoding CTA.
//
// lut: indexed by the next kLutBits stream bits.  Each entry describes the
// whole codes (at most four) that fit in those bits, decoded greedily:
//   .x  the decoded exponents, first code in bits 0..7, zero beyond the last
//       code.  Each exponent byte is stored rotated right by one bit
//       (ror8(e) = e >> 1 | (e & 1) << 7): the byte then holds the BF16
//       word's high-byte exponent bits in bits 0..6 and its low-byte
//       exponent bit in bit 7, so merging with the sign/mantissa byte takes
//       one bit-select per output byte.
//   .y  control word:
//       bits  3..5   number of codes (1..4), so bits 0..10 equal 8 * count
//                    (the decoder adds the whole word to its byte position;
//                    bits 0..2 and 6..10 are zero)
//       bits 12..15  start of the second code, relative to the window (15
//                    when absent); bits 16..19 the third; bits 20..23 the
//                    fourth
//       bit  26      set when the first code is longer than kLutBits bits
//                    (or invalid): no codes, and the code is decoded by the
//                    length search below
//       bits 28..31  bits consumed by the codes (1..kLutBits; kLutBits when
//                    flagged)
// limit/base/sym: canonical decoding of a long code from a 32-bit
// left-justified window: its length L is the smallest with window <
// limit[L], its exponent sym[(window >> (32-L)) + base[L]] (rotated as above).
// codelen: code length of each exponent value (not rotated).
constexpr int kLutBits = 11;
constexpr int kLutSize = 1 << kLutBits;

struct alignas(8) LutEntry {
  uint32_t x;  // exponents
  uint32_t y;  // control
};

struct alignas(16) DecodeTables {
  LutEntry lut[kLutSize];
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

constexpr uint32_t kLutMaxCodes = 4;
constexpr uint32_t kCtrlCountShift = 3;
constexpr uint32_t kCtrlStartShift = 12;      // second code; +4 per further code
constexpr uint32_t kCtrlNoStart = 15u;        // start field of an absent code
constexpr uint32_t kCtrlLongFlag = 1u << 26;
constexpr uint32_t kCtrlUsedShift = 28;
// bits that are zero in every valid control word: 0..2, 6..11, 24, 25, 27
constexpr uint32_t kCtrlReserved = 0x0B000FC7u;
static_assert((kCtrlReserved & ((7u << kCtrlCountShift) | (0xFFFu << kCtrlStartShift) |
                                kCtrlLongFlag | (15u << kCtrlUsedShift))) == 0,
              "reserved bits are disjoint from the fields");

#ifdef __CUDACC__
#define DF11I_HD __host__ __device__
#else
#define DF11I_HD
#endif

DF11I_HD inline constexpr uint32_t ror8(uint32_t e) { return ((e >> 1) | (e << 7)) & 0xFFu; }

// Control word of an entry with `count` codes starting at offsets starts[1..]
// (starts[0] = 0) and consuming `used` bits.
DF11I_HD inline constexpr uint32_t lut_ctrl(uint32_t count, uint32_t s2, uint32_t s3, uint32_t s4,
                                            uint32_t used) {
  return (count << kCtrlCountShift) | (s2 << kCtrlStartShift) | (s3 << (kCtrlStartShift + 4)) |
         (s4 << (kCtrlStartShift + 8)) | (used << kCtrlUsedShift);
}

// Encoder tile: 256 threads x 16 values.
constexpr int kEncThreads = 256;
constexpr int kEncPerThread = 16;
constexpr int kEncTile = kEncThreads * kEncPerThread;

}  // namespace df11i
