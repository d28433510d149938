/*
 * df11_rans.h -- C ABI of the rANS variant of the exponent coding, a
 * comparison codec for the DF11 format of df11.h.
 *
 * Source: the page "DFloat11: Nén suy luận GPU không mất dữ liệu, giảm LLM
 * xuống còn 70% kích thước" (vi.news.hada.io/topic?id=20542).  Its Hacker
 * News discussion names rANS as a coder that suits SIMD hardware better than
 * Huffman codes; the page fixes no rANS format.  The coding step is range ANS
 * as defined by J. Duda ("Asymmetric numeral systems", 2013).  Everything
 * else below is this library's own reading, chosen for a warp of 32 lanes:
 *
 *   - Sign and mantissa stay verbatim in the sign/mantissa plane of df11.h;
 *     only the 8-bit exponents are rANS coded.
 *   - Probabilities: each exponent present with count c gets a frequency
 *     f >= 1 out of M = 4096 (largest-remainder apportionment of c*M/n, rare
 *     exponents raised to 1, ties to the smaller exponent; an excess is taken
 *     back one at a time from the most over-served exponent with f > 1).
 *     cum[s] = sum of f[t] for t < s.
 *   - State: 32-bit, kept in [2^16, 2^32); renormalisation moves 16-bit words.
 *     Decoding: slot = x mod M, s the exponent with cum[s] <= slot <
 *     cum[s] + f[s], x = f[s] * (x / M) + slot - cum[s]; if x < 2^16,
 *     x = (x << 16) | next word.
 *   - Interleaving: units of DF11_RANS_UNIT = 16384 values; value
 *     u*16384 + 32*k + l is the k-th symbol of state l of unit u.  Decoding
 *     runs steps k = 0..511 and, within a step, states l = 0..31, and reads
 *     the unit's words in that order.  The encoder starts every state at 2^16
 *     and runs the exact reverse; a decoded unit ends with every state back at
 *     2^16.  A unit's 512 steps form 8 segments of 64.
 *
 * Format (little-endian):
 *   stream         the units back to back, unit u at byte 16*off16[u]:
 *                    32 uint32  initial decoder states (final encoder states)
 *                     8 uint16  index of the first word read in each segment
 *                     W uint16  the words, in decoding order
 *                    zeros up to the next multiple of 16 bytes
 *                  (DF11_RANS_HEADER_BYTES = 144 bytes before the words)
 *   off16          uint32[U+1], U = ceil(n / 16384): unit starts in 16-byte
 *                  units; off16[U] * 16 = stream bytes.
 *   sign_mantissa  n bytes, as in df11.h.
 *   freq           256 frequencies (kept on the host; 512 bytes stored).
 *
 * Conventions are those of df11.h: d_* are device pointers, the caller owns
 * every buffer, device calls are asynchronous on the caller's stream and
 * return argument and launch errors only; data errors go to *d_status (first
 * error wins, the caller zeroes it).  Device pointers are 16-byte aligned.
 * n <= DF11_MAX_N.
 */
#ifndef DF11_RANS_H
#define DF11_RANS_H

#include "df11.h"

#ifdef __cplusplus
extern "C" {
#endif

#define DF11_RANS_PROB_BITS 12u       /* M = 4096                                */
#define DF11_RANS_LANES 32u           /* interleaved states per unit             */
#define DF11_RANS_STEPS 512u          /* symbols per state per unit              */
#define DF11_RANS_SEGMENTS 8u         /* word-start entries per unit header      */
#define DF11_RANS_UNIT 16384u         /* values per unit                         */
#define DF11_RANS_HEADER_BYTES 144u   /* 32 states + 8 segment starts            */
#define DF11_RANS_TABLES_BYTES 17408u /* device tables: 4096 + 256 uint32        */
#define DF11_RANS_MAX_BATCH 32u       /* matrices per decode launch (more = split) */

/*
 * df11_rans_freqs -- host.  Frequencies out of 4096 from a 256-bin exponent
 * histogram (df11_histogram), by the apportionment above.  One exponent
 * alone gets 4096; an empty histogram gives all zeros.
 */
df11_status df11_rans_freqs(const uint64_t hist256[256], uint32_t freq[256]);

/*
 * df11_rans_build_tables -- host.  The device tables of one frequency set,
 * written to h_tables (bytes >= DF11_RANS_TABLES_BYTES) for the caller to
 * copy to device memory:
 *   uint32 slot[4096]  decoding: exponent in bits 0..7, slot - cum in bits
 *                      8..19, f - 1 in bits 20..31
 *   uint32 enc[256]    encoding: f in bits 0..15 (0: exponent absent), cum
 *                      in bits 16..31
 * DF11_ERR_INVALID_ARG unless the frequencies sum to 4096 (or are all zero).
 */
df11_status df11_rans_build_tables(const uint32_t freq[256], void *h_tables, size_t bytes);

/* Units of a matrix of n values: ceil(n / DF11_RANS_UNIT). */
uint64_t df11_rans_units(uint64_t n);

/*
 * df11_rans_encode_sizes -- first encoding pass.  Runs every unit's encoder
 * without writing it, to count its words, and lays the units out.
 *   d_w            n BF16 words.
 *   d_tables       device copy of df11_rans_build_tables' output.
 *   d_unit_words   uint32[U] workspace: words of each unit (read by
 *                  df11_rans_encode).
 *   d_off16        uint32[U+1]: the off16 array of the format; the stream
 *                  needs d_off16[U] * 16 bytes.
 *   d_status       DF11_ERR_SYMBOL_NOT_IN_CODEBOOK if a value's exponent has
 *                  frequency 0.
 * Two kernel launches (count, prefix sum).  n == 0 writes d_off16[0] = 0.
 */
df11_status df11_rans_encode_sizes(const uint16_t *d_w, uint64_t n, const void *d_tables,
                                   uint32_t *d_unit_words, uint32_t *d_off16,
                                   uint32_t *d_status, df11_stream_t stream);

/*
 * df11_rans_encode -- second pass: writes the stream (every byte up to
 * d_off16[U] * 16, padding included) and the sign/mantissa plane (n bytes).
 * d_unit_words and d_off16 as left by df11_rans_encode_sizes; a unit whose
 * word count differs from them sets DF11_ERR_CORRUPT.  One kernel launch.
 */
df11_status df11_rans_encode(const uint16_t *d_w, uint64_t n, const void *d_tables,
                             const uint32_t *d_unit_words, const uint32_t *d_off16,
                             uint8_t *d_stream, uint8_t *d_sign_mantissa, uint32_t *d_status,
                             df11_stream_t stream);

/*
 * df11_rans_validate -- host.  Checks stored rANS metadata before it is
 * trusted, without decoding:
 *   - off16 has U + 1 entries, starts at 0, never decreases, and its last
 *     entry times 16 equals stream_bytes;
 *   - every unit holds its 144-byte header and at most one word per value
 *     (plus padding below 16 bytes);
 *   - each unit's segment word starts begin at 0, never decrease, and stay
 *     within the unit's words;
 *   - every initial state is at least 2^16 (the encoder never ends below),
 *     and a state that codes no value (lanes past n in the last unit) is
 *     exactly 2^16.
 *   h_stream  the stream (host copy), stream_bytes bytes.
 *   h_off16   off16_count entries (host copy).
 * DF11_ERR_INVALID_ARG for null pointers or a wrong off16_count,
 * DF11_ERR_TOO_LARGE for n > DF11_MAX_N, DF11_ERR_CORRUPT otherwise.
 * What only a decode can check (every word read, states back at 2^16) is
 * left to df11_rans_decode_batch.
 */
df11_status df11_rans_validate(uint64_t n, const uint8_t *h_stream, uint64_t stream_bytes,
                               const uint32_t *h_off16, uint64_t off16_count);

/* One rANS-coded matrix (host struct of device pointers). */
typedef struct {
  uint64_t n;
  const uint8_t *stream;         /* d_off16[U] * 16 bytes                   */
  const uint32_t *off16;         /* U + 1 entries                           */
  const uint8_t *sign_mantissa;  /* n bytes                                 */
  const void *tables;            /* DF11_RANS_TABLES_BYTES                  */
} df11_rans_matrix;

/*
 * df11_rans_decode_batch -- decode count matrices into BF16 (d_outs[i]: n
 * uint16, written in full), one launch per DF11_RANS_MAX_BATCH matrices.
 * Each warp decodes one unit at a time with its 32 states in lockstep.
 *   d_status  DF11_ERR_CORRUPT if a unit's layout, segment starts, final
 *             states or word count disagree with the decoding (that unit's
 *             output is then unspecified; nothing outside d_outs is written).
 */
df11_status df11_rans_decode_batch(const df11_rans_matrix *ms, uint32_t count,
                                   uint16_t *const *d_outs, uint32_t *d_status,
                                   df11_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* DF11_RANS_H */
