// df11_host.cpp -- host half of the DF11 library: codebook construction,
// buffer sizing, decode-table construction and metadata validation.
//
// Method: "DFloat11: Nén suy luận GPU không mất dữ liệu, giảm LLM xuống còn 70%
// kích thước" (vi.news.hada.io/topic?id=20542), sections "Định dạng DFloat11"
// (Huffman code of the exponents), "Giải mã dựa trên LUT phân cấp" (table
// decoding, code lengths up to 32) and "Kernel GPU hai giai đoạn và metadata
// bổ trợ" (chunks, gaps, block positions).
//
// The codebook and table construction themselves live in df11_codebook.h,
// shared with the device's codebook kernel.
#include <algorithm>
#include <cstring>
#include <memory>

#include "df11.h"
#include "df11_codebook.h"
#include "df11_internal.h"

using df11i::DecodeTables;

extern "C" const char *df11_status_string(df11_status s) {
  switch (s) {
    case DF11_OK: return "ok";
    case DF11_ERR_INVALID_ARG: return "invalid argument";
    case DF11_ERR_TOO_LARGE: return "matrix larger than 2^32-1 values";
    case DF11_ERR_CUDA: return "CUDA error";
    case DF11_ERR_CORRUPT: return "corrupt stream or metadata";
    case DF11_ERR_SYMBOL_NOT_IN_CODEBOOK: return "value without a code in the codebook";
    case DF11_ERR_TIMEOUT: return "bounded wait in a kernel ran out";
    case DF11_ERR_NO_DEVICE: return "no usable CUDA device";
  }
  return "unknown status";
}

namespace {

inline uint64_t ceil_div(uint64_t a, uint64_t b) { return (a + b - 1) / b; }
inline uint64_t round_up(uint64_t a, uint64_t b) { return ceil_div(a, b) * b; }

}  // namespace

extern "C" df11_status df11_build_codebook(const uint64_t hist256[256], uint32_t cap,
                                           df11_codebook *out) {
  if (!hist256 || !out || cap < 1 || cap > DF11_MAX_CODE_LEN) return DF11_ERR_INVALID_ARG;
  std::unique_ptr<df11cb::Scratch> sc(new df11cb::Scratch());
  return df11cb::build_codebook(hist256, cap, out, *sc);
}

extern "C" df11_status df11_encoded_sizes(const df11_codebook *cb, const uint64_t hist256[256],
                                          uint64_t n, df11_sizes *out) {
  if (!cb || !hist256 || !out) return DF11_ERR_INVALID_ARG;
  if (n > DF11_MAX_N) return DF11_ERR_TOO_LARGE;
  uint64_t counted = 0, bits = 0;
  for (int s = 0; s < 256; ++s) {
    if (!hist256[s]) continue;
    if (!cb->len[s]) return DF11_ERR_SYMBOL_NOT_IN_CODEBOOK;
    counted += hist256[s];
    bits += hist256[s] * (uint64_t)cb->len[s];
  }
  if (counted != n) return DF11_ERR_INVALID_ARG;
  return df11_sizes_from_bits(n, bits, out);
}

extern "C" df11_status df11_sizes_from_bits(uint64_t n, uint64_t bits, df11_sizes *out) {
  if (!out) return DF11_ERR_INVALID_ARG;
  if (n > DF11_MAX_N) return DF11_ERR_TOO_LARGE;
  if (bits > n * (uint64_t)DF11_MAX_CODE_LEN || bits < n) return DF11_ERR_INVALID_ARG;
  std::memset(out, 0, sizeof(*out));
  const uint64_t C = ceil_div(bits, DF11_CHUNK_BITS);
  const uint64_t B = ceil_div(C, DF11_BLOCK_CHUNKS);
  out->n = n;
  out->total_bits = bits;
  out->n_chunks = C;
  out->n_blocks = B;
  out->stream_bytes = 8 * C;
  out->gaps_bytes = ceil_div(DF11_GAP_BITS * C, 8);
  out->block_pos_bytes = 4 * (B + 1);
  out->sign_mantissa_bytes = n;
  out->stored_bytes = out->stream_bytes + out->gaps_bytes + out->block_pos_bytes +
                      out->sign_mantissa_bytes + 256;
  // whole-block bulk copies: 2048 B of stream + the next chunk, 160 B of gaps,
  // the sign/mantissa bytes of a block rounded out to 16 B
  out->stream_alloc = 8 * DF11_BLOCK_CHUNKS * B + 16;
  out->gaps_alloc = (DF11_GAP_BITS * DF11_BLOCK_CHUNKS / 8) * B + 16;
  out->block_pos_alloc = round_up(4 * (B + 1), 16);
  out->sign_mantissa_alloc = round_up(n, 16) + 16;
  out->tables_bytes = sizeof(DecodeTables);
  out->workspace_bytes = 8 * (ceil_div(n, df11i::kEncTile) + 1) + 16;
  return DF11_OK;
}

extern "C" size_t df11_tables_bytes(void) { return sizeof(DecodeTables); }

extern "C" df11_status df11_build_tables(const df11_codebook *cb, void *h_tables, size_t bytes) {
  if (!cb || !h_tables || bytes < sizeof(DecodeTables)) return DF11_ERR_INVALID_ARG;
  std::unique_ptr<DecodeTables> t(new DecodeTables());
  std::memset(t.get(), 0, sizeof(DecodeTables));
  df11cb::TableAux aux;
  df11_status st = df11cb::table_header(cb, t.get(), aux);
  if (st != DF11_OK) return st;
  for (uint32_t v = 0; v < (uint32_t)df11i::kLutSize; ++v)
    t->lut[v] = df11cb::lut_entry_for(*t, aux, cb->max_len, v);
  std::memcpy(h_tables, t.get(), sizeof(DecodeTables));
  return DF11_OK;
}

extern "C" df11_status df11_validate(uint64_t n, uint64_t total_bits, uint32_t min_len,
                                     const uint8_t *h_gaps, uint64_t gaps_bytes,
                                     const uint32_t *h_block_pos, uint64_t block_pos_count) {
  if (n > DF11_MAX_N) return DF11_ERR_TOO_LARGE;
  if (min_len < 1 || min_len > DF11_MAX_CODE_LEN) return DF11_ERR_INVALID_ARG;
  const uint64_t C = ceil_div(total_bits, DF11_CHUNK_BITS);
  const uint64_t B = ceil_div(C, DF11_BLOCK_CHUNKS);
  if ((n == 0) != (total_bits == 0)) return DF11_ERR_CORRUPT;
  if (total_bits < n * (uint64_t)min_len || total_bits > n * (uint64_t)DF11_MAX_CODE_LEN)
    return DF11_ERR_CORRUPT;
  if (gaps_bytes < ceil_div(DF11_GAP_BITS * C, 8) || block_pos_count < B + 1)
    return DF11_ERR_INVALID_ARG;
  if ((C && !h_gaps) || !h_block_pos) return DF11_ERR_INVALID_ARG;
  for (uint64_t c = 0; c < C; ++c) {
    uint64_t bit = DF11_GAP_BITS * c;
    unsigned hi = h_gaps[bit >> 3];
    unsigned lo = (bit >> 3) + 1 < gaps_bytes ? h_gaps[(bit >> 3) + 1] : 0;
    unsigned g = (((hi << 8) | lo) >> (11 - (bit & 7))) & 31u;
    uint64_t avail = std::min<uint64_t>(DF11_CHUNK_BITS, total_bits - DF11_CHUNK_BITS * c);
    if (g > avail || (g == avail && c + 1 != C)) return DF11_ERR_CORRUPT;
  }
  if (h_block_pos[0] != 0 || h_block_pos[B] != n) return DF11_ERR_CORRUPT;
  const uint64_t per_chunk = ceil_div(DF11_CHUNK_BITS, min_len);
  for (uint64_t b = 0; b < B; ++b) {
    if (h_block_pos[b + 1] < h_block_pos[b]) return DF11_ERR_CORRUPT;
    if (h_block_pos[b + 1] - h_block_pos[b] > per_chunk * DF11_BLOCK_CHUNKS) return DF11_ERR_CORRUPT;
  }
  return DF11_OK;
}
