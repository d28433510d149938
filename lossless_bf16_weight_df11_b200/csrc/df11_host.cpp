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
#include <array>
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
    case DF11_ERR_BOUNDS: return "bounds check failed (checked build)";
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
  out->run_index_bytes = 2 * (DF11_BLOCK_CHUNKS / 2) * B;
  out->seg_index_bytes = round_up(4 * (ceil_div(n, DF11_SEGMENT) + 1), 16);
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

// ---------------------------------------------------------------- codebook from lengths

extern "C" df11_status df11_codebook_from_lengths(const uint8_t len[256], uint32_t cap,
                                                  df11_codebook *out) {
  if (!len || !out || cap < 1 || cap > DF11_MAX_CODE_LEN) return DF11_ERR_INVALID_ARG;
  uint32_t len_count[DF11_MAX_CODE_LEN + 1] = {0};
  // Kraft sum in units of 2^-32: a prefix code needs sum <= 1
  uint64_t kraft = 0;
  for (int s = 0; s < 256; ++s) {
    if (len[s] > DF11_MAX_CODE_LEN) return DF11_ERR_INVALID_ARG;
    if (len[s]) {
      ++len_count[len[s]];
      kraft += 1ull << (32 - len[s]);
    }
  }
  if (kraft > (1ull << 32)) return DF11_ERR_INVALID_ARG;
  std::memset(out, 0, sizeof(*out));
  uint64_t next[DF11_MAX_CODE_LEN + 1];
  df11cb::first_codes(len_count, next);
  out->min_len = DF11_MAX_CODE_LEN;
  for (int s = 0; s < 256; ++s) {
    out->len[s] = len[s];
    out->code[s] = df11cb::canonical_code(len, next, s);
    if (len[s]) {
      ++out->n_symbols;
      out->max_len = std::max<uint32_t>(out->max_len, len[s]);
      out->min_len = std::min<uint32_t>(out->min_len, len[s]);
    }
  }
  if (!out->n_symbols) out->min_len = 0;
  out->cap = cap;
  return DF11_OK;
}

// ---------------------------------------------------------------- .df11 container

namespace {

constexpr uint8_t kMagic[4] = {'D', 'F', '1', '1'};

// CRC-32 of IEEE 802.3 (reflected, polynomial 0xEDB88320, initial and final
// value 0xFFFFFFFF), table driven.
uint32_t crc32_update(uint32_t crc, const uint8_t *p, uint64_t n) {
  static const std::array<uint32_t, 256> table = [] {  // thread-safe static init
    std::array<uint32_t, 256> t{};
    for (uint32_t i = 0; i < 256; ++i) {
      uint32_t c = i;
      for (int k = 0; k < 8; ++k) c = (c & 1u) ? 0xEDB88320u ^ (c >> 1) : c >> 1;
      t[i] = c;
    }
    return t;
  }();
  crc = ~crc;
  for (uint64_t i = 0; i < n; ++i) crc = table[(crc ^ p[i]) & 0xFFu] ^ (crc >> 8);
  return ~crc;
}

inline void put_u32(uint8_t *p, uint32_t v) {
  for (int i = 0; i < 4; ++i) p[i] = (uint8_t)(v >> (8 * i));
}
inline void put_u64(uint8_t *p, uint64_t v) {
  for (int i = 0; i < 8; ++i) p[i] = (uint8_t)(v >> (8 * i));
}
inline uint32_t get_u32(const uint8_t *p) {
  uint32_t v = 0;
  for (int i = 0; i < 4; ++i) v |= (uint32_t)p[i] << (8 * i);
  return v;
}
inline uint64_t get_u64(const uint8_t *p) {
  uint64_t v = 0;
  for (int i = 0; i < 8; ++i) v |= (uint64_t)p[i] << (8 * i);
  return v;
}

// Offsets of the container's sections (each at a multiple of 16 bytes), or
// false for an invalid (n, total_bits).
struct FileLayout {
  df11_sizes sz;
  uint64_t gaps, block_pos, stream, sign_mantissa, crc, total;
};

inline uint64_t round16u(uint64_t x) { return (x + 15u) & ~15ull; }

bool file_layout(uint64_t n, uint64_t total_bits, FileLayout *L) {
  if (df11_sizes_from_bits(n, total_bits, &L->sz) != DF11_OK) return false;
  L->gaps = DF11_FILE_HEADER_BYTES;
  L->block_pos = round16u(L->gaps + L->sz.gaps_bytes);
  L->stream = round16u(L->block_pos + L->sz.block_pos_bytes);
  L->sign_mantissa = round16u(L->stream + L->sz.stream_bytes);
  L->crc = round16u(L->sign_mantissa + L->sz.sign_mantissa_bytes);
  L->total = L->crc + 4;
  return true;
}

bool shape_matches(uint32_t ndim, const uint64_t *shape, uint64_t n) {
  if (ndim > 4) return false;
  if (ndim == 0) return true;
  unsigned __int128 prod = 1;
  for (uint32_t i = 0; i < ndim; ++i) prod *= shape[i];
  for (uint32_t i = ndim; i < 4; ++i)
    if (shape[i]) return false;
  return prod == n;
}

}  // namespace

extern "C" uint64_t df11_file_bytes(uint64_t n, uint64_t total_bits) {
  FileLayout L;
  return file_layout(n, total_bits, &L) ? L.total : 0;
}

extern "C" df11_status df11_write(const df11_host_matrix *m, void *buf, uint64_t buf_bytes,
                                  uint64_t *written) {
  if (!m || !buf || !written || !m->lengths) return DF11_ERR_INVALID_ARG;
  FileLayout L;
  if (!file_layout(m->n, m->total_bits, &L)) return DF11_ERR_INVALID_ARG;
  const df11_sizes &sz = L.sz;
  if ((sz.gaps_bytes && !m->gaps) || !m->block_pos || (sz.stream_bytes && !m->stream) ||
      (m->n && !m->sign_mantissa))
    return DF11_ERR_INVALID_ARG;
  if (!shape_matches(m->ndim, m->shape, m->n)) return DF11_ERR_INVALID_ARG;
  df11_codebook cb;
  if (df11_codebook_from_lengths(m->lengths, m->cap ? m->cap : DF11_MAX_CODE_LEN, &cb) != DF11_OK)
    return DF11_ERR_INVALID_ARG;
  if (buf_bytes < L.total) return DF11_ERR_INVALID_ARG;
  uint8_t *p = static_cast<uint8_t *>(buf);
  std::memset(p, 0, L.total);
  std::memcpy(p, kMagic, 4);
  put_u32(p + 4, DF11_FILE_VERSION);
  put_u64(p + 8, m->n);
  put_u64(p + 16, m->total_bits);
  put_u32(p + 24, m->cap);
  put_u32(p + 28, m->max_block_codes);
  put_u32(p + 32, m->ndim);
  for (uint32_t i = 0; i < 4; ++i) put_u64(p + 40 + 8 * i, i < m->ndim ? m->shape[i] : 0);
  std::memcpy(p + 72, m->lengths, 256);
  if (sz.gaps_bytes) std::memcpy(p + L.gaps, m->gaps, sz.gaps_bytes);
  for (uint64_t b = 0; b <= sz.n_blocks; ++b) put_u32(p + L.block_pos + 4 * b, m->block_pos[b]);
  if (sz.stream_bytes) std::memcpy(p + L.stream, m->stream, sz.stream_bytes);
  if (m->n) std::memcpy(p + L.sign_mantissa, m->sign_mantissa, m->n);
  put_u32(p + L.crc, crc32_update(0, p, L.crc));
  *written = L.total;
  return DF11_OK;
}

extern "C" df11_status df11_read(const void *buf, uint64_t buf_bytes, df11_host_matrix *out) {
  if (!buf || !out) return DF11_ERR_INVALID_ARG;
  const uint8_t *p = static_cast<const uint8_t *>(buf);
  if (buf_bytes < DF11_FILE_HEADER_BYTES + 4) return DF11_ERR_CORRUPT;
  if (std::memcmp(p, kMagic, 4) != 0 || get_u32(p + 4) != DF11_FILE_VERSION) return DF11_ERR_CORRUPT;
  df11_host_matrix m;
  std::memset(&m, 0, sizeof(m));
  m.n = get_u64(p + 8);
  m.total_bits = get_u64(p + 16);
  m.cap = get_u32(p + 24);
  m.max_block_codes = get_u32(p + 28);
  m.ndim = get_u32(p + 32);
  for (int i = 0; i < 4; ++i) m.shape[i] = get_u64(p + 40 + 8 * i);
  if (get_u32(p + 36) != 0 || !shape_matches(m.ndim, m.shape, m.n)) return DF11_ERR_CORRUPT;
  FileLayout L;
  if (!file_layout(m.n, m.total_bits, &L) || L.total != buf_bytes) return DF11_ERR_CORRUPT;
  if (crc32_update(0, p, L.crc) != get_u32(p + L.crc)) return DF11_ERR_CORRUPT;
  m.lengths = p + 72;
  df11_codebook cb;
  if (df11_codebook_from_lengths(m.lengths, DF11_MAX_CODE_LEN, &cb) != DF11_OK) return DF11_ERR_CORRUPT;
  // the arrays are returned in place: block positions are little-endian
  // uint32 in the file, as in memory on every CUDA host, at a 16-byte offset
  if (((uintptr_t)p & 3u) != 0) return DF11_ERR_INVALID_ARG;
  m.gaps = p + L.gaps;
  m.block_pos = reinterpret_cast<const uint32_t *>(p + L.block_pos);
  m.stream = p + L.stream;
  m.sign_mantissa = p + L.sign_mantissa;
  if (m.n) {
    const df11_status st = df11_validate(m.n, m.total_bits, cb.min_len ? cb.min_len : 1, m.gaps,
                                         L.sz.gaps_bytes, m.block_pos, L.sz.n_blocks + 1);
    if (st != DF11_OK) return DF11_ERR_CORRUPT;
  }
  *out = m;
  return DF11_OK;
}
