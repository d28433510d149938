// df11_host.cpp -- host half of the DF11 library: codebook construction,
// buffer sizing, decode-table construction and metadata validation.
//
// Method: "DFloat11: Nén suy luận GPU không mất dữ liệu, giảm LLM xuống còn 70%
// kích thước" (vi.news.hada.io/topic?id=20542), sections "Định dạng DFloat11"
// (Huffman code of the exponents), "Giải mã dựa trên LUT phân cấp" (table
// decoding, code lengths up to 32) and "Kernel GPU hai giai đoạn và metadata
// bổ trợ" (chunks, gaps, block positions).
//
// The codebook rule (which the page leaves open) is: Huffman with every merge
// taking the two smallest (weight, id) nodes, leaves numbered by (count asc,
// value asc) before the internal nodes, which are numbered in creation order;
// if the longest code exceeds the cap, package-merge with leaves before
// equal-weight packages and the 2(m-1) cheapest items of the last list taken;
// then the multiset of lengths is handed to values by (count desc, value asc);
// canonical codes as in RFC 1951 section 3.2.2.
#include <algorithm>
#include <cstring>
#include <vector>

#include "df11.h"
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

// Values with a nonzero count in (count asc, value asc) order.
std::vector<int> ascending_symbols(const uint64_t *hist) {
  std::vector<int> v;
  for (int s = 0; s < 256; ++s)
    if (hist[s]) v.push_back(s);
  std::stable_sort(v.begin(), v.end(), [&](int a, int b) { return hist[a] < hist[b]; });
  return v;
}

// Two-queue Huffman: leaves in ascending order, internal nodes in creation
// order (their weights never decrease).  The smaller front wins; a leaf wins
// a tie because every leaf id is below every internal id.  Writes the depth
// of leaf i (in `order`) to depth[i]; returns the longest.
int huffman_depths(const uint64_t *hist, const std::vector<int> &order, std::vector<int> &depth) {
  const int m = (int)order.size();
  depth.assign(m, 0);
  if (m == 1) {
    depth[0] = 1;
    return 1;
  }
  std::vector<uint64_t> iw;  // internal weights
  std::vector<int> parent(2 * m - 1, -1);
  iw.reserve(m);
  int li = 0, qi = 0;
  auto pop = [&]() -> int {  // returns node id: leaves 0..m-1, internal m..
    bool leaf;
    if (li >= m) leaf = false;
    else if (qi >= (int)iw.size()) leaf = true;
    else leaf = hist[order[li]] <= iw[qi];
    return leaf ? li++ : m + qi++;
  };
  auto weight_of = [&](int id) { return id < m ? hist[order[id]] : iw[id - m]; };
  for (int k = 0; k < m - 1; ++k) {
    int a = pop();
    int b = pop();
    int id = m + (int)iw.size();
    iw.push_back(weight_of(a) + weight_of(b));
    parent[a] = id;
    parent[b] = id;
  }
  // the root is the last internal node; depths top-down in reverse creation order
  std::vector<int> d(2 * m - 1, 0);
  for (int id = 2 * m - 3; id >= 0; --id) d[id] = d[parent[id]] + 1;
  int longest = 0;
  for (int i = 0; i < m; ++i) {
    depth[i] = d[i];
    longest = std::max(longest, d[i]);
  }
  return longest;
}

// Package-merge in counting form.  Each level's list is kept as weights plus,
// per position, whether the item is a leaf.  The selected items of a level
// always form a prefix of its list; a prefix holding P packages selects the
// first 2P items of the next deeper list, and a leaf's code length is the
// number of levels whose selected prefix contains it (leaves appear in every
// list in ascending order, so the selected leaves are the first few).
int package_merge_depths(const uint64_t *hist, const std::vector<int> &order, int cap,
                         std::vector<int> &depth) {
  const int m = (int)order.size();
  depth.assign(m, 0);
  if (m == 1) {
    depth[0] = 1;
    return 1;
  }
  if (cap < 31 && (1ull << cap) < (uint64_t)m) return -1;
  // lists[d] for d = 1..cap; lists[cap] = leaves
  std::vector<std::vector<uint64_t>> w(cap + 1);
  std::vector<std::vector<uint8_t>> is_leaf(cap + 1);
  for (int i = 0; i < m; ++i) {
    w[cap].push_back(hist[order[i]]);
    is_leaf[cap].push_back(1);
  }
  for (int d = cap - 1; d >= 1; --d) {
    const auto &deeper = w[d + 1];
    size_t npk = deeper.size() / 2;
    size_t li = 0, pi = 0;
    while (li < (size_t)m || pi < npk) {
      bool leaf;
      uint64_t pw = pi < npk ? deeper[2 * pi] + deeper[2 * pi + 1] : 0;
      if (li >= (size_t)m) leaf = false;
      else if (pi >= npk) leaf = true;
      else leaf = hist[order[li]] <= pw;
      if (leaf) {
        w[d].push_back(hist[order[li++]]);
        is_leaf[d].push_back(1);
      } else {
        w[d].push_back(pw);
        is_leaf[d].push_back(0);
        ++pi;
      }
    }
  }
  size_t take = 2 * (size_t)(m - 1);
  int longest = 0;
  for (int d = 1; d <= cap && take > 0; ++d) {
    size_t leaves = 0, packages = 0;
    for (size_t k = 0; k < take && k < w[d].size(); ++k) {
      if (is_leaf[d][k]) ++leaves;
      else ++packages;
    }
    for (size_t i = 0; i < leaves; ++i) {
      depth[i] += 1;
      longest = std::max(longest, depth[i]);
    }
    take = 2 * packages;
  }
  return longest;
}

// (count desc, value asc) order gets the ascending lengths.
void normalise(const uint64_t *hist, uint8_t *len) {
  std::vector<int> syms;
  std::vector<int> lens;
  for (int s = 0; s < 256; ++s)
    if (len[s]) {
      syms.push_back(s);
      lens.push_back(len[s]);
    }
  std::sort(lens.begin(), lens.end());
  std::stable_sort(syms.begin(), syms.end(), [&](int a, int b) { return hist[a] > hist[b]; });
  for (size_t i = 0; i < syms.size(); ++i) len[syms[i]] = (uint8_t)lens[i];
}

void canonical(df11_codebook *cb) {
  uint32_t count[DF11_MAX_CODE_LEN + 1] = {0};
  for (int s = 0; s < 256; ++s)
    if (cb->len[s]) ++count[cb->len[s]];
  uint64_t next[DF11_MAX_CODE_LEN + 2] = {0};
  uint64_t c = 0;
  for (unsigned l = 1; l <= DF11_MAX_CODE_LEN; ++l) {
    c = (c + count[l - 1] * (l > 1 ? 1u : 0u)) << 1;
    next[l] = c;
  }
  for (int s = 0; s < 256; ++s) {
    cb->code[s] = 0;
    if (cb->len[s]) cb->code[s] = (uint32_t)next[cb->len[s]]++;
  }
}

inline uint64_t ceil_div(uint64_t a, uint64_t b) { return (a + b - 1) / b; }
inline uint64_t round_up(uint64_t a, uint64_t b) { return ceil_div(a, b) * b; }

}  // namespace

extern "C" df11_status df11_build_codebook(const uint64_t hist256[256], uint32_t cap,
                                           df11_codebook *out) {
  if (!hist256 || !out || cap < 1 || cap > DF11_MAX_CODE_LEN) return DF11_ERR_INVALID_ARG;
  std::memset(out, 0, sizeof(*out));
  out->cap = cap;
  std::vector<int> order = ascending_symbols(hist256);
  const int m = (int)order.size();
  if (m == 0) return DF11_OK;
  std::vector<int> depth;
  int longest = huffman_depths(hist256, order, depth);
  if (longest > (int)cap) {
    longest = package_merge_depths(hist256, order, (int)cap, depth);
    if (longest < 0) return DF11_ERR_INVALID_ARG;
  }
  for (int i = 0; i < m; ++i) out->len[order[i]] = (uint8_t)depth[i];
  normalise(hist256, out->len);
  canonical(out);
  out->n_symbols = (uint32_t)m;
  out->max_len = 0;
  out->min_len = DF11_MAX_CODE_LEN;
  for (int s = 0; s < 256; ++s)
    if (out->len[s]) {
      out->max_len = std::max<uint32_t>(out->max_len, out->len[s]);
      out->min_len = std::min<uint32_t>(out->min_len, out->len[s]);
    }
  return DF11_OK;
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
  DecodeTables t;
  std::memset(&t, 0, sizeof(t));
  // canonical structure: codes of length L are first[L] .. first[L]+count[L]-1
  uint64_t count[DF11_MAX_CODE_LEN + 1] = {0};
  uint64_t first[DF11_MAX_CODE_LEN + 1] = {0};
  int rank_start[DF11_MAX_CODE_LEN + 2] = {0};
  for (int s = 0; s < 256; ++s) {
    if (cb->len[s] > DF11_MAX_CODE_LEN) return DF11_ERR_INVALID_ARG;
    if (cb->len[s]) ++count[cb->len[s]];
  }
  int r = 0;
  for (unsigned l = 1; l <= DF11_MAX_CODE_LEN; ++l) {
    rank_start[l] = r;
    for (int s = 0; s < 256; ++s)
      if (cb->len[s] == l) {
        if (r == rank_start[l]) first[l] = cb->code[s];
        t.sym[r++] = (uint8_t)s;
      }
  }
  // a length without codes still gets the canonical start so limits stay monotone
  {
    uint64_t c = 0;
    for (unsigned l = 1; l <= DF11_MAX_CODE_LEN; ++l) {
      c = (c + (l > 1 ? count[l - 1] : 0)) << 1;
      if (!count[l]) first[l] = c;
      else if (first[l] != c) return DF11_ERR_INVALID_ARG;  // not canonical
    }
  }
  for (unsigned l = 1; l <= DF11_MAX_CODE_LEN; ++l) {
    t.limit[l] = (first[l] + count[l]) << (32 - l);
    t.base[l] = (uint32_t)((int64_t)rank_start[l] - (int64_t)first[l]);
  }
  t.limit[0] = 0;
  for (int s = 0; s < 256; ++s) t.codelen[s] = cb->len[s];
  t.max_len = cb->max_len;
  t.min_len = cb->min_len;
  t.n_symbols = cb->n_symbols;
  t.lut_bits = df11i::kLutBits;
  const int K = df11i::kLutBits;
  const unsigned maxl = cb->max_len ? cb->max_len : 1;
  for (uint32_t v = 0; v < (uint32_t)df11i::kLutSize; ++v) {
    uint32_t used = 0, nsym = 0, syms = 0;
    while (nsym < 3) {
      // the code starting at bit `used` of the K-bit window v, if whole
      uint64_t window = ((uint64_t)v << (32 - K)) << used;  // left-justified, zeros after
      window &= 0xFFFFFFFFull;
      int found = -1;
      unsigned L = 0;
      for (L = 1; L <= maxl && used + L <= (unsigned)K; ++L) {
        if (window < t.limit[L]) {
          uint64_t c = window >> (32 - L);
          if (count[L] && c >= first[L] && c - first[L] < count[L])
            found = t.sym[rank_start[L] + (c - first[L])];
          break;
        }
      }
      if (found < 0) break;
      syms |= (uint32_t)found << (8 * nsym);
      ++nsym;
      used += L;
    }
    t.lut[v] = nsym ? df11i::lut_entry(syms, nsym, used)
                    : (df11i::lut_entry(0, 0, (uint32_t)K) | df11i::kLutLongFlag);
  }
  std::memcpy(h_tables, &t, sizeof(t));
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
