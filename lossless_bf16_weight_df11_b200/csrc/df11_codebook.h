// df11_codebook.h -- the codebook and decode-table construction of the DF11
// library, written once for the host (df11_build_codebook, df11_build_tables)
// and the device (df11_build_codebook_device).  Not part of the public ABI.
//
// Page: "DFloat11: Nén suy luận GPU không mất dữ liệu, giảm LLM xuống còn 70% kích
// thước" (vi.news.hada.io/topic?id=20542), sections "Định dạng DFloat11"
// (Huffman code of the exponents) and "Giải mã dựa trên LUT phân cấp" (table
// decoding, code lengths up to 32).
//
// The codebook rule (the page leaves it open):
//   - Huffman, every merge taking the two smallest (weight, id) nodes, leaves
//     numbered by (count asc, value asc) before the internal nodes, which are
//     numbered in creation order (two queues: leaves in order, internal nodes
//     in creation order, a leaf winning a tie);
//   - if the longest code exceeds the cap, package-merge with leaves before
//     equal-weight packages and the 2(m-1) cheapest items of the top list;
//   - the multiset of lengths handed to values by (count desc, value asc);
//   - canonical codes as in RFC 1951 section 3.2.2.
//
// Steps that depend on one value only (ranks, lengths after normalisation,
// canonical codes, table entries) are per-value functions, so the device can
// run them on 256 threads; the two tree constructions are sequential.
#pragma once

#include <stdint.h>

#include "df11.h"
#include "df11_internal.h"

#ifdef __CUDACC__
#define DF11_HD __host__ __device__
#else
#define DF11_HD
#endif

namespace df11cb {

constexpr int kMaxSyms = 256;
constexpr int kMaxList = 2 * kMaxSyms;  // items of a package-merge list (< 2m)
constexpr int kListWords = kMaxList / 32;

// Working memory of the sequential steps (about 11 KiB).
struct Scratch {
  uint64_t hist_sorted[kMaxSyms];           // counts in (count asc, value asc) order
  uint8_t depth[kMaxSyms];                  // code length of the i-th leaf in that order
  uint64_t internal_w[kMaxSyms];            // Huffman internal-node weights
  int16_t parent[kMaxList];                 // Huffman parents (leaves 0..m-1, internal m..)
  uint8_t node_depth[kMaxList];
  uint64_t list_a[kMaxList], list_b[kMaxList];       // package-merge: two levels' weights
  uint32_t leaf_bits[DF11_MAX_CODE_LEN + 1][kListWords];  // per level: item is a leaf
  uint16_t list_len[DF11_MAX_CODE_LEN + 1];
};

// Canonical structure of a codebook, for the tables: codes of length L are
// first[L] .. first[L] + count[L] - 1, at ranks rank_start[L] .. in sym[].
struct TableAux {
  uint64_t count[DF11_MAX_CODE_LEN + 1];
  uint64_t first[DF11_MAX_CODE_LEN + 1];
  int32_t rank_start[DF11_MAX_CODE_LEN + 2];
};

// Position of value s among the present values in (count asc, value asc).
DF11_HD inline int ascending_rank(const uint64_t *hist, int s) {
  int r = 0;
  for (int t = 0; t < kMaxSyms; ++t)
    if (hist[t] && (hist[t] < hist[s] || (hist[t] == hist[s] && t < s))) ++r;
  return r;
}

// Position of value s among the present values in (count desc, value asc).
DF11_HD inline int descending_rank(const uint64_t *hist, int s) {
  int r = 0;
  for (int t = 0; t < kMaxSyms; ++t)
    if (hist[t] && (hist[t] > hist[s] || (hist[t] == hist[s] && t < s))) ++r;
  return r;
}

// Two-queue Huffman over sc.hist_sorted[0..m); lengths to sc.depth; returns
// the longest.
DF11_HD inline int huffman_depths(int m, Scratch &sc) {
  if (m < 1 || m > kMaxSyms) return -1;
  if (m == 1) {
    sc.depth[0] = 1;
    return 1;
  }
  int li = 0, qi = 0, nq = 0;
  for (int k = 0; k < m - 1; ++k) {
    int pick[2];
    for (int j = 0; j < 2; ++j) {
      bool leaf;
      if (li >= m) leaf = false;
      else if (qi >= nq) leaf = true;
      else leaf = sc.hist_sorted[li] <= sc.internal_w[qi];
      pick[j] = leaf ? li++ : m + qi++;
    }
    uint64_t w = 0;
    for (int j = 0; j < 2; ++j)
      w += pick[j] < m ? sc.hist_sorted[pick[j]] : sc.internal_w[pick[j] - m];
    const int id = m + nq;
    sc.internal_w[nq++] = w;
    sc.parent[pick[0]] = (int16_t)id;
    sc.parent[pick[1]] = (int16_t)id;
  }
  // the root is the last internal node (id 2m-2); depths top-down
  sc.node_depth[2 * m - 2] = 0;
  int longest = 0;
  for (int id = 2 * m - 3; id >= 0; --id) {
    sc.node_depth[id] = (uint8_t)(sc.node_depth[sc.parent[id]] + 1);
    if (id < m) {
      sc.depth[id] = sc.node_depth[id];
      if (sc.depth[id] > longest) longest = sc.depth[id];
    }
  }
  return longest;
}

// Package-merge in counting form.  Level cap holds the leaves; level d < cap
// merges the leaves with the packages (consecutive pairs) of level d+1, a
// leaf first on equal weight.  Only each level's leaf flags are kept: the
// selected items of a level form a prefix; a prefix holding P packages
// selects the first 2P items of the level below, and a leaf's length is the
// number of levels whose selected prefix contains it.  Returns the longest
// length, or -1 when 2^cap < m.
DF11_HD inline int package_merge_depths(int m, int cap, Scratch &sc) {
  if (m < 1 || m > kMaxSyms || cap < 1 || cap > (int)DF11_MAX_CODE_LEN) return -1;
  if (m == 1) {
    sc.depth[0] = 1;
    return 1;
  }
  if (cap < 31 && (1ull << cap) < (uint64_t)m) return -1;
  uint64_t *deeper = sc.list_a, *cur = sc.list_b;
  for (int w = 0; w < kListWords; ++w) sc.leaf_bits[cap][w] = 0;
  for (int i = 0; i < m; ++i) {
    deeper[i] = sc.hist_sorted[i];
    sc.leaf_bits[cap][i >> 5] |= 1u << (i & 31);
  }
  sc.list_len[cap] = (uint16_t)m;
  for (int d = cap - 1; d >= 1; --d) {
    const int npk = sc.list_len[d + 1] / 2;
    int li = 0, pi = 0, k = 0;
    for (int w = 0; w < kListWords; ++w) sc.leaf_bits[d][w] = 0;
    while (li < m || pi < npk) {
      const uint64_t pw = pi < npk ? deeper[2 * pi] + deeper[2 * pi + 1] : 0;
      bool leaf;
      if (li >= m) leaf = false;
      else if (pi >= npk) leaf = true;
      else leaf = sc.hist_sorted[li] <= pw;
      if (leaf) {
        cur[k] = sc.hist_sorted[li++];
        sc.leaf_bits[d][k >> 5] |= 1u << (k & 31);
      } else {
        cur[k] = pw;
        ++pi;
      }
      ++k;
    }
    sc.list_len[d] = (uint16_t)k;
    uint64_t *t = deeper;
    deeper = cur;
    cur = t;
  }
  for (int i = 0; i < m; ++i) sc.depth[i] = 0;
  int take = 2 * (m - 1), longest = 0;
  for (int d = 1; d <= cap && take > 0; ++d) {
    const int lim = take < sc.list_len[d] ? take : sc.list_len[d];
    int leaves = 0;
    for (int k = 0; k < lim; ++k) leaves += (sc.leaf_bits[d][k >> 5] >> (k & 31)) & 1u;
    for (int i = 0; i < leaves; ++i) {
      ++sc.depth[i];
      if (sc.depth[i] > longest) longest = sc.depth[i];
    }
    take = 2 * (lim - leaves);
  }
  return longest;
}

// Length of value s after normalisation: the lengths of the tree, sorted
// ascending, are handed out in (count desc, value asc) order.
// len_count[L] = how many leaves of the tree got length L.
DF11_HD inline uint8_t normalised_length(const uint64_t *hist, const uint32_t *len_count, int s) {
  if (!hist[s]) return 0;
  int k = descending_rank(hist, s);
  for (int L = 1; L <= (int)DF11_MAX_CODE_LEN; ++L) {
    if (k < (int)len_count[L]) return (uint8_t)L;
    k -= (int)len_count[L];
  }
  return 0;  // unreachable for a consistent len_count
}

// RFC 1951 3.2.2: the first code of each length (next_code), then codes in
// increasing value order within a length.
DF11_HD inline void first_codes(const uint32_t *len_count, uint64_t *next) {
  uint64_t c = 0;
  next[0] = 0;
  for (unsigned l = 1; l <= DF11_MAX_CODE_LEN; ++l) {
    c = (c + (l > 1 ? len_count[l - 1] : 0u)) << 1;
    next[l] = c;
  }
}

DF11_HD inline uint32_t canonical_code(const uint8_t *len, const uint64_t *next, int s) {
  if (!len[s]) return 0;
  uint64_t c = next[len[s]];
  for (int t = 0; t < s; ++t) c += len[t] == len[s];
  return (uint32_t)c;
}

// The whole codebook, sequentially (the host's path).  hist: 256 counts.
DF11_HD inline df11_status build_codebook(const uint64_t *hist, uint32_t cap, df11_codebook *out,
                                          Scratch &sc) {
  if (cap < 1 || cap > DF11_MAX_CODE_LEN) return DF11_ERR_INVALID_ARG;
  uint8_t *raw = reinterpret_cast<uint8_t *>(out);
  for (unsigned i = 0; i < sizeof(*out); ++i) raw[i] = 0;
  out->cap = cap;
  int m = 0;
  for (int s = 0; s < kMaxSyms; ++s)
    if (hist[s]) ++m;
  if (m == 0) return DF11_OK;
  for (int s = 0; s < kMaxSyms; ++s)
    if (hist[s]) sc.hist_sorted[ascending_rank(hist, s)] = hist[s];
  int longest = huffman_depths(m, sc);
  if (longest < 0) return DF11_ERR_INVALID_ARG;
  if (longest > (int)cap) {
    longest = package_merge_depths(m, (int)cap, sc);
    if (longest < 0) return DF11_ERR_INVALID_ARG;
  }
  uint32_t len_count[DF11_MAX_CODE_LEN + 1] = {0};
  for (int i = 0; i < m; ++i) ++len_count[sc.depth[i]];
  for (int s = 0; s < kMaxSyms; ++s) out->len[s] = normalised_length(hist, len_count, s);
  uint64_t next[DF11_MAX_CODE_LEN + 1];
  first_codes(len_count, next);
  for (int s = 0; s < kMaxSyms; ++s) out->code[s] = canonical_code(out->len, next, s);
  out->n_symbols = (uint32_t)m;
  out->max_len = 0;
  out->min_len = DF11_MAX_CODE_LEN;
  for (int s = 0; s < kMaxSyms; ++s)
    if (out->len[s]) {
      if (out->len[s] > out->max_len) out->max_len = out->len[s];
      if (out->len[s] < out->min_len) out->min_len = out->len[s];
    }
  return DF11_OK;
}

// The per-length part of the decode tables: counts, canonical first codes,
// rank starts, limit/base, and the scalar fields (everything but sym[] and
// the lookup table); t must be zeroed.  DF11_ERR_INVALID_ARG for a length
// above 32 or codes that are not canonical.
DF11_HD inline df11_status table_lengths(const df11_codebook *cb, df11i::DecodeTables *t,
                                         TableAux &aux) {
  bool seen[DF11_MAX_CODE_LEN + 1];
  for (int l = 0; l <= (int)DF11_MAX_CODE_LEN; ++l) {
    aux.count[l] = aux.first[l] = 0;
    seen[l] = false;
  }
  for (int s = 0; s < kMaxSyms; ++s) {
    const unsigned L = cb->len[s];
    if (L > DF11_MAX_CODE_LEN) return DF11_ERR_INVALID_ARG;
    if (!L) continue;
    ++aux.count[L];
    if (!seen[L]) {  // the smallest value of each length holds its first code
      seen[L] = true;
      aux.first[L] = cb->code[s];
    }
  }
  int r = 0;
  for (unsigned l = 0; l <= DF11_MAX_CODE_LEN + 1; ++l) {
    aux.rank_start[l] = r;
    if (l >= 1 && l <= DF11_MAX_CODE_LEN) r += (int)aux.count[l];
  }
  // a length without codes still gets the canonical start so limits stay monotone
  uint64_t c = 0;
  for (unsigned l = 1; l <= DF11_MAX_CODE_LEN; ++l) {
    c = (c + (l > 1 ? aux.count[l - 1] : 0)) << 1;
    if (!aux.count[l]) aux.first[l] = c;
    else if (aux.first[l] != c) return DF11_ERR_INVALID_ARG;  // not canonical
  }
  for (unsigned l = 1; l <= DF11_MAX_CODE_LEN; ++l) {
    t->limit[l] = (aux.first[l] + aux.count[l]) << (32 - l);
    t->base[l] = (uint32_t)((int64_t)aux.rank_start[l] - (int64_t)aux.first[l]);
  }
  t->limit[0] = 0;
  t->max_len = cb->max_len;
  t->min_len = cb->min_len;
  t->n_symbols = cb->n_symbols;
  t->lut_bits = df11i::kLutBits;
  return DF11_OK;
}

// The per-value part: value s (with a code) goes to sym[] at its rank in
// (length asc, value asc) order, rotated as the decoder stores exponents
// (df11i::ror8), and its length to codelen[s].
DF11_HD inline void table_value(const df11_codebook *cb, df11i::DecodeTables *t, int s) {
  const unsigned L = cb->len[s];
  t->codelen[s] = (uint8_t)L;
  if (!L) return;
  int r = 0;
  for (int u = 0; u < kMaxSyms; ++u) {
    const unsigned Lu = cb->len[u];
    r += Lu && (Lu < L || (Lu == L && u < s));
  }
  t->sym[r] = (uint8_t)df11i::ror8((uint32_t)s);
}

// Everything of the decode tables but the lookup table, sequentially; t must
// be zeroed.
DF11_HD inline df11_status table_header(const df11_codebook *cb, df11i::DecodeTables *t,
                                        TableAux &aux) {
  const df11_status st = table_lengths(cb, t, aux);
  if (st != DF11_OK) return st;
  for (int s = 0; s < kMaxSyms; ++s) table_value(cb, t, s);
  return DF11_OK;
}

// Lookup-table entry for the kLutBits-bit window v: the whole codes (at most
// four) in it, decoded greedily, with the start of each code after the first,
// or the long-code flag when the window does not hold a whole first code.
DF11_HD inline df11i::LutEntry lut_entry_for(const df11i::DecodeTables &t, const TableAux &aux,
                                             uint32_t max_len, uint32_t v) {
  const int K = df11i::kLutBits;
  const unsigned maxl = max_len ? max_len : 1;
  uint32_t used = 0, nsym = 0, syms = 0;
  uint32_t start[df11i::kLutMaxCodes] = {0, df11i::kCtrlNoStart, df11i::kCtrlNoStart,
                                         df11i::kCtrlNoStart};
  while (nsym < df11i::kLutMaxCodes) {
    uint64_t window = ((uint64_t)v << (32 - K)) << used;  // left-justified, zeros after
    window &= 0xFFFFFFFFull;
    int found = -1;
    unsigned L = 0;
    for (L = 1; L <= maxl && used + L <= (unsigned)K; ++L) {
      if (window < t.limit[L]) {
        const uint64_t code = window >> (32 - L);
        if (aux.count[L] && code >= aux.first[L] && code - aux.first[L] < aux.count[L])
          found = t.sym[aux.rank_start[L] + (code - aux.first[L])];
        break;
      }
    }
    if (found < 0) break;
    syms |= (uint32_t)found << (8 * nsym);  // sym[] holds rotated exponents
    start[nsym] = used;
    ++nsym;
    used += L;
  }
  df11i::LutEntry e;
  if (nsym) {
    e.x = syms;
    e.y = df11i::lut_ctrl(nsym, start[1], start[2], start[3], used);
  } else {
    e.x = 0;
    // no codes; the bits consumed are the window's, so that a decoder that
    // does not test the flag (codebooks within the table's reach, where a
    // flagged window only occurs in a corrupt stream) still moves on
    e.y = df11i::lut_ctrl(0, df11i::kCtrlNoStart, df11i::kCtrlNoStart, df11i::kCtrlNoStart,
                          (uint32_t)K) |
          df11i::kCtrlLongFlag;
  }
  return e;
}

}  // namespace df11cb
