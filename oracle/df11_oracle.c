/*
 * df11_oracle.c -- plain, slow, single-threaded CPU oracle for the DF11 codec.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the CPU
 * baseline arm of bench.py may load this code.  It shares no source, header,
 * table or helper with the CUDA library, and the library never calls it.
 *
 * Source of the method: the page "DFloat11: Nén suy luận GPU không mất dữ liệu,
 * giảm LLM xuống còn 70% kích thước" (vi.news.hada.io/topic?id=20542).  Sections
 * are cited by their headings:
 *   [Exponent]  "Dư địa nén còn lại trong exponent của BFloat16"
 *   [Format]    "Định dạng DFloat11"
 *   [LUT]       "Giải mã dựa trên LUT phân cấp"
 *   [Kernel]    "Kernel GPU hai giai đoạn và metadata bổ trợ"
 *
 * Everything is written as the definition, step by step and bit by bit: the
 * encoder emits one bit at a time, both decoders consume one bit at a time,
 * the Huffman builder searches the live node list for its two smallest nodes,
 * and package-merge keeps explicit item lists with leaf multiplicities.
 *
 * Readings where the page is silent (each one is listed with its reason in the
 * design notes of the repository):
 *   R1 sign/mantissa byte: sign in bit 7, mantissa in bits 6..0.
 *   R2 Huffman tie-break: leaves ordered by (count asc, symbol asc) get ids
 *      0..m-1, internal nodes get ids m, m+1, ... in creation order, and each
 *      merge takes the two live nodes with the smallest (weight, id).
 *      One symbol -> length 1.
 *   R3 length cap (32): if Huffman exceeds it, package-merge with leaves in the
 *      same order, packages placed after equal-weight leaves, and the first
 *      2(m-1) items of the last list selected.
 *   R4 normalisation: the multiset of lengths is handed out again so that
 *      symbols sorted by (count desc, symbol asc) get lengths in ascending
 *      order.  Canonical codes follow the DEFLATE convention (RFC 1951 3.2.2).
 *   R5 bit order: code bits are written most significant first; stream bit k
 *      is bit (7 - k%8) of byte k/8; the stream is zero-padded to whole
 *      64-bit chunks.
 *   R6 gaps: gap[c] = (first code start >= 64c, or total_bits if none) - 64c.
 *   R8 gap packing: 5 bits per chunk, most significant bit first.
 *   R7 block positions: 256 chunks per block; pos[b] = number of codes that
 *      start before bit 64*256*b; pos[B] = n; stored as uint32.
 *   R12 run index (device-side metadata derived from the stream): for run r
 *      of block b (chunks 2r and 2r+1 of the block), the number of codes that
 *      start in the block before the run, as uint16.
 *   R13 segment index (device-side metadata derived from the stream): for
 *      every 64th value, the stream bit at which its code starts, then
 *      total_bits; uint32.
 *
 * Parity status: every function here is pinned by a test in
 * tests/test_oracle_pins.py (closed forms, brute force, textbook identities,
 * invariants).  The tie-break (R2), the package-merge item order (R3), the
 * normalisation (R4) and the 256-chunk block (R7) are readings of the page,
 * not facts printed on it: parity on those is parity with the reading.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define OR_CHUNK_BITS 64u       /* [Kernel]: one thread owns n = 8 bytes   */
#define OR_BLOCK_CHUNKS 256u    /* R7                                        */
#define OR_GAP_BITS 5u          /* [Kernel]: gaps lie in [0,31], 5 bits      */
#define OR_MAX_CAP 32           /* [Kernel]: longest code is 32 bits         */

enum {
  OR_OK = 0,
  OR_ERR_ARG = 1,
  OR_ERR_SYMBOL = 2,   /* a value to encode has no code                  */
  OR_ERR_CORRUPT = 3,  /* the stream or its metadata is inconsistent     */
};

/* ------------------------------------------------------------------ */
/* Step 1: split a BF16 word into its exponent and sign+mantissa byte. */
/* [Exponent]: 1 sign bit, 8 exponent bits, 7 mantissa bits.           */
/* [Format]: sign and mantissa are kept as they are, in a byte array.  */
/* ------------------------------------------------------------------ */
void oracle_split(const uint16_t *w, uint64_t n, uint8_t *exponent,
                  uint8_t *sign_mantissa) {
  for (uint64_t i = 0; i < n; i++) {
    unsigned word = w[i];
    unsigned sign = (word >> 15) & 1u;
    unsigned expo = (word >> 7) & 0xFFu;
    unsigned mant = word & 0x7Fu;
    exponent[i] = (uint8_t)expo;
    sign_mantissa[i] = (uint8_t)((sign << 7) | mant); /* R1 */
  }
}

/* The inverse of oracle_split. */
void oracle_merge(const uint8_t *exponent, const uint8_t *sign_mantissa,
                  uint64_t n, uint16_t *w) {
  for (uint64_t i = 0; i < n; i++) {
    unsigned sign = (sign_mantissa[i] >> 7) & 1u;
    unsigned mant = sign_mantissa[i] & 0x7Fu;
    unsigned expo = exponent[i];
    w[i] = (uint16_t)((sign << 15) | (expo << 7) | mant);
  }
}

/* ------------------------------------------------------------------ */
/* Step 2: exponent histogram ([Exponent]: the exponent distribution). */
/* ------------------------------------------------------------------ */
void oracle_histogram(const uint8_t *exponent, uint64_t n, uint64_t hist[256]) {
  for (int s = 0; s < 256; s++) hist[s] = 0;
  for (uint64_t i = 0; i < n; i++) hist[exponent[i]] += 1;
}

/* Shannon entropy of the histogram in bits per symbol ([Exponent]). */
double oracle_entropy(const uint64_t hist[256]) {
  double total = 0.0, h = 0.0;
  for (int s = 0; s < 256; s++) total += (double)hist[s];
  if (total <= 0.0) return 0.0;
  for (int s = 0; s < 256; s++) {
    if (hist[s] == 0) continue;
    double p = (double)hist[s] / total;
    h -= p * log2(p);
  }
  return h;
}

/* Symbols with nonzero count, ordered by (count asc, symbol asc).
 * Insertion sort: plain and obviously right for 256 items. */
static int present_symbols_ascending(const uint64_t hist[256], int order[256]) {
  int m = 0;
  for (int s = 0; s < 256; s++) {
    if (hist[s] == 0) continue;
    int j = m;
    while (j > 0) {
      int prev = order[j - 1];
      int prev_after = hist[prev] > hist[s] ||
                       (hist[prev] == hist[s] && prev > s);
      if (!prev_after) break;
      order[j] = prev;
      j--;
    }
    order[j] = s;
    m++;
  }
  return m;
}

/* ------------------------------------------------------------------ */
/* Step 3: Huffman code lengths ([Format]: a Huffman tree built from   */
/* the exponent distribution; frequent values get short codes).  R2.  */
/* Returns the longest length (0 when the histogram is empty).         */
/* ------------------------------------------------------------------ */
int oracle_huffman_lengths(const uint64_t hist[256], uint8_t len[256]) {
  int order[256];
  uint64_t weight[511];
  int parent[511];
  int alive[511];
  for (int s = 0; s < 256; s++) len[s] = 0;
  int m = present_symbols_ascending(hist, order);
  if (m == 0) return 0;
  if (m == 1) {
    len[order[0]] = 1;
    return 1;
  }
  int nodes = m;
  for (int i = 0; i < m; i++) {
    weight[i] = hist[order[i]];
    parent[i] = -1;
    alive[i] = 1;
  }
  for (int live = m; live > 1; live--) {
    int pick[2];
    for (int k = 0; k < 2; k++) {
      int best = -1;
      for (int id = 0; id < nodes; id++) {
        if (!alive[id]) continue;
        /* ids grow with creation order, so the first live node met with
           the smallest weight is the one with the smallest (weight, id) */
        if (best < 0 || weight[id] < weight[best]) best = id;
      }
      alive[best] = 0;
      pick[k] = best;
    }
    weight[nodes] = weight[pick[0]] + weight[pick[1]];
    parent[nodes] = -1;
    alive[nodes] = 1;
    parent[pick[0]] = nodes;
    parent[pick[1]] = nodes;
    nodes++;
  }
  int longest = 0;
  for (int i = 0; i < m; i++) {
    int depth = 0;
    for (int id = i; parent[id] >= 0; id = parent[id]) depth++;
    len[order[i]] = (uint8_t)depth;
    if (depth > longest) longest = depth;
  }
  return longest;
}

/* ------------------------------------------------------------------ */
/* Step 3b: optimal length-limited code by package-merge (Larmore and  */
/* Hirschberg, 1990).  R3.  Every item carries how many times each     */
/* leaf occurs inside it; a code length is the number of selected      */
/* items a symbol occurs in.  Returns the longest length, or -1 if the */
/* cap cannot hold m symbols.                                          */
/* ------------------------------------------------------------------ */
typedef struct {
  uint64_t weight;
  uint8_t mult[256]; /* multiplicity of each leaf (index into order[]) */
} pm_item;

int oracle_package_merge(const uint64_t hist[256], int cap, uint8_t len[256]) {
  int order[256];
  for (int s = 0; s < 256; s++) len[s] = 0;
  int m = present_symbols_ascending(hist, order);
  if (m == 0) return 0;
  if (cap < 1 || cap > OR_MAX_CAP) return -1;
  if (m == 1) {
    len[order[0]] = 1;
    return 1;
  }
  if (cap < 31 && ((uint64_t)1 << cap) < (uint64_t)m) return -1;

  /* a list never holds more than m leaves plus m packages */
  size_t list_cap = (size_t)2 * (size_t)m;
  pm_item *prev = (pm_item *)calloc(list_cap, sizeof(pm_item));
  pm_item *cur = (pm_item *)calloc(list_cap, sizeof(pm_item));
  pm_item *pkg = (pm_item *)calloc(list_cap, sizeof(pm_item));
  if (!prev || !cur || !pkg) {
    free(prev);
    free(cur);
    free(pkg);
    return -1;
  }

  /* the deepest list (denomination 2^-cap) holds the leaves only */
  size_t prev_n = 0;
  for (int i = 0; i < m; i++) {
    memset(&prev[prev_n], 0, sizeof(pm_item));
    prev[prev_n].weight = hist[order[i]];
    prev[prev_n].mult[i] = 1;
    prev_n++;
  }
  for (int level = cap - 1; level >= 1; level--) {
    /* package consecutive pairs of the list one level deeper */
    size_t pkg_n = 0;
    for (size_t k = 0; k + 1 < prev_n; k += 2) {
      pkg[pkg_n].weight = prev[k].weight + prev[k + 1].weight;
      for (int i = 0; i < m; i++)
        pkg[pkg_n].mult[i] = (uint8_t)(prev[k].mult[i] + prev[k + 1].mult[i]);
      pkg_n++;
    }
    /* merge leaves and packages by weight; a leaf goes first on a tie */
    size_t li = 0, pi = 0, cur_n = 0;
    while (li < (size_t)m || pi < pkg_n) {
      int take_leaf;
      if (li >= (size_t)m) take_leaf = 0;
      else if (pi >= pkg_n) take_leaf = 1;
      else take_leaf = hist[order[li]] <= pkg[pi].weight;
      if (take_leaf) {
        memset(&cur[cur_n], 0, sizeof(pm_item));
        cur[cur_n].weight = hist[order[li]];
        cur[cur_n].mult[li] = 1;
        li++;
      } else {
        cur[cur_n] = pkg[pi];
        pi++;
      }
      cur_n++;
    }
    pm_item *t = prev;
    prev = cur;
    cur = t;
    prev_n = cur_n;
  }
  /* select the 2(m-1) cheapest items of the shallowest list */
  size_t take = (size_t)2 * (size_t)(m - 1);
  int longest = 0;
  unsigned count[256];
  for (int i = 0; i < m; i++) count[i] = 0;
  for (size_t k = 0; k < take && k < prev_n; k++)
    for (int i = 0; i < m; i++) count[i] += prev[k].mult[i];
  for (int i = 0; i < m; i++) {
    len[order[i]] = (uint8_t)count[i];
    if ((int)count[i] > longest) longest = (int)count[i];
  }
  free(prev);
  free(cur);
  free(pkg);
  return longest;
}

/* ------------------------------------------------------------------ */
/* Step 3c: normalisation (R4).                                        */
/* ------------------------------------------------------------------ */
void oracle_normalize_lengths(const uint64_t hist[256], uint8_t len[256]) {
  int syms[256];
  int lens[256];
  int m = 0;
  for (int s = 0; s < 256; s++)
    if (len[s] > 0) syms[m++] = s;
  /* lengths ascending */
  for (int i = 0; i < m; i++) lens[i] = len[syms[i]];
  for (int i = 1; i < m; i++)
    for (int j = i; j > 0 && lens[j - 1] > lens[j]; j--) {
      int t = lens[j];
      lens[j] = lens[j - 1];
      lens[j - 1] = t;
    }
  /* symbols by (count desc, symbol asc) */
  for (int i = 1; i < m; i++)
    for (int j = i; j > 0; j--) {
      int a = syms[j - 1], b = syms[j];
      int swap = hist[a] < hist[b] || (hist[a] == hist[b] && a > b);
      if (!swap) break;
      syms[j - 1] = b;
      syms[j] = a;
    }
  for (int i = 0; i < m; i++) len[syms[i]] = (uint8_t)lens[i];
}

/* ------------------------------------------------------------------ */
/* Step 3d: canonical codes, DEFLATE convention (RFC 1951 3.2.2).      */
/* ------------------------------------------------------------------ */
void oracle_canonical_codes(const uint8_t len[256], uint32_t code[256]) {
  uint64_t bl_count[OR_MAX_CAP + 1];
  uint64_t next_code[OR_MAX_CAP + 2];
  for (int b = 0; b <= OR_MAX_CAP; b++) bl_count[b] = 0;
  for (int s = 0; s < 256; s++)
    if (len[s] > 0) bl_count[len[s]]++;
  uint64_t c = 0;
  bl_count[0] = 0;
  for (int bits = 1; bits <= OR_MAX_CAP; bits++) {
    c = (c + bl_count[bits - 1]) << 1;
    next_code[bits] = c;
  }
  for (int s = 0; s < 256; s++) {
    code[s] = 0;
    if (len[s] == 0) continue;
    code[s] = (uint32_t)next_code[len[s]];
    next_code[len[s]]++;
  }
}

/* Whole codebook: Huffman, cap by package-merge when needed, normalise,
 * canonical codes.  Returns the longest length, or -1 on a bad cap. */
int oracle_codebook(const uint64_t hist[256], int cap, uint8_t len[256],
                    uint32_t code[256]) {
  int longest = oracle_huffman_lengths(hist, len);
  if (longest > cap) longest = oracle_package_merge(hist, cap, len);
  if (longest < 0) return -1;
  oracle_normalize_lengths(hist, len);
  oracle_canonical_codes(len, code);
  return longest;
}

/* Total number of code bits for a sequence of exponents. */
int oracle_total_bits(const uint8_t *exponent, uint64_t n, const uint8_t len[256],
                      uint64_t *total_bits) {
  uint64_t t = 0;
  for (uint64_t i = 0; i < n; i++) {
    if (len[exponent[i]] == 0) return OR_ERR_SYMBOL;
    t += len[exponent[i]];
  }
  *total_bits = t;
  return OR_OK;
}

static void put_bit(uint8_t *stream, uint64_t k, unsigned bit) {
  if (bit) stream[k >> 3] |= (uint8_t)(0x80u >> (k & 7u)); /* R5 */
}

static unsigned get_bit(const uint8_t *stream, uint64_t k) {
  return (stream[k >> 3] >> (7u - (unsigned)(k & 7u))) & 1u;
}

/* ------------------------------------------------------------------ */
/* Step 4: bit-serial encoder.  [Format]: the exponent codes are packed */
/* into the byte array EncodedExponent.  [Kernel]: per chunk the bit    */
/* offset of its first code (gaps, R6) and per block the output index   */
/* of its first code (R7).                                              */
/* stream must hold 8*C zeroed bytes, gap C bytes, pos B+1 entries,     */
/* where C = ceil(total_bits/64) and B = ceil(C/256).                   */
/* ------------------------------------------------------------------ */
int oracle_encode(const uint8_t *exponent, uint64_t n, const uint8_t len[256],
                  const uint32_t code[256], uint64_t total_bits, uint8_t *stream,
                  uint8_t *gap, uint32_t *pos) {
  uint64_t chunks = (total_bits + OR_CHUNK_BITS - 1) / OR_CHUNK_BITS;
  uint64_t blocks = (chunks + OR_BLOCK_CHUNKS - 1) / OR_BLOCK_CHUNKS;
  uint64_t block_bits = (uint64_t)OR_CHUNK_BITS * OR_BLOCK_CHUNKS;
  if (n > 0xFFFFFFFFull) return OR_ERR_ARG;
  uint64_t bit = 0, next_chunk = 0, next_block = 0;
  for (uint64_t i = 0; i < n; i++) {
    unsigned s = exponent[i];
    unsigned l = len[s];
    if (l == 0) return OR_ERR_SYMBOL;
    uint64_t start = bit;
    while (next_chunk < chunks && next_chunk * OR_CHUNK_BITS <= start) {
      gap[next_chunk] = (uint8_t)(start - next_chunk * OR_CHUNK_BITS);
      next_chunk++;
    }
    while (next_block < blocks && next_block * block_bits <= start) {
      pos[next_block] = (uint32_t)i;
      next_block++;
    }
    for (int k = (int)l - 1; k >= 0; k--) {
      put_bit(stream, bit, (code[s] >> k) & 1u);
      bit++;
    }
  }
  if (bit != total_bits) return OR_ERR_ARG;
  while (next_chunk < chunks) {
    gap[next_chunk] = (uint8_t)(total_bits - next_chunk * OR_CHUNK_BITS);
    next_chunk++;
  }
  while (next_block < blocks) {
    pos[next_block] = (uint32_t)n;
    next_block++;
  }
  pos[blocks] = (uint32_t)n;
  for (uint64_t c = 0; c < chunks; c++)
    if (gap[c] > 31) return OR_ERR_CORRUPT;
  return OR_OK;
}

/* ------------------------------------------------------------------ */
/* Run index: for each 128-bit run (two consecutive chunks, the part of */
/* a block one decoding thread takes), the output position of its first */
/* code within its block.  [Kernel] gives one output position per       */
/* thread block; this is the same count one level finer.  R12 (reading):*/
/* run_pos[128*b + r] = number of codes that start at bits              */
/* [16384*b, 16384*b + 128*r); every block has 128 entries (runs past   */
/* the end of the stream hold the block's total).  Written from the     */
/* code lengths, one code start at a time.                              */
/* run_pos must hold 128*B entries, B = ceil(C/256).                    */
/* ------------------------------------------------------------------ */
int oracle_run_index(const uint8_t *exponent, uint64_t n, const uint8_t len[256],
                     uint64_t total_bits, uint16_t *run_pos) {
  uint64_t chunks = (total_bits + OR_CHUNK_BITS - 1) / OR_CHUNK_BITS;
  uint64_t blocks = (chunks + OR_BLOCK_CHUNKS - 1) / OR_BLOCK_CHUNKS;
  uint64_t runs = blocks * (OR_BLOCK_CHUNKS / 2);
  uint64_t run_bits = 2 * OR_CHUNK_BITS;
  uint64_t runs_per_block = OR_BLOCK_CHUNKS / 2;
  uint64_t bit = 0, next_run = 0, block_first = 0;
  for (uint64_t i = 0; i < n; i++) {
    unsigned l = len[exponent[i]];
    if (l == 0) return OR_ERR_SYMBOL;
    /* every run boundary at or before this code's start: the codes of
       the boundary's block that started before it are i - (block's first) */
    while (next_run < runs && next_run * run_bits <= bit) {
      if (next_run % runs_per_block == 0) block_first = i;
      uint64_t before = i - block_first;
      if (before > 0xFFFFu) return OR_ERR_CORRUPT;
      run_pos[next_run] = (uint16_t)before;
      next_run++;
    }
    bit += l;
  }
  if (bit != total_bits) return OR_ERR_ARG;
  while (next_run < runs) {
    if (next_run % runs_per_block == 0) block_first = n;
    run_pos[next_run] = (uint16_t)(n - block_first);
    next_run++;
  }
  return OR_OK;
}

/* ------------------------------------------------------------------ */
/* Segment index: the stream bit at which every 64th code starts.       */
/* [Kernel] ties threads to chunks of the stream and finds output       */
/* positions by counting; this is the converse map, from an output      */
/* position to a stream position, at a fixed output step.  R13          */
/* (reading): seg[j] = sum of the code lengths of values 0..64j-1 for   */
/* j = 0..S-1, S = ceil(n/64), and seg[S] = total_bits; uint32, so the  */
/* stream must hold fewer than 2^32 bits.  Written from the code        */
/* lengths, one value at a time.  seg must hold S+1 entries.            */
/* ------------------------------------------------------------------ */
int oracle_segment_index(const uint8_t *exponent, uint64_t n, const uint8_t len[256],
                         uint64_t total_bits, uint32_t *seg) {
  uint64_t segments = (n + 63) / 64;
  uint64_t bit = 0;
  if (total_bits > 0xFFFFFFFFull) return OR_ERR_ARG;
  for (uint64_t i = 0; i < n; i++) {
    unsigned l = len[exponent[i]];
    if (l == 0) return OR_ERR_SYMBOL;
    if (i % 64 == 0) seg[i / 64] = (uint32_t)bit; /* code i starts here */
    bit += l;
  }
  if (bit != total_bits) return OR_ERR_ARG;
  seg[segments] = (uint32_t)total_bits;
  return OR_OK;
}

/* Gaps packed as 5-bit fields, most significant bit first (R8).
 * packed must hold ceil(5*C/8) zeroed bytes. */
void oracle_pack_gaps(const uint8_t *gap, uint64_t chunks, uint8_t *packed) {
  uint64_t k = 0;
  for (uint64_t c = 0; c < chunks; c++)
    for (int b = (int)OR_GAP_BITS - 1; b >= 0; b--) {
      put_bit(packed, k, (gap[c] >> b) & 1u);
      k++;
    }
}

void oracle_unpack_gaps(const uint8_t *packed, uint64_t chunks, uint8_t *gap) {
  uint64_t k = 0;
  for (uint64_t c = 0; c < chunks; c++) {
    unsigned g = 0;
    for (unsigned b = 0; b < OR_GAP_BITS; b++) {
      g = (g << 1) | get_bit(packed, k);
      k++;
    }
    gap[c] = (uint8_t)g;
  }
}

/* Canonical decoding tables: for every length, the first code, the number
 * of codes, and where its symbols start in the (length, symbol) order. */
typedef struct {
  uint64_t first[OR_MAX_CAP + 1];
  uint64_t count[OR_MAX_CAP + 1];
  uint64_t offset[OR_MAX_CAP + 1];
  int symbol[256];
} canon_tables;

static void build_canon(const uint8_t len[256], const uint32_t code[256],
                        canon_tables *t) {
  for (int l = 0; l <= OR_MAX_CAP; l++) {
    t->first[l] = 0;
    t->count[l] = 0;
    t->offset[l] = 0;
  }
  int k = 0;
  for (int l = 1; l <= OR_MAX_CAP; l++) {
    t->offset[l] = (uint64_t)k;
    int first_seen = 0;
    for (int s = 0; s < 256; s++) {
      if (len[s] != l) continue;
      if (!first_seen) {
        t->first[l] = code[s];
        first_seen = 1;
      }
      t->symbol[k++] = s;
      t->count[l]++;
    }
  }
}

/* Read one code bit by bit starting at bit p; returns its symbol and sets
 * *used to its length, or returns -1 when no code matches within 32 bits
 * or the stream ends first. */
static int read_one_code(const uint8_t *stream, uint64_t stream_bits, uint64_t p,
                         const canon_tables *t, unsigned *used) {
  uint64_t value = 0;
  for (unsigned l = 1; l <= OR_MAX_CAP; l++) {
    if (p + l - 1 >= stream_bits) return -1;
    value = (value << 1) | get_bit(stream, p + l - 1);
    if (t->count[l] > 0 && value >= t->first[l] &&
        value - t->first[l] < t->count[l]) {
      *used = l;
      return t->symbol[t->offset[l] + (value - t->first[l])];
    }
  }
  return -1;
}

/* ------------------------------------------------------------------ */
/* Step 5a: bit-serial decode from the start of the stream, n codes.   */
/* ------------------------------------------------------------------ */
int oracle_decode_serial(const uint8_t *stream, uint64_t total_bits, uint64_t n,
                         const uint8_t len[256], const uint32_t code[256],
                         uint8_t *exponent) {
  canon_tables t;
  build_canon(len, code, &t);
  uint64_t p = 0;
  for (uint64_t i = 0; i < n; i++) {
    unsigned used = 0;
    int s = read_one_code(stream, total_bits, p, &t, &used);
    if (s < 0) return OR_ERR_CORRUPT;
    exponent[i] = (uint8_t)s;
    p += used;
  }
  return p == total_bits ? OR_OK : OR_ERR_CORRUPT;
}

/* ------------------------------------------------------------------ */
/* Step 5b: decode driven by the metadata ([Kernel]): every chunk is    */
/* started at its gap and decodes the codes that start inside it (a     */
/* code that runs past the chunk end belongs to the chunk it starts in); */
/* block b writes from output index pos[b] on.  stream must hold         */
/* 8*C bytes; no code may run past total_bits.                          */
/* ------------------------------------------------------------------ */
int oracle_decode_chunked(const uint8_t *stream, const uint8_t *gap,
                          const uint32_t *pos,
                          uint64_t total_bits, uint64_t n, const uint8_t len[256],
                          const uint32_t code[256], uint8_t *exponent) {
  canon_tables t;
  build_canon(len, code, &t);
  uint64_t chunks = (total_bits + OR_CHUNK_BITS - 1) / OR_CHUNK_BITS;
  uint64_t blocks = (chunks + OR_BLOCK_CHUNKS - 1) / OR_BLOCK_CHUNKS;
  if (pos[0] != 0 || pos[blocks] != n) return OR_ERR_CORRUPT;
  for (uint64_t b = 0; b < blocks; b++) {
    uint64_t out = pos[b];
    uint64_t end_chunk = (b + 1) * OR_BLOCK_CHUNKS;
    if (end_chunk > chunks) end_chunk = chunks;
    for (uint64_t c = b * OR_BLOCK_CHUNKS; c < end_chunk; c++) {
      uint64_t chunk_start = c * OR_CHUNK_BITS;
      uint64_t limit = chunk_start + OR_CHUNK_BITS;
      if (limit > total_bits) limit = total_bits;
      if (gap[c] > 31) return OR_ERR_CORRUPT;
      uint64_t p = chunk_start + gap[c];
      while (p < limit) {
        unsigned used = 0;
        int s = read_one_code(stream, total_bits, p, &t, &used);
        if (s < 0) return OR_ERR_CORRUPT;
        if (out >= pos[b + 1]) return OR_ERR_CORRUPT;
        exponent[out++] = (uint8_t)s;
        p += used;
      }
    }
    if (out != pos[b + 1]) return OR_ERR_CORRUPT;
  }
  return OR_OK;
}

/* ======================================================================
 * rANS variant of the exponent coding (a comparison codec).  The method's
 * pages only name rANS as an alternative to Huffman; the format below is a
 * reading, written here from the definition of range ANS (Duda 2013) with
 * its usual byte-oriented renormalisation:
 *   Q1 probabilities: each exponent present with count c gets a frequency
 *      f >= 1 out of M = 4096; f = floor(c*M/n) (at least 1), then the sum is
 *      brought to M one step at a time: while below, +1 to the symbol with
 *      the largest deficit c*M - f*n (ties: smaller symbol); while above, -1
 *      to the symbol with f > 1 and the smallest deficit (ties: smaller
 *      symbol).  One symbol alone gets f = M.  cum[s] = sum of f[t], t < s.
 *   Q2 state: 32-bit, kept in [2^16, 2^32); renormalisation moves 16-bit
 *      words.  Encoding symbol s: if x >= f[s] << 20, emit the low 16 bits
 *      and shift right by 16; then x = (x / f[s]) * M + x % f[s] + cum[s].
 *      Decoding: slot = x % M, s the symbol with cum[s] <= slot < cum[s] +
 *      f[s], x = f[s] * (x / M) + slot - cum[s]; if x < 2^16, x = (x << 16)
 *      | next word.
 *   Q3 interleaving: values are grouped in units of 16384; value
 *      u*16384 + 32*k + l is coded by state l (0..31) of unit u as its k-th
 *      symbol.  Decoding runs k = 0..511 and, for each k, l = 0..31; the
 *      words are read in that order from one stream per unit.  Encoding
 *      runs the exact reverse order, each state starting at 2^16.  A unit's
 *      steps form 8 segments of 64.
 *   Q4 unit layout: the 32 final encoder states (little-endian uint32,
 *      the decoder's initial states), then 8 little-endian uint16: the
 *      index of the first word read in each segment (the first is 0), then
 *      the words in decoding order (little-endian uint16), zero-padded to a
 *      multiple of 16 bytes.  off16[u] = start of unit u in 16-byte units;
 *      off16[U] = total.
 *   Q5 integrity: after decoding a unit every state is back at 2^16 and
 *      every word has been read.
 * ====================================================================== */

#define OR_RANS_BITS 12u
#define OR_RANS_M (1u << OR_RANS_BITS)
#define OR_RANS_L (1u << 16)
#define OR_RANS_LANES 32u
#define OR_RANS_STEPS 512u
#define OR_RANS_SEG_STEPS 64u
#define OR_RANS_SEGS (OR_RANS_STEPS / OR_RANS_SEG_STEPS)
#define OR_RANS_UNIT (OR_RANS_LANES * OR_RANS_STEPS)
#define OR_RANS_HEADER (4 * OR_RANS_LANES + 2 * OR_RANS_SEGS)

int oracle_rans_freqs(const uint64_t hist[256], uint32_t freq[256]) {
  uint64_t n = 0;
  int present = 0, only = -1;
  for (int s = 0; s < 256; s++) {
    n += hist[s];
    if (hist[s]) { present++; only = s; }
  }
  for (int s = 0; s < 256; s++) freq[s] = 0;
  if (n == 0) return OR_OK;
  if (present == 1) { freq[only] = OR_RANS_M; return OR_OK; }
  int64_t sum = 0;
  for (int s = 0; s < 256; s++) {
    if (!hist[s]) continue;
    uint64_t f = hist[s] * OR_RANS_M / n;
    freq[s] = f ? (uint32_t)f : 1u;
    sum += freq[s];
  }
  while (sum != (int64_t)OR_RANS_M) {
    int pick = -1;
    int64_t best = 0;
    for (int s = 0; s < 256; s++) {
      if (!hist[s]) continue;
      int64_t d = (int64_t)(hist[s] * OR_RANS_M) - (int64_t)freq[s] * (int64_t)n;  /* deficit */
      if (sum < (int64_t)OR_RANS_M) {
        if (pick < 0 || d > best) { pick = s; best = d; }
      } else {
        if (freq[s] > 1 && (pick < 0 || d < best)) { pick = s; best = d; }
      }
    }
    if (pick < 0) return OR_ERR_ARG;
    if (sum < (int64_t)OR_RANS_M) { freq[pick]++; sum++; }
    else { freq[pick]--; sum--; }
  }
  return OR_OK;
}

static void rans_cum(const uint32_t freq[256], uint32_t cum[257]) {
  cum[0] = 0;
  for (int s = 0; s < 256; s++) cum[s + 1] = cum[s] + freq[s];
}

/* Bytes the encoded stream needs at most: per unit the header and one word
 * per value, padded. */
uint64_t oracle_rans_bound(uint64_t n) {
  uint64_t units = (n + OR_RANS_UNIT - 1) / OR_RANS_UNIT;
  return units * (OR_RANS_HEADER + 2 * OR_RANS_UNIT + 16);
}

int oracle_rans_encode(const uint8_t *exponent, uint64_t n, const uint32_t freq[256],
                       uint8_t *stream, uint64_t cap, uint32_t *off16, uint64_t *bytes) {
  uint32_t cum[257];
  rans_cum(freq, cum);
  uint64_t units = (n + OR_RANS_UNIT - 1) / OR_RANS_UNIT;
  uint16_t *words = (uint16_t *)malloc(sizeof(uint16_t) * (OR_RANS_UNIT + 1));
  if (!words) return OR_ERR_ARG;
  uint64_t at = 0;  /* bytes written so far */
  for (uint64_t u = 0; u < units; u++) {
    uint32_t x[OR_RANS_LANES];
    for (unsigned l = 0; l < OR_RANS_LANES; l++) x[l] = OR_RANS_L;
    uint64_t nw = 0;  /* words emitted, in reverse decoding order */
    uint64_t seg_words[OR_RANS_SEGS];
    for (unsigned g = 0; g < OR_RANS_SEGS; g++) seg_words[g] = 0;
    for (int k = (int)OR_RANS_STEPS - 1; k >= 0; k--) {
      for (int l = (int)OR_RANS_LANES - 1; l >= 0; l--) {
        uint64_t i = u * OR_RANS_UNIT + (uint64_t)k * OR_RANS_LANES + (uint64_t)l;
        if (i >= n) continue;
        unsigned s = exponent[i];
        uint32_t f = freq[s];
        if (f == 0) { free(words); return OR_ERR_SYMBOL; }
        if ((uint64_t)x[l] >= ((uint64_t)f << 20)) {  /* Q2: x_max = (L / M) * 2^16 * f */
          words[nw++] = (uint16_t)(x[l] & 0xFFFFu);
          x[l] >>= 16;
          seg_words[(unsigned)k / OR_RANS_SEG_STEPS]++;  /* read by the decoder at step k */
        }
        x[l] = (x[l] / f) * OR_RANS_M + x[l] % f + cum[s];
      }
    }
    uint64_t ubytes = OR_RANS_HEADER + 2 * nw;
    uint64_t padded = (ubytes + 15) / 16 * 16;
    if (at + padded > cap) { free(words); return OR_ERR_ARG; }
    off16[u] = (uint32_t)(at / 16);
    uint8_t *p = stream + at;
    for (unsigned l = 0; l < OR_RANS_LANES; l++)
      for (unsigned b = 0; b < 4; b++) p[4 * l + b] = (uint8_t)(x[l] >> (8 * b));
    uint64_t first = 0;  /* decoding index of each segment's first word */
    for (unsigned g = 0; g < OR_RANS_SEGS; g++) {
      p[4 * OR_RANS_LANES + 2 * g] = (uint8_t)(first & 0xFF);
      p[4 * OR_RANS_LANES + 2 * g + 1] = (uint8_t)(first >> 8);
      first += seg_words[g];
    }
    for (uint64_t j = 0; j < nw; j++) {  /* decoding order: last emitted first */
      uint16_t wv = words[nw - 1 - j];
      p[OR_RANS_HEADER + 2 * j] = (uint8_t)(wv & 0xFF);
      p[OR_RANS_HEADER + 2 * j + 1] = (uint8_t)(wv >> 8);
    }
    for (uint64_t j = ubytes; j < padded; j++) p[j] = 0;
    at += padded;
  }
  off16[units] = (uint32_t)(at / 16);
  *bytes = at;
  free(words);
  return OR_OK;
}

int oracle_rans_decode(const uint8_t *stream, const uint32_t *off16, uint64_t n,
                       const uint32_t freq[256], uint8_t *exponent) {
  uint32_t cum[257];
  rans_cum(freq, cum);
  uint64_t units = (n + OR_RANS_UNIT - 1) / OR_RANS_UNIT;
  for (uint64_t u = 0; u < units; u++) {
    const uint8_t *p = stream + (uint64_t)off16[u] * 16;
    uint64_t ubytes = ((uint64_t)off16[u + 1] - off16[u]) * 16;
    if (ubytes < OR_RANS_HEADER) return OR_ERR_CORRUPT;
    uint64_t nwords = (ubytes - OR_RANS_HEADER) / 2, wp = 0;
    uint32_t x[OR_RANS_LANES];
    for (unsigned l = 0; l < OR_RANS_LANES; l++)
      x[l] = (uint32_t)p[4 * l] | (uint32_t)p[4 * l + 1] << 8 | (uint32_t)p[4 * l + 2] << 16 |
             (uint32_t)p[4 * l + 3] << 24;
    for (unsigned k = 0; k < OR_RANS_STEPS; k++) {
      if (k % OR_RANS_SEG_STEPS == 0) {  /* the recorded start of the segment */
        unsigned g = k / OR_RANS_SEG_STEPS;
        uint64_t first = (uint64_t)p[4 * OR_RANS_LANES + 2 * g] |
                         (uint64_t)p[4 * OR_RANS_LANES + 2 * g + 1] << 8;
        if (first != wp) return OR_ERR_CORRUPT;
      }
      for (unsigned l = 0; l < OR_RANS_LANES; l++) {
        uint64_t i = u * OR_RANS_UNIT + (uint64_t)k * OR_RANS_LANES + l;
        if (i >= n) continue;
        uint32_t slot = x[l] % OR_RANS_M;
        int s = -1;
        for (int t = 0; t < 256; t++)
          if (freq[t] && cum[t] <= slot && slot < cum[t] + freq[t]) { s = t; break; }
        if (s < 0) return OR_ERR_CORRUPT;
        exponent[i] = (uint8_t)s;
        x[l] = freq[s] * (x[l] / OR_RANS_M) + slot - cum[s];
        if (x[l] < OR_RANS_L) {
          if (wp >= nwords) return OR_ERR_CORRUPT;
          uint32_t wv = (uint32_t)p[OR_RANS_HEADER + 2 * wp] |
                        (uint32_t)p[OR_RANS_HEADER + 2 * wp + 1] << 8;
          wp++;
          x[l] = (x[l] << 16) | wv;
        }
      }
    }
    for (unsigned l = 0; l < OR_RANS_LANES; l++)
      if (x[l] != OR_RANS_L) return OR_ERR_CORRUPT;          /* Q5 */
    for (uint64_t j = wp; j < nwords; j++)                   /* only padding may remain */
      if (p[OR_RANS_HEADER + 2 * j] || p[OR_RANS_HEADER + 2 * j + 1]) return OR_ERR_CORRUPT;
  }
  return OR_OK;
}
