/*
 * df11.h -- C ABI of the DF11 lossless BF16 weight codec for NVIDIA B200
 * (sm_100a).
 *
 * The method: the page "DFloat11: Nén suy luận GPU không mất dữ liệu, giảm LLM
 * xuống còn 70% kích thước" (vi.news.hada.io/topic?id=20542).  Citations below
 * name its sections:
 *   [Exponent] "Dư địa nén còn lại trong exponent của BFloat16"
 *   [Format]   "Định dạng DFloat11"
 *   [GPU]      "Giải nén tối ưu cho suy luận GPU"
 *   [LUT]      "Giải mã dựa trên LUT phân cấp"
 *   [Kernel]   "Kernel GPU hai giai đoạn và metadata bổ trợ"
 *   [Block]    "Giải nén theo từng transformer block"
 *
 * A BF16 weight keeps its sign and 7 mantissa bits verbatim in one byte of the
 * sign/mantissa plane; its 8-bit exponent is replaced by a canonical Huffman
 * code built from the exponent histogram and capped at 32 bits.  The codes are
 * packed into a bitstream read by the decoder in 64-bit chunks, with a 5-bit
 * gap per chunk (offset of the first code that starts in it) and one 32-bit
 * output position per block of 256 chunks.
 *
 * Format (all little-endian, byte arrays unless stated):
 *   stream         8*C bytes; code bits most significant first, stream bit k
 *                  is bit 7-(k%8) of byte k/8; zero padding after total_bits.
 *                  C = ceil(total_bits/64) chunks.
 *   gaps           ceil(5C/8) bytes; 5-bit fields, most significant bit first;
 *                  gap[c] = (first code start >= 64c, else total_bits) - 64c.
 *   block_pos      uint32[B+1], B = ceil(C/256); block_pos[b] = number of
 *                  codes starting before bit 16384*b; block_pos[B] = n.
 *   sign_mantissa  n bytes; (w >> 8 & 0x80) | (w & 0x7F).
 *   code lengths   256 bytes (the codebook; canonical codes follow, RFC 1951).
 *
 * Conventions shared by every entry point:
 *   - Pointers named d_* are device pointers; h_* and plain structs are host
 *     memory.  The library never allocates device memory: the caller owns
 *     every buffer (sizes come from df11_encoded_sizes).
 *   - Device calls are asynchronous on the caller's stream (NULL = the legacy
 *     default stream) and return a status for argument and launch errors
 *     only.  Errors found in the data (a corrupt stream, a symbol without a
 *     code) are written to the caller's device word *d_status (0 = OK; the
 *     first error wins; the caller zeroes it).
 *   - Host calls are synchronous and pure.
 *   - A matrix holds at most DF11_MAX_N values (output positions are 32-bit,
 *     [Kernel]); larger requests return DF11_ERR_TOO_LARGE.
 */
#ifndef DF11_H
#define DF11_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define DF11_CHUNK_BITS 64u        /* [Kernel]: the page's per-thread n = 8 bytes */
#define DF11_BLOCK_CHUNKS 256u     /* chunks per block of output positions      */
#define DF11_GAP_BITS 5u           /* [Kernel]: gaps in [0,31], 5 bits each      */
#define DF11_MAX_CODE_LEN 32u      /* [Kernel]/[LUT]: longest code, 32 bits      */
#define DF11_MAX_N 0xFFFFFFFFull   /* [Kernel]: 32-bit block output positions    */
#define DF11_MAX_BATCH 32u         /* matrices per decode launch (more = split)  */
#define DF11_TABLE_BITS 11u        /* reach of the decode table: codebooks whose
                                      codes are all this short decode on the
                                      fast path; longer codes (up to 32) take a
                                      length search.  The codec's default cap.  */

/* A CUDA stream (cudaStream_t), passed as an opaque pointer. */
typedef struct CUstream_st *df11_stream_t;

typedef enum {
  DF11_OK = 0,
  DF11_ERR_INVALID_ARG = 1,            /* bad pointer, size, alignment or cap  */
  DF11_ERR_TOO_LARGE = 2,              /* n > DF11_MAX_N                        */
  DF11_ERR_CUDA = 3,                   /* a CUDA launch or query failed         */
  DF11_ERR_CORRUPT = 4,                /* stream/metadata inconsistent          */
  DF11_ERR_SYMBOL_NOT_IN_CODEBOOK = 5, /* a value to encode has no code         */
  DF11_ERR_TIMEOUT = 6,                /* a bounded wait inside a kernel ran out */
  DF11_ERR_NO_DEVICE = 7,              /* no usable CUDA device                 */
  DF11_ERR_BOUNDS = 8                  /* a bounds check of the checked build
                                          (DF11_CHECKED) failed; the access was
                                          skipped.  The product build never
                                          reports it                            */
} df11_status;

/* Canonical, length-limited code for the 256 exponent values. */
typedef struct {
  uint8_t len[256];    /* code length of each exponent value, 0 = no code      */
  uint32_t code[256];  /* canonical code, right-aligned in len bits            */
  uint32_t max_len;    /* longest length (<= cap)                              */
  uint32_t min_len;    /* shortest nonzero length                              */
  uint32_t n_symbols;  /* number of values with a code                         */
  uint32_t cap;        /* the length cap the code was built under              */
} df11_codebook;

/* Byte counts for one matrix.  *_bytes: what the format stores (used for the
 * compression ratio).  *_alloc: what the device buffers must hold, padded so
 * the decoder can fetch whole blocks with 16-byte bulk copies. */
typedef struct {
  uint64_t n, total_bits, n_chunks, n_blocks;
  uint64_t stream_bytes, gaps_bytes, block_pos_bytes, sign_mantissa_bytes;
  uint64_t stored_bytes;       /* sum of the four above + 256 code lengths      */
  uint64_t stream_alloc, gaps_alloc, block_pos_alloc, sign_mantissa_alloc;
  uint64_t tables_bytes;       /* df11_build_tables output                      */
  uint64_t workspace_bytes;    /* df11_encode scratch                           */
  uint64_t run_index_bytes;    /* df11_build_run_index output (128 uint16 per
                                  block; 16-byte multiple)                      */
  uint64_t seg_index_bytes;    /* df11_build_segment_index output (uint32 per
                                  DF11_SEGMENT values, plus one; rounded up to
                                  16 bytes)                                     */
} df11_sizes;

/* One compressed matrix in device memory (non-owning).  Every pointer must be
 * 16-byte aligned and its buffer at least the *_alloc size. */
typedef struct {
  uint64_t n;                  /* number of BF16 values                         */
  uint64_t total_bits;         /* exponent code bits                            */
  const uint8_t *stream;       /* EncodedExponent ([Format])                    */
  const uint8_t *gaps;         /* packed 5-bit gaps ([Kernel])                  */
  const uint32_t *block_pos;   /* per-block output positions ([Kernel])         */
  const uint8_t *sign_mantissa;/* PackedSignMantissa ([Format])                 */
  const void *tables;          /* device copy of df11_build_tables output       */
  uint32_t min_len;            /* shortest code length (codebook.min_len)       */
  uint32_t max_block_codes;    /* most codes starting in one block of 256
                                  chunks (df11_encoded.block_max), or 0 to
                                  assume the most that min_len allows; sizes
                                  the decoder's staging (a block exceeding it
                                  is reported as corrupt)                       */
  const uint16_t *run_index;   /* optional (NULL: not used): the matrix's run
                                  index from df11_build_run_index, 16-byte
                                  aligned.  With it the decoder places every
                                  thread's outputs before decoding them       */
  const uint32_t *seg_index;   /* optional (NULL: not used): the matrix's
                                  segment index from df11_build_segment_index,
                                  4-byte aligned.  With it every decoding lane
                                  starts at a known stream bit and decodes a
                                  known number of values                       */
} df11_matrix;

/* Encoder outputs in device memory (sizes from df11_encoded_sizes). */
typedef struct {
  uint8_t *stream;
  uint8_t *gaps;
  uint32_t *block_pos;
  uint8_t *sign_mantissa;
  uint32_t *block_max;         /* optional device word (may be NULL): receives
                                  the most codes starting in any one block     */
} df11_encoded;

/* Human-readable name of a status code (static string). */
const char *df11_status_string(df11_status s);

/*
 * df11_histogram -- 256-bin histogram of the exponent field of n BF16 words.
 * [Exponent]: the codec starts from the exponent distribution of the weights.
 *   d_w       n uint16 BF16 bit patterns, 16-byte aligned.
 *   d_hist256 256 uint64 counts, overwritten.
 * Two kernel launches (clear, count).  n == 0 writes zeros.
 */
df11_status df11_histogram(const uint16_t *d_w, uint64_t n, uint64_t *d_hist256,
                           df11_stream_t stream);

/*
 * df11_build_codebook -- host.  [Format]: Huffman code from the exponent
 * histogram, frequent values short.  [LUT]/[Kernel]: lengths capped at 32.
 * Huffman with ties broken by (weight, creation order; leaves before internal
 * nodes), package-merge when the longest code exceeds cap, lengths handed to
 * symbols by (count desc, value asc), canonical codes (RFC 1951).
 *   hist256   256 counts (host).   cap  1..32.
 * Returns DF11_ERR_INVALID_ARG if cap cannot hold the alphabet.  An empty
 * histogram gives an empty codebook (n_symbols 0).
 */
df11_status df11_build_codebook(const uint64_t hist256[256], uint32_t cap,
                                df11_codebook *out);

/*
 * df11_encoded_sizes -- host.  Exact sizes of every buffer of a matrix with
 * histogram hist256 coded by cb: total_bits = sum(hist[e] * len[e]).
 * Returns DF11_ERR_SYMBOL_NOT_IN_CODEBOOK if a counted value has no code and
 * DF11_ERR_TOO_LARGE if n > DF11_MAX_N.
 */
df11_status df11_encoded_sizes(const df11_codebook *cb, const uint64_t hist256[256],
                               uint64_t n, df11_sizes *out);

/*
 * df11_sizes_from_bits -- host.  The sizes df11_encoded_sizes gives, from n
 * and total_bits alone (for a codebook built on the device: its total_bits
 * comes back from df11_build_codebook_device).  DF11_ERR_INVALID_ARG unless
 * n <= total_bits <= 32 n.
 */
df11_status df11_sizes_from_bits(uint64_t n, uint64_t total_bits, df11_sizes *out);

/*
 * df11_build_codebook_device -- S3 on the device: the codebook, its decode
 * tables and the encoded size from a device histogram, in one kernel launch
 * (one CTA), with no host round trip.  [Format], [LUT]: the same rule as
 * df11_build_codebook; the results equal, byte for byte, those of
 * df11_build_codebook + df11_build_tables + df11_encoded_sizes on the host
 * (one implementation serves both).
 *   d_hist256     256 uint64 counts (df11_histogram's output).
 *   cap           1..32 (checked on the host).
 *   d_cb          device df11_codebook, written.
 *   d_tables      df11_tables_bytes() device bytes (16-byte aligned), written.
 *   d_total_bits  device uint64: sum over e of hist[e] * len[e], written.
 *   d_status      DF11_ERR_INVALID_ARG if 2^cap is below the number of
 *                 distinct exponents (then nothing else is written).
 */
df11_status df11_build_codebook_device(const uint64_t *d_hist256, uint32_t cap,
                                       df11_codebook *d_cb, void *d_tables,
                                       uint64_t *d_total_bits, uint32_t *d_status,
                                       df11_stream_t stream);

/* Bytes of the decode tables of one codebook (a constant). */
size_t df11_tables_bytes(void);

/*
 * df11_build_tables -- host.  Decode tables for cb, written to h_tables
 * (bytes >= df11_tables_bytes()); the caller copies them to device memory and
 * points df11_matrix.tables at the copy.  [LUT]: table lookups replace the
 * bit-serial tree walk; here one 2048-entry table maps the next
 * DF11_TABLE_BITS (11) stream bits to up to four whole codes (8 bytes an
 * entry: the exponents and the start of each code), and codes longer than 11
 * bits go through a canonical length search.  The decoder checks every entry
 * before use: a table that could make it write outside its staging is
 * rejected and the matrix reported as DF11_ERR_CORRUPT.
 */
df11_status df11_build_tables(const df11_codebook *cb, void *h_tables, size_t bytes);

/*
 * df11_encode -- compress n BF16 words.  [Format] + [Kernel].
 *   d_w           n uint16, 16-byte aligned.
 *   cb            host codebook (from df11_build_codebook).
 *   total_bits    from df11_encoded_sizes (checked on the device).
 *   out           device buffers of at least the *_alloc sizes; overwritten,
 *                 padding included.
 *   d_workspace   scratch of sizes.workspace_bytes bytes (16-byte aligned).
 *   d_status      device word; DF11_ERR_SYMBOL_NOT_IN_CODEBOOK or
 *                 DF11_ERR_CORRUPT (total_bits mismatch) on data errors.
 * Three kernel launches: length sums per tile, their prefix sum, packing.
 */
df11_status df11_encode(const uint16_t *d_w, uint64_t n, const df11_codebook *cb,
                        uint64_t total_bits, const df11_encoded *out, void *d_workspace,
                        size_t workspace_bytes, uint32_t *d_status, df11_stream_t stream);

/*
 * df11_encode_device_codebook -- df11_encode with the codebook in device
 * memory (d_cb, as written by df11_build_codebook_device), for a compressor
 * that keeps every step on the device.  total_bits is the value
 * df11_build_codebook_device wrote (the caller reads it back to size the
 * buffers).  A length above 32 in d_cb is treated as 32 and a code that does
 * not fit its length is cut to it; the device check of total_bits then
 * reports DF11_ERR_CORRUPT.  Otherwise as df11_encode.
 */
df11_status df11_encode_device_codebook(const uint16_t *d_w, uint64_t n, const df11_codebook *d_cb,
                                        uint64_t total_bits, const df11_encoded *out,
                                        void *d_workspace, size_t workspace_bytes,
                                        uint32_t *d_status, df11_stream_t stream);

/*
 * df11_encode_static_ws -- df11_encode for callers that cannot allocate
 * device memory where they call the codec: for instance code running inside
 * another framework's execution callback without access to its allocator,
 * or a process that reserved all device memory up front.  The page has no
 * counterpart to this entry point; it exists for such callers only.
 * Arguments and results are those of df11_encode, without the workspace: the
 * scratch (per-tile bit offsets) lives in a fixed array in the library's own
 * device memory, which every GPU that loads the library holds (512 KiB) until
 * the process exits.  Nothing is allocated.
 *   n <= DF11_STATIC_WS_MAX_N, else DF11_ERR_TOO_LARGE (nothing launched).
 * The first call on each device looks up the array's device address (with
 * that device current); make that first call before any stream capture.  The
 * address is kept for the life of the process: resetting a device
 * (cudaDeviceReset) after that first call is not supported.
 * All calls share the one array: calls whose work overlaps on the GPU (other
 * streams, other host threads) race on it and must be serialised by the
 * caller.  Each call rewrites every entry it reads, so nothing needs clearing
 * between calls.
 */
#define DF11_STATIC_WS_MAX_N 268431360ull /* 65535 tiles of 4096 values */
df11_status df11_encode_static_ws(const uint16_t *d_w, uint64_t n, const df11_codebook *cb,
                                  uint64_t total_bits, const df11_encoded *out,
                                  uint32_t *d_status, df11_stream_t stream);

/*
 * df11_decode -- decompress one matrix into BF16.  [GPU], [Kernel].
 *   m      host struct describing device buffers.
 *   d_out  n uint16 BF16 words, 16-byte aligned; written in full.
 *   d_status  DF11_ERR_CORRUPT if a block's decoded count disagrees with its
 *          stored positions, a code is invalid or the tables are malformed;
 *          DF11_ERR_TIMEOUT if a bulk copy did not land within the kernel's
 *          bounded wait (the kernel then stops, with nothing of its own in
 *          flight).
 * Detection of corrupt data is limited to what the format lets the decoder
 * check: every block's code count against its stored positions and every
 * code against the codebook.  The format carries no checksum, so a
 * corruption of the stream or of the sign/mantissa plane that keeps those
 * counts can decode, silently, to other BF16 values.  Memory safety does not
 * depend on the data: whatever the buffers hold, the decoder reads and writes
 * only inside the allocations the format defines.
 * One kernel launch (the batch kernel with one matrix).
 */
df11_status df11_decode(const df11_matrix *m, uint16_t *d_out, uint32_t *d_status,
                        df11_stream_t stream);

/*
 * df11_decode_block_batch -- decompress several matrices (e.g. the seven of a
 * transformer block) in one launch.  [Block]: all matrices of a block are
 * decompressed as one batch just before the block's forward pass.
 *   ms      host array of count matrices, each with its own tables.
 *   d_outs  host array of count device pointers (16-byte aligned).
 * One launch per DF11_MAX_BATCH matrices.  When every matrix of a launch has
 * a run index (df11_matrix.run_index), the launch takes the indexed decoder,
 * and each thread's decoded count is also checked against the index.
 * Otherwise, when every matrix has a segment index (df11_matrix.seg_index;
 * total_bits < 2^32), it takes the segment decoder: each segment's decode
 * must end exactly where the next segment starts.  Without either index
 * every block's count is checked against its stored position.
 */
df11_status df11_decode_block_batch(const df11_matrix *ms, uint32_t count,
                                    uint16_t *const *d_outs, uint32_t *d_status,
                                    df11_stream_t stream);

/*
 * df11_build_run_index -- the run index of one matrix: for every run of two
 * consecutive chunks (chunks 2r and 2r+1 of block b, the share of one
 * decoding thread), the number of codes that start in the block before the
 * run, as uint16 at d_run_index[128 b + r]; runs past the end of the stream
 * hold their block's total.  [Kernel] stores one output position per thread
 * block; this is the same count for every pair of chunks.  It is derived from
 * the stream (not stored in the format): built once when a matrix is placed
 * on the device, it costs 2 bytes per 128 stream bits of device memory and of
 * decode traffic, and lets df11_decode place each thread's outputs before it
 * decodes them (no per-unit prefix sum, no second pass over the exponents).
 *   m            the matrix (its run_index field is ignored).
 *   d_run_index  sizes.run_index_bytes device bytes, 16-byte aligned; written.
 *   d_status     DF11_ERR_CORRUPT if a block's code count disagrees with its
 *                stored positions or a code is invalid (the index is then
 *                unusable).
 * One kernel launch.
 */
df11_status df11_build_run_index(const df11_matrix *m, uint16_t *d_run_index, uint32_t *d_status,
                                 df11_stream_t stream);

/*
 * df11_build_segment_index -- the segment index of one matrix: for every
 * segment of DF11_SEGMENT consecutive values, the stream bit at which the
 * code of its first value starts, as uint32 at d_seg_index[j] (value
 * DF11_SEGMENT * j), j < S = ceil(n / DF11_SEGMENT); d_seg_index[S] =
 * total_bits.  [Kernel] stores, per thread block, where in the output a
 * block's codes go; this is the converse map (where in the stream an output
 * position's code is) at a fixed step of outputs.  It is derived from the
 * stream (not stored in the format): built once when a matrix is placed on
 * the device, it costs 4 bytes per 64 values (0.0625 B per weight) of device
 * memory and of decode traffic, and lets df11_decode give every lane exactly
 * DF11_SEGMENT values to decode from a known stream bit: no counting pass, no
 * prefix sum and no relocation of the exponents.
 *   m            the matrix (its run_index and seg_index fields are ignored).
 *   d_seg_index  sizes.seg_index_bytes device bytes, 4-byte aligned; written.
 *   d_status     DF11_ERR_CORRUPT if a block's code count disagrees with its
 *                stored positions or a code is invalid (the index is then
 *                unusable).
 * Returns DF11_ERR_TOO_LARGE when total_bits >= 2^32 (the entries are 32-bit;
 * such a matrix decodes without this index).  One kernel launch (a memset for
 * n = 0).
 */
#define DF11_SEGMENT 64u
df11_status df11_build_segment_index(const df11_matrix *m, uint32_t *d_seg_index,
                                     uint32_t *d_status, df11_stream_t stream);

/* Activations and sums of one matrix for df11_decode_matmul_batch.  The
 * matrix W holds rows x cols values in row-major order (the order it was
 * compressed in): rows output features, cols input features. */
#define DF11_MATMUL_MAX_BATCH 8u    /* activation rows per fused launch          */
#define DF11_MATMUL_MIN_COLS 256u   /* cols: a multiple of 8, at least this      */
typedef struct {
  uint32_t rows, cols;
  const uint16_t *x;  /* device: batch x cols BF16 activations, row-major,
                         16-byte aligned                                     */
  float *y;           /* device: batch x rows FP32; the products are ADDED
                         (zero it first for y = x W^T), 4-byte aligned      */
} df11_matmul_io;

/*
 * df11_decode_matmul_batch -- for every matrix W of the batch,
 *   y[j][r] += sum_c W[r][c] * x[j][c]   (j < batch),
 * with W decoded on the fly and never written to device memory.  [GPU]: the
 * BF16 weights are decompressed right before the matmul that uses them and
 * discarded after; here the decode and the small-batch matmul are one kernel
 * (batch 1..DF11_MATMUL_MAX_BATCH, the memory-bound inference case).  The
 * format has no counterpart; this entry point adds no metadata.
 *   ms, io   host arrays of count matrices and their activations and sums
 *   batch    activation rows, 1..DF11_MATMUL_MAX_BATCH
 *   d_status as for df11_decode (corrupt metadata: DF11_ERR_CORRUPT, the
 *            offending units contribute nothing)
 * Products are accumulated in FP32: exact BF16 x BF16 products summed in an
 * unspecified order (a row is split over several CTAs and combined with
 * atomic adds), so sums may differ in the last bits from run to run.
 * Errors: DF11_ERR_INVALID_ARG for rows * cols != n, cols not a multiple of 8
 * or below DF11_MATMUL_MIN_COLS, batch out of range, misaligned pointers;
 * otherwise as df11_decode_block_batch.
 */
df11_status df11_decode_matmul_batch(const df11_matrix *ms, const df11_matmul_io *io,
                                     uint32_t count, uint32_t batch, uint32_t *d_status,
                                     df11_stream_t stream);

/*
 * df11_decode_gemm_batch -- the same product for larger batches, on the
 * tensor cores:  y[j][r] += sum_c W[r][c] * x[j][c]  (j < batch), with W
 * decoded through its segment index straight into the B operand of
 * tcgen05.mma (never written to device memory) and FP32 accumulators in
 * tensor memory.  [GPU]: decompression right before the matmul, discarded
 * after; each weight is decoded once per DF11_GEMM_MAX_BATCH activation rows.
 *   ms, io   host arrays of count matrices and their activations and sums;
 *            every matrix needs its segment index (df11_matrix.seg_index),
 *            cols a multiple of DF11_SEGMENT and total_bits < 2^32; x 16-byte
 *            and y 4-byte aligned.  Nothing else of the matrix is read but
 *            the stream, the sign/mantissa plane and the tables.
 *   batch    activation rows, >= 1; one pass per DF11_GEMM_MAX_BATCH rows
 *            (W is decoded again for each pass).
 *   d_status DF11_ERR_CORRUPT when a segment does not decode to exactly
 *            DF11_SEGMENT values ending where the next one starts (its
 *            weights then count as zero); DF11_ERR_TIMEOUT when a bounded
 *            wait inside the kernel ran out (y is then left unchanged for the
 *            tiles concerned).
 * Products are exact in FP32 and summed in FP32 in the tensor cores' order,
 * so the result agrees with an exact sum within cols * 2^-23 * sum |w x| per
 * entry (the same bound as df11_decode_matmul_batch's).
 * One launch per DF11_MAX_BATCH matrices and pass; one CTA per 128 rows of W.
 */
#define DF11_GEMM_MAX_BATCH 256u
df11_status df11_decode_gemm_batch(const df11_matrix *ms, const df11_matmul_io *io,
                                   uint32_t count, uint32_t batch, uint32_t *d_status,
                                   df11_stream_t stream);

/*
 * df11_validate -- host.  Checks stored metadata before it is trusted:
 * sizes derived from n and total_bits, every gap <= 31 and below its chunk's
 * code limit, block positions from 0 to n, non-decreasing, and no block
 * holding more codes than 256 chunks of codes of length >= min_len can start.
 *   h_gaps       packed gaps (host copy), >= ceil(5C/8) bytes.
 *   h_block_pos  B+1 positions (host copy).
 */
df11_status df11_validate(uint64_t n, uint64_t total_bits, uint32_t min_len,
                          const uint8_t *h_gaps, uint64_t gaps_bytes,
                          const uint32_t *h_block_pos, uint64_t block_pos_count);

/*
 * Serialised form of one compressed matrix (the ".df11" container).  [Format]:
 * what a DF11 model stores per weight matrix is its code lengths, the
 * exponent bitstream with its gaps and block positions, and the sign/mantissa
 * plane; this fixes a byte layout for them (the page names the parts, not a
 * file layout).  All fields little-endian:
 *   0    char[4]    "DF11"
 *   4    uint32     version (1)
 *   8    uint64     n
 *   16   uint64     total_bits
 *   24   uint32     cap (the length cap the code was built under)
 *   28   uint32     max_block_codes (0 = not recorded)
 *   32   uint32     ndim (0..4)
 *   36   uint32     0
 *   40   uint64[4]  shape (unused dimensions 0; their product is n if ndim)
 *   72   uint8[256] code lengths
 *   328  uint8[8]   0
 *   336  gaps (ceil(5C/8) bytes), then block_pos (uint32[B+1]), stream (8C
 *        bytes), sign_mantissa (n bytes) and a uint32 CRC-32 (IEEE 802.3, as
 *        zlib's crc32) of every byte before it; each of these five starts at
 *        the next multiple of 16 bytes, the gap before it zero
 * The container's checksum covers the whole matrix; the DF11 format itself
 * has none (df11_decode).
 */
#define DF11_FILE_VERSION 1u
#define DF11_FILE_HEADER_BYTES 336u

/* One matrix as host arrays (non-owning; stored sizes, no padding). */
typedef struct {
  uint64_t n, total_bits;
  uint32_t cap, max_block_codes;
  uint32_t ndim;
  uint64_t shape[4];
  const uint8_t *lengths;        /* 256 code lengths                         */
  const uint8_t *gaps;           /* df11_sizes.gaps_bytes                    */
  const uint32_t *block_pos;     /* n_blocks + 1 entries                     */
  const uint8_t *stream;         /* df11_sizes.stream_bytes                  */
  const uint8_t *sign_mantissa;  /* n bytes                                  */
} df11_host_matrix;

/* Bytes df11_write produces for a matrix of n values and total_bits code
 * bits (0 if the pair is invalid, see df11_sizes_from_bits). */
uint64_t df11_file_bytes(uint64_t n, uint64_t total_bits);

/*
 * df11_write -- host.  Serialise m into buf (buf_bytes >= df11_file_bytes).
 * DF11_ERR_INVALID_ARG for a null array, ndim > 4, a shape whose product is
 * not n, or a buffer too small; the lengths must describe a code (lengths
 * <= 32, Kraft sum <= 1).  *written receives the byte count.
 */
df11_status df11_write(const df11_host_matrix *m, void *buf, uint64_t buf_bytes,
                       uint64_t *written);

/*
 * df11_read -- host.  Parse a serialised matrix: checks the magic, version,
 * sizes (derived from n and total_bits, df11_sizes_from_bits) against
 * buf_bytes, the CRC-32, and the stored metadata (df11_validate), then points
 * out's arrays into buf (zero copy; buf must outlive them).  Returns
 * DF11_ERR_CORRUPT for a bad magic, version, size, checksum or metadata.
 */
df11_status df11_read(const void *buf, uint64_t buf_bytes, df11_host_matrix *out);

/*
 * df11_codebook_from_lengths -- host.  The codebook whose lengths are len
 * (code values canonical, RFC 1951 section 3.2.2, as df11_build_codebook
 * assigns them): what a reader rebuilds from a stored matrix.
 * DF11_ERR_INVALID_ARG if a length exceeds 32 or the lengths over-fill the
 * code space (Kraft sum > 1).
 */
df11_status df11_codebook_from_lengths(const uint8_t len[256], uint32_t cap, df11_codebook *out);

/*
 * df11_decode_host_scratch_bytes -- host.  Device scratch that
 * df11_decode_host_batch needs for these matrices: every matrix's decode
 * tables, plus three slots each as large as the largest piece needs (its
 * device arrays, run index and BF16 output; pieces as df11_decode_host_batch
 * cuts them).  Reads each matrix's code lengths and a few of its block
 * positions.  0 if a matrix's (n, total_bits) pair is invalid
 * (df11_sizes_from_bits) or the call would reject its metadata.
 */
uint64_t df11_decode_host_scratch_bytes(const df11_host_matrix *ms, uint32_t count);

/*
 * df11_decode_host_batch -- decode matrices held in HOST memory into HOST
 * memory: the [Kernel] decode with its host-to-device and device-to-host
 * copies, pipelined.  Every matrix is cut into pieces of whole decode units:
 * the call's first piece is 256 blocks of 256 chunks long at most, every
 * later one twice the one before, up to 4096 blocks (about 26 M values for
 * exponent codes of 2.6 bits); a cut is moved on by a unit where the codes
 * running over it would leave the piece fewer than codebook.min_len bits per
 * value.  Per piece: its stored arrays are copied
 * into a slot of d_scratch, its block positions are made relative to its
 * first value, its run index is built (df11_build_run_index), it is decoded
 * (df11_decode), and its BF16 bit patterns are copied to their place in
 * h_outs[i].  Each matrix's decode tables are built on the device from its
 * code lengths.  The copies in, the kernels and the copies out run on three
 * streams the call creates and releases, so both copy directions and the
 * kernels overlap from piece to piece.  The work starts after what is already
 * queued on `stream`, and `stream` waits for all of it: a synchronize of
 * `stream` makes every h_outs[i] ready.
 *
 *   ms        count host matrices (df11_host_matrix, as df11_read gives; the
 *             code lengths rebuild each codebook, df11_codebook_from_lengths)
 *   h_outs    count host buffers of n uint16 each.  Page-locked host memory
 *             (cudaHostAlloc) for ms' arrays and h_outs lets the copies run
 *             asynchronously at full PCIe speed; pageable memory works, with
 *             copies that the driver stages through its own buffers
 *   d_scratch device memory, 256-byte aligned, of at least
 *             df11_decode_host_scratch_bytes(ms, count) bytes; the call owns
 *             it until `stream` has passed the call
 *   d_status  device status word, as df11_decode
 *
 * The host checks every matrix first, and queues nothing when it fails:
 * DF11_ERR_INVALID_ARG for a null pointer, code lengths that do not form a
 * code or whose shortest code is longer than 8 bits, a max_block_codes above
 * what the shortest code allows, or too little scratch; DF11_ERR_TOO_LARGE
 * for n above DF11_MAX_N; DF11_ERR_CORRUPT when block_pos[0] is not 0,
 * block_pos[n_blocks] is not n, or the positions at a cut leave a piece an
 * impossible size.  DF11_ERR_CUDA if a stream, event, copy or launch fails
 * once queuing started (what was queued still finishes before `stream` goes
 * on).  Other data errors go to d_status, as in df11_decode.
 */
df11_status df11_decode_host_batch(const df11_host_matrix *ms, uint32_t count,
                                   uint16_t *const *h_outs, void *d_scratch,
                                   uint64_t scratch_bytes, uint32_t *d_status,
                                   df11_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* DF11_H */
