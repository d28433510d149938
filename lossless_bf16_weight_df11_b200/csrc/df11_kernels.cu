// df11_kernels.cu -- sm_100a kernels of the DF11 codec and their C-ABI
// launchers.
//
// Method: "DFloat11: Nén suy luận GPU không mất dữ liệu, giảm LLM xuống còn 70%
// kích thước" (vi.news.hada.io/topic?id=20542).  Sections cited:
//   [Exponent] "Dư địa nén còn lại trong exponent của BFloat16"
//   [Format]   "Định dạng DFloat11"
//   [GPU]      "Giải nén tối ưu cho suy luận GPU"
//   [LUT]      "Giải mã dựa trên LUT phân cấp"
//   [Kernel]   "Kernel GPU hai giai đoạn và metadata bổ trợ"
//   [Block]    "Giải nén theo từng transformer block"
//
// Kernels:
//   hist_kernel         exponent histogram, lane-private 16-bit counters in
//                       shared memory (bank = lane, no conflicts, no atomics
//                       on the hot loop)
//   enc_sum_kernel      code-length sum per 4096-value tile; clears the
//                       stream and gap buffers
//   enc_scan_kernel     exclusive prefix sum of the tile sums (bit offsets)
//   enc_pack_kernel     packs codes MSB-first, writes gaps, block positions
//                       and the sign/mantissa plane
//   decode_kernel       persistent CTAs over the (matrix, block) list of a
//                       batch; each block of 256 chunks is fetched with bulk
//                       copies (TMA, no multicast) one block ahead, decoded
//                       with a 12-bit shared-memory table, placed by a CTA
//                       prefix sum of per-chunk code counts, merged with the
//                       sign/mantissa bytes and stored as 16-byte BF16 rows
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>
#include <mutex>

#include "df11.h"
#include "df11_internal.h"

using df11i::DecodeTables;

namespace {

constexpr int kT = DF11_BLOCK_CHUNKS;  // chunks per block = threads per decode CTA
constexpr int kLutShift = 64 - df11i::kLutBits;
constexpr uint32_t kWaitLimit = 1u << 22;  // bounded mbarrier polls

__device__ __forceinline__ void set_status(uint32_t *st, uint32_t code) {
  if (st) atomicCAS(st, 0u, code);
}

__device__ __forceinline__ uint32_t bswap32(uint32_t x) { return __byte_perm(x, 0, 0x0123); }

__device__ __forceinline__ uint64_t bswap64(uint64_t x) {
  uint32_t lo = (uint32_t)x, hi = (uint32_t)(x >> 32);
  return ((uint64_t)bswap32(lo) << 32) | bswap32(hi);
}

// ============================================================ histogram

constexpr int kHistWarps = 4;
constexpr int kHistThreads = kHistWarps * 32;
constexpr size_t kHistSmem = (size_t)kHistWarps * 128 * 32 * 4;  // 64 KiB
constexpr uint32_t kHistFlushEvery = 8000;  // < 65535 / 8 increments per lane

__global__ void hist_clear_kernel(unsigned long long *hist) { hist[threadIdx.x] = 0ull; }

// Counters: lane l of warp w keeps 256 16-bit counters, two per 32-bit word;
// bins 2j, 2j+1 live in word (w*128 + j)*32 + l, so every lane hits its own
// bank.  Warps flush to the global 64-bit histogram before a counter can wrap.
__device__ __forceinline__ void hist_flush(const uint32_t *warp_base, int lane,
                                           unsigned long long *hist) {
  __syncwarp();
  for (int b = lane; b < 256; b += 32) {
    const uint32_t *row = warp_base + (b >> 1) * 32;
    const int sh = (b & 1) * 16;
    uint32_t sum = 0;
#pragma unroll 8
    for (int l = 0; l < 32; ++l) sum += (row[l] >> sh) & 0xFFFFu;
    if (sum) atomicAdd(hist + b, (unsigned long long)sum);
  }
  __syncwarp();
}

__global__ void __launch_bounds__(kHistThreads) hist_kernel(const uint16_t *__restrict__ w,
                                                             uint64_t n,
                                                             unsigned long long *__restrict__ hist) {
  extern __shared__ uint32_t hcnt[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t *warp_base = hcnt + warp * 128 * 32;
  uint32_t *mine = warp_base + lane;
  for (int j = 0; j < 128; ++j) mine[j * 32] = 0u;
  __syncwarp();
  const uint4 *wv = reinterpret_cast<const uint4 *>(w);
  const uint64_t nvec = n >> 3;
  const uint64_t warps_total = (uint64_t)gridDim.x * kHistWarps;
  const uint64_t gwarp = (uint64_t)blockIdx.x * kHistWarps + warp;
  auto add2 = [&](uint32_t v) {
    uint32_t e0 = (v >> 7) & 0xFFu, e1 = (v >> 23) & 0xFFu;
    mine[(e0 >> 1) * 32] += 1u << ((e0 & 1u) * 16);
    mine[(e1 >> 1) * 32] += 1u << ((e1 & 1u) * 16);
  };
  uint32_t since = 0;
  // warp-uniform loop: each step a warp reads 4 x 32 consecutive 16-byte vectors
  for (uint64_t base = gwarp * 128; base < nvec; base += warps_total * 128) {
    uint4 q[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      uint64_t i = base + u * 32 + lane;
      q[u] = i < nvec ? __ldg(wv + i) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      uint64_t i = base + u * 32 + lane;
      if (i < nvec) {
        add2(q[u].x);
        add2(q[u].y);
        add2(q[u].z);
        add2(q[u].w);
      }
    }
    since += 4;
    if (since >= kHistFlushEvery) {
      hist_flush(warp_base, lane, hist);
      for (int j = 0; j < 128; ++j) mine[j * 32] = 0u;
      __syncwarp();
      since = 0;
    }
  }
  hist_flush(warp_base, lane, hist);
  // the n % 8 values after the last whole vector
  if (blockIdx.x == 0 && threadIdx.x < (n & 7)) {
    uint32_t v = w[(nvec << 3) + threadIdx.x];
    atomicAdd(hist + ((v >> 7) & 0xFFu), 1ull);
  }
}

// ============================================================ encode

struct EncCodebook {
  uint32_t code[256];
  uint8_t len[256];
};

__device__ __forceinline__ void load_tile_values(const uint16_t *__restrict__ w, uint64_t n,
                                                 uint64_t i0, uint16_t v[16]) {
  if (i0 + 16 <= n) {
    const uint4 *p = reinterpret_cast<const uint4 *>(w + i0);
    uint4 a = __ldg(p), b = __ldg(p + 1);
    uint32_t words[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      v[2 * k] = (uint16_t)(words[k] & 0xFFFFu);
      v[2 * k + 1] = (uint16_t)(words[k] >> 16);
    }
  } else {
#pragma unroll
    for (int k = 0; k < 16; ++k) v[k] = (i0 + k < n) ? w[i0 + k] : (uint16_t)0;
  }
}

// Sum of code lengths of each tile of kEncTile values; also clears the
// stream and gap buffers (their padding must read as zero bits).
__global__ void __launch_bounds__(df11i::kEncThreads) enc_sum_kernel(
    const uint16_t *__restrict__ w, uint64_t n, EncCodebook cb, uint64_t *__restrict__ tile_sum,
    uint64_t n_tiles, uint4 *__restrict__ stream, uint64_t stream_vecs, uint4 *__restrict__ gaps,
    uint64_t gap_vecs, uint32_t *status) {
  __shared__ uint8_t s_len[256];
  __shared__ uint32_t s_warp[df11i::kEncThreads / 32];
  const int t = threadIdx.x;
  s_len[t] = cb.len[t];
  const uint64_t gtid = (uint64_t)blockIdx.x * blockDim.x + t;
  const uint64_t gstride = (uint64_t)gridDim.x * blockDim.x;
  for (uint64_t i = gtid; i < stream_vecs; i += gstride) stream[i] = make_uint4(0, 0, 0, 0);
  for (uint64_t i = gtid; i < gap_vecs; i += gstride) gaps[i] = make_uint4(0, 0, 0, 0);
  __syncthreads();
  const uint64_t tile = blockIdx.x;
  if (tile >= n_tiles) return;
  uint16_t v[16];
  const uint64_t i0 = tile * df11i::kEncTile + (uint64_t)t * df11i::kEncPerThread;
  load_tile_values(w, n, i0, v);
  uint32_t sum = 0;
  bool missing = false;
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    if (i0 + k < n) {
      uint32_t l = s_len[(v[k] >> 7) & 0xFFu];
      missing |= (l == 0);
      sum += l;
    }
  }
  if (missing) set_status(status, DF11_ERR_SYMBOL_NOT_IN_CODEBOOK);
#pragma unroll
  for (int d = 16; d > 0; d >>= 1) sum += __shfl_down_sync(0xffffffffu, sum, d);
  if ((t & 31) == 0) s_warp[t >> 5] = sum;
  __syncthreads();
  if (t == 0) {
    uint64_t tot = 0;
    for (int i = 0; i < df11i::kEncThreads / 32; ++i) tot += s_warp[i];
    tile_sum[tile] = tot;
  }
}

// Exclusive prefix sum of the tile sums, in place, by one CTA; the grand
// total lands in tile_sum[n_tiles] and must equal total_bits.
constexpr int kScanThreads = 1024;
__global__ void __launch_bounds__(kScanThreads) enc_scan_kernel(
    uint64_t *__restrict__ tile_sum, uint64_t n_tiles, uint64_t total_bits, uint32_t *block_pos,
    uint64_t n_blocks, uint64_t n, uint32_t *status) {
  __shared__ uint64_t s_warp[kScanThreads / 32];
  __shared__ uint64_t s_total;
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  uint64_t carry = 0;
  for (uint64_t base = 0; base < n_tiles; base += 4 * kScanThreads) {
    uint64_t v[4], s = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      uint64_t idx = base + 4 * (uint64_t)t + j;
      v[j] = idx < n_tiles ? tile_sum[idx] : 0ull;
      s += v[j];
    }
    uint64_t incl = s;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      uint64_t o = __shfl_up_sync(0xffffffffu, incl, d);
      if (lane >= d) incl += o;
    }
    if (lane == 31) s_warp[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      uint64_t x = s_warp[lane];
      uint64_t xi = x;
#pragma unroll
      for (int d = 1; d < 32; d <<= 1) {
        uint64_t o = __shfl_up_sync(0xffffffffu, xi, d);
        if (lane >= d) xi += o;
      }
      s_warp[lane] = xi - x;
      if (lane == 31) s_total = xi;
    }
    __syncthreads();
    uint64_t run = carry + s_warp[warp] + incl - s;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      uint64_t idx = base + 4 * (uint64_t)t + j;
      if (idx < n_tiles) tile_sum[idx] = run;
      run += v[j];
    }
    carry += s_total;
    __syncthreads();
  }
  if (t == 0) {
    tile_sum[n_tiles] = carry;
    if (carry != total_bits) set_status(status, DF11_ERR_CORRUPT);
    block_pos[n_blocks] = (uint32_t)n;
  }
}

// Pack the codes of one tile.  Codes are OR-ed into a shared big-endian bit
// buffer covering the tile's bit range, then written out as 32-bit words
// (byte-swapped to the MSB-first byte order); the two edge words are shared
// with the neighbouring tiles and are OR-ed atomically into the cleared
// stream.  The thread that owns the first code starting in a chunk writes
// that chunk's 5-bit gap; the one that owns the first code starting in a
// block of 256 chunks writes the block's output position.
__global__ void __launch_bounds__(df11i::kEncThreads) enc_pack_kernel(
    const uint16_t *__restrict__ w, uint64_t n, EncCodebook cb,
    const uint64_t *__restrict__ tile_start, uint64_t total_bits, uint8_t *__restrict__ stream,
    uint64_t stream_alloc, uint8_t *__restrict__ gaps, uint64_t gaps_alloc,
    uint32_t *__restrict__ block_pos, uint64_t n_blocks, uint8_t *__restrict__ sign_mantissa) {
  constexpr int kWords = df11i::kEncTile * DF11_MAX_CODE_LEN / 32 + 2;
  __shared__ uint32_t s_bits[kWords];
  __shared__ uint32_t s_code[256];
  __shared__ uint8_t s_len[256];
  __shared__ uint32_t s_warp[df11i::kEncThreads / 32];
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  s_code[t] = cb.code[t];
  s_len[t] = cb.len[t];
  const uint64_t tile = blockIdx.x;
  const uint64_t S = tile_start[tile], E = tile_start[tile + 1];
  const uint64_t S0 = S & ~31ull;
  const uint32_t nwords = (uint32_t)((E - S0 + 31) >> 5);
  for (uint32_t k = t; k < nwords + 1 && k < (uint32_t)kWords; k += df11i::kEncThreads) s_bits[k] = 0u;
  __syncthreads();

  uint16_t v[16];
  const uint64_t i0 = tile * df11i::kEncTile + (uint64_t)t * df11i::kEncPerThread;
  load_tile_values(w, n, i0, v);
  uint32_t lens[16];
  uint32_t sum = 0;
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    lens[k] = (i0 + k < n) ? s_len[(v[k] >> 7) & 0xFFu] : 0u;
    sum += lens[k];
  }
  uint32_t incl = sum;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    uint32_t o = __shfl_up_sync(0xffffffffu, incl, d);
    if (lane >= d) incl += o;
  }
  if (lane == 31) s_warp[warp] = incl;
  __syncthreads();
  uint32_t wpre = 0;
  for (int i = 0; i < warp; ++i) wpre += s_warp[i];
  uint32_t rel = (uint32_t)(S - S0) + wpre + incl - sum;  // bit offset in s_bits
  uint64_t start = S + wpre + incl - sum;                 // absolute bit offset
  // length of the value before this thread's first one
  uint32_t prev_len = 0;
  if (i0 > 0 && i0 < n) prev_len = s_len[(w[i0 - 1] >> 7) & 0xFFu];
  const uint64_t C = (total_bits + 63) >> 6;
  uint32_t *gaps32 = reinterpret_cast<uint32_t *>(gaps);
  const uint64_t gap_words = gaps_alloc >> 2;
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    const uint64_t i = i0 + k;
    if (i >= n) break;
    const uint32_t L = lens[k];
    if (L == 0) continue;
    const uint32_t code = s_code[(v[k] >> 7) & 0xFFu];
    // code bits [rel, rel+L) of the big-endian buffer
    const uint32_t wi = rel >> 5, off = rel & 31u;
    const uint64_t placed = ((uint64_t)code << (64 - L)) >> off;
    if (wi < (uint32_t)kWords) atomicOr(&s_bits[wi], (uint32_t)(placed >> 32));
    if ((uint32_t)placed && wi + 1 < (uint32_t)kWords) atomicOr(&s_bits[wi + 1], (uint32_t)placed);
    const uint64_t prev = start - prev_len;
    if (i == 0 || (prev >> 6) != (start >> 6)) {
      // first code starting in chunk start/64 -> gap
      const uint64_t c = start >> 6;
      const uint32_t g = (uint32_t)(start & 63u);
      const uint64_t q = 5 * c;
      const uint64_t gw = q >> 5;
      const uint64_t y = (uint64_t)g << (59 - (uint32_t)(q & 31u));
      if (gw < gap_words) atomicOr(&gaps32[gw], bswap32((uint32_t)(y >> 32)));
      if ((uint32_t)y && gw + 1 < gap_words) atomicOr(&gaps32[gw + 1], bswap32((uint32_t)y));
    }
    if (i == 0 || (prev >> 14) != (start >> 14)) {
      const uint64_t b = start >> 14;
      if (b < n_blocks) block_pos[b] = (uint32_t)i;
    }
    if (i + 1 == n) {
      // the last chunk / block may begin inside the final code
      if (C > 0 && (start >> 6) < C - 1) {
        const uint64_t c = C - 1;
        const uint32_t g = (uint32_t)(total_bits - 64 * c);
        const uint64_t q = 5 * c;
        const uint64_t gw = q >> 5;
        const uint64_t y = (uint64_t)g << (59 - (uint32_t)(q & 31u));
        if (gw < gap_words) atomicOr(&gaps32[gw], bswap32((uint32_t)(y >> 32)));
        if ((uint32_t)y && gw + 1 < gap_words) atomicOr(&gaps32[gw + 1], bswap32((uint32_t)y));
      }
      if (n_blocks > 0 && (start >> 14) < n_blocks - 1) block_pos[n_blocks - 1] = (uint32_t)n;
    }
    prev_len = L;
    rel += L;
    start += L;
  }
  // sign/mantissa plane ([Format]: kept verbatim, one byte per value)
  if (i0 + 16 <= n) {
    uint32_t pk[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint32_t x = 0;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        uint32_t wv = v[4 * q + j];
        x |= (((wv >> 8) & 0x80u) | (wv & 0x7Fu)) << (8 * j);
      }
      pk[q] = x;
    }
    *reinterpret_cast<uint4 *>(sign_mantissa + i0) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
  } else {
    for (int k = 0; k < 16 && i0 + k < n; ++k)
      sign_mantissa[i0 + k] = (uint8_t)(((v[k] >> 8) & 0x80u) | (v[k] & 0x7Fu));
  }
  __syncthreads();
  uint32_t *stream32 = reinterpret_cast<uint32_t *>(stream);
  const uint64_t g0 = S0 >> 5;
  const uint64_t stream_words = stream_alloc >> 2;
  for (uint32_t k = t; k < nwords && k < (uint32_t)kWords; k += df11i::kEncThreads) {
    const uint64_t gw = g0 + k;
    if (gw >= stream_words) break;
    const uint32_t val = bswap32(s_bits[k]);
    if (k == 0 || k + 1 == nwords) atomicOr(&stream32[gw], val);
    else stream32[gw] = val;
  }
}

// ============================================================ decode

struct DecMat {
  const uint8_t *stream;
  const uint8_t *gaps;
  const uint32_t *pos;
  const uint8_t *sm;
  const DecodeTables *tables;
  uint16_t *out;
  uint64_t n;
  uint64_t total_bits;
  uint64_t n_chunks;
};

struct DecParams {
  DecMat m[DF11_MAX_BATCH];
  uint64_t block_start[DF11_MAX_BATCH + 1];  // prefix sums of blocks per matrix
  uint32_t count;
  uint32_t stage_cap;  // bytes: max codes per block rounded up to 16
  uint32_t *status;
};

constexpr uint32_t kStreamStage = 8 * kT + 16;         // a block of chunks + the next one
constexpr uint32_t kGapStage = DF11_GAP_BITS * kT / 8;  // 160 B
constexpr uint32_t kGapStagePad = kGapStage + 16;

struct StageLayout {
  uint32_t stream, gaps, sm, size;
};

__host__ __device__ inline StageLayout stage_layout(uint32_t cap) {
  StageLayout L;
  L.stream = 0;
  L.gaps = kStreamStage;
  L.sm = L.gaps + kGapStagePad;
  L.size = L.sm + cap + 32;
  return L;
}

struct SmemLayout {
  uint32_t tables, stage0, stage1, staging, bars, meta, warp, total;
};

__host__ __device__ inline SmemLayout smem_layout(uint32_t cap) {
  SmemLayout S;
  StageLayout L = stage_layout(cap);
  S.tables = 0;
  S.stage0 = (uint32_t)sizeof(DecodeTables);
  S.stage1 = S.stage0 + L.size;
  S.staging = S.stage1 + L.size;
  S.bars = S.staging + cap + 16;
  S.meta = S.bars + 16;
  S.warp = S.meta + 2 * 16;
  S.total = S.warp + 16 * 4;
  return S;
}

__device__ __forceinline__ uint32_t smem_addr(const void *p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count));
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
               "r"(bytes)
               : "memory");
}

// Bulk copy global -> shared (TMA, CTA-local, no multicast).  Both addresses
// 16-byte aligned, size a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_addr(dst)),
      "l"(src), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}

__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t phase) {
  const uint32_t a = smem_addr(bar);
  for (uint32_t it = 0; it < kWaitLimit; ++it) {
    uint32_t done;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, "
        "p;\n}\n"
        : "=r"(done)
        : "r"(a), "r"(phase)
        : "memory");
    if (done) return true;
  }
  return false;
}

// Stream bits [p, p+64) of the 128-bit pair (hi, lo), p in [0, 63].
__device__ __forceinline__ uint64_t window64(uint64_t hi, uint64_t lo, uint32_t p) {
  return (hi << p) | ((lo >> 1) >> (63 - p));
}

// Length of a code longer than the table's reach: the smallest L with
// window < limit[L] (canonical codes are ordered by length when
// left-justified); 0 if none (invalid code).
__device__ __forceinline__ uint32_t long_code_len(uint32_t w32, const DecodeTables &tab) {
  const uint32_t maxl = min(tab.max_len, (uint32_t)DF11_MAX_CODE_LEN);
  for (uint32_t L = df11i::kLutBits + 1; L <= maxl; ++L)
    if ((uint64_t)w32 < tab.limit[L]) return L;
  return 0;
}

// Codes of one chunk: those that start in [p, lim).  WRITE = false counts
// them; WRITE = true also stores their exponents to dst[0..count).
template <bool WRITE>
__device__ __forceinline__ uint32_t chunk_codes(uint64_t hi, uint64_t lo, uint32_t p, uint32_t lim,
                                                const DecodeTables &tab, uint8_t *dst, bool &bad) {
  uint32_t cnt = 0;
  while (p < lim) {
    const uint64_t w = window64(hi, lo, p);
    const uint32_t e = tab.lut[(uint32_t)(w >> kLutShift)];
    const uint32_t used = e & 0xFu, ns = (e >> 4) & 0x3u;
    if (used == 0) {  // first code longer than the table's reach (or invalid)
      const uint32_t w32 = (uint32_t)(w >> 32);
      const uint32_t L = long_code_len(w32, tab);
      if (L == 0) {
        bad = true;
        break;
      }
      if (WRITE) dst[cnt] = tab.sym[((w32 >> (32 - L)) + tab.base[L]) & 0xFFu];
      ++cnt;
      p += L;
      continue;
    }
    if (p + used <= lim) {
      if (WRITE) {
        dst[cnt] = (uint8_t)(e >> 8);
        if (ns > 1) dst[cnt + 1] = (uint8_t)(e >> 16);
        if (ns > 2) dst[cnt + 2] = (uint8_t)(e >> 24);
      }
      cnt += ns;
      p += used;
      continue;
    }
    // the entry runs past the limit: keep the codes that start before it
    if (WRITE) dst[cnt] = (uint8_t)(e >> 8);
    ++cnt;
    uint32_t q = p + tab.codelen[(e >> 8) & 0xFFu];
    if (ns > 1 && q < lim) {
      if (WRITE) dst[cnt] = (uint8_t)(e >> 16);
      ++cnt;
      q += tab.codelen[(e >> 16) & 0xFFu];
      if (ns > 2 && q < lim) {
        if (WRITE) dst[cnt] = (uint8_t)(e >> 24);
        ++cnt;
      }
    }
    break;
  }
  return cnt;
}

// 4 exponents + 4 sign/mantissa bytes -> 4 BF16 words (two 32-bit halves).
__device__ __forceinline__ void merge4(uint32_t e4, uint32_t s4, uint32_t &w01, uint32_t &w23) {
  const uint32_t hi4 = (s4 & 0x80808080u) | ((e4 >> 1) & 0x7F7F7F7Fu);
  const uint32_t lo4 = (s4 & 0x7F7F7F7Fu) | ((e4 << 7) & 0x80808080u);
  w01 = __byte_perm(lo4, hi4, 0x5140);
  w23 = __byte_perm(lo4, hi4, 0x7362);
}

struct BlockRef {
  uint32_t m;
  uint64_t b;
};

__device__ __forceinline__ BlockRef locate(const DecParams &P, uint64_t g, uint32_t hint) {
  uint32_t m = hint;
  while (m + 1 < P.count && g >= P.block_start[m + 1]) ++m;
  return BlockRef{m, g - P.block_start[m]};
}

__global__ void __launch_bounds__(kT, 3) decode_kernel(const __grid_constant__ DecParams P) {
  extern __shared__ __align__(128) uint8_t smem[];
  const uint32_t cap = P.stage_cap;
  const SmemLayout S = smem_layout(cap);
  const StageLayout L = stage_layout(cap);
  DecodeTables &tab = *reinterpret_cast<DecodeTables *>(smem + S.tables);
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + S.bars);
  uint32_t *meta = reinterpret_cast<uint32_t *>(smem + S.meta);  // [stage][P0, P1, m, -]
  uint32_t *warp_tot = reinterpret_cast<uint32_t *>(smem + S.warp);
  uint8_t *staging = smem + S.staging;
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;

  const uint64_t total = P.block_start[P.count];
  const uint64_t g0 = (uint64_t)blockIdx.x * total / gridDim.x;
  const uint64_t g1 = (uint64_t)(blockIdx.x + 1) * total / gridDim.x;
  if (g0 >= g1) return;

  // thread 0 fetches the block after next's positions one iteration early
  uint32_t nxt_p0 = 0, nxt_p1 = 0, nxt_m = 0;
  uint32_t hint = 0;
  auto issue = [&](uint64_t g, uint32_t stage, uint32_t p0, uint32_t p1, uint32_t m) {
    const DecMat &M = P.m[m];
    const uint64_t b = g - P.block_start[m];
    uint8_t *st = smem + (stage ? S.stage1 : S.stage0);
    // positions are trusted only as far as they stay inside the matrix and
    // the stage; anything else is flagged as corrupt after the count
    const bool sane = p1 >= p0 && p1 <= M.n && p1 - p0 <= P.stage_cap;
    const uint32_t sm_lo = p0 & ~15u;
    const uint32_t sm_bytes = sane ? (uint32_t)((((uint64_t)p1 + 15u) & ~15ull) - sm_lo) : 0u;
    meta[stage * 4 + 0] = p0;
    meta[stage * 4 + 1] = p1;
    meta[stage * 4 + 2] = m;
    meta[stage * 4 + 3] = (uint32_t)b;
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    mbar_expect_tx(&bars[stage], kStreamStage + kGapStage + sm_bytes);
    bulk_g2s(st + L.stream, M.stream + b * (8 * kT), kStreamStage, &bars[stage]);
    bulk_g2s(st + L.gaps, M.gaps + b * kGapStage, kGapStage, &bars[stage]);
    if (sm_bytes) bulk_g2s(st + L.sm, M.sm + sm_lo, sm_bytes, &bars[stage]);
  };
  auto fetch_pos = [&](uint64_t g) {
    BlockRef r = locate(P, g, hint);
    hint = r.m;
    nxt_m = r.m;
    nxt_p0 = __ldg(P.m[r.m].pos + r.b);
    nxt_p1 = __ldg(P.m[r.m].pos + r.b + 1);
  };

  if (t == 0) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    fetch_pos(g0);
    issue(g0, 0, nxt_p0, nxt_p1, nxt_m);
    if (g0 + 1 < g1) fetch_pos(g0 + 1);
  }
  __syncthreads();

  uint32_t cur_m = 0xFFFFFFFFu;
  for (uint64_t g = g0, it = 0; g < g1; ++g, ++it) {
    const uint32_t s = (uint32_t)(it & 1);
    const bool ok_wait = mbar_wait(&bars[s], (uint32_t)((it >> 1) & 1));
    if (__syncthreads_or(!ok_wait)) {
      // the only copy in flight is the one just waited for (the next block's
      // copy is issued after this wait), so the CTA can leave
      if (t == 0) set_status(P.status, DF11_ERR_TIMEOUT);
      return;
    }
    if (t == 0 && g + 1 < g1) {
      issue(g + 1, s ^ 1, nxt_p0, nxt_p1, nxt_m);
      if (g + 2 < g1) fetch_pos(g + 2);
    }
    const uint32_t *mt = meta + s * 4;
    const uint32_t P0 = mt[0], P1 = mt[1], m = mt[2];
    const uint64_t b = mt[3];
    if (m != cur_m) {
      // new matrix: its decode tables into shared memory
      const uint4 *src = reinterpret_cast<const uint4 *>(P.m[m].tables);
      uint4 *dst = reinterpret_cast<uint4 *>(&tab);
      for (uint32_t k = t; k < sizeof(DecodeTables) / 16; k += kT) dst[k] = __ldg(src + k);
      cur_m = m;
      __syncthreads();
    }
    const DecMat &M = P.m[m];
    const uint8_t *st = smem + (s ? S.stage1 : S.stage0);

    // ---- this thread's chunk
    const uint64_t c = b * kT + t;
    uint64_t hi = 0, lo = 0;
    uint32_t p = 0, lim = 0;
    if (c < M.n_chunks) {
      const uint64_t *s64 = reinterpret_cast<const uint64_t *>(st + L.stream);
      hi = bswap64(s64[t]);
      lo = bswap64(s64[t + 1]);
      const uint64_t rem = M.total_bits - c * 64;
      lim = rem < 64 ? (uint32_t)rem : 64u;
      const uint8_t *gp = st + L.gaps;
      const uint32_t q = 5u * t;
      const uint32_t two = ((uint32_t)gp[q >> 3] << 8) | gp[(q >> 3) + 1];
      p = (two >> (11 - (q & 7u))) & 31u;
    }
    // ---- phase 1: count the codes that start in the chunk
    bool bad = false;
    const uint32_t cnt = chunk_codes<false>(hi, lo, p, lim, tab, nullptr, bad);
    // ---- CTA prefix sum of the counts
    uint32_t incl = cnt;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const uint32_t o = __shfl_up_sync(0xffffffffu, incl, d);
      if (lane >= d) incl += o;
    }
    const bool warp_bad = __any_sync(0xffffffffu, bad);
    if (lane == 31) warp_tot[warp] = incl | (warp_bad ? 0x80000000u : 0u);
    __syncthreads();
    uint32_t wpre = 0, tot = 0;
    bool any_bad = false;
#pragma unroll
    for (int i = 0; i < kT / 32; ++i) {
      const uint32_t x = warp_tot[i];
      any_bad |= (x >> 31) != 0;
      const uint32_t v = x & 0x7FFFFFFFu;
      tot += v;
      if (i < warp) wpre += v;
    }
    const bool ok = !any_bad && P1 >= P0 && P1 <= M.n && tot == P1 - P0 && tot <= cap;
    if (!ok && t == 0) set_status(P.status, DF11_ERR_CORRUPT);
    // ---- phase 2: decode into the staging row at this thread's offset
    if (ok) chunk_codes<true>(hi, lo, p, lim, tab, staging + (P0 & 7u) + wpre + incl - cnt, bad);
    __syncthreads();
    // ---- merge with the sign/mantissa bytes; 16-byte BF16 stores
    if (ok) {
      const uint32_t base8 = P0 & ~7u;
      const uint32_t sm_lo = P0 & ~15u;
      const uint32_t ng = (P1 - base8 + 7) >> 3;
      const uint8_t *smst = st + L.sm;
      uint16_t *out = M.out;
      for (uint32_t k = t; k < ng; k += kT) {
        const uint64_t o = (uint64_t)base8 + 8ull * k;
        const uint2 e8 = *reinterpret_cast<const uint2 *>(staging + 8 * k);
        const uint2 s8 = *reinterpret_cast<const uint2 *>(smst + (uint32_t)(o - sm_lo));
        uint4 r;
        merge4(e8.x, s8.x, r.x, r.y);
        merge4(e8.y, s8.y, r.z, r.w);
        if (o >= P0 && o + 8 <= P1) {
          *reinterpret_cast<uint4 *>(out + o) = r;
        } else {
          const uint32_t wv[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const uint64_t oj = o + j;
            if (oj >= P0 && oj < P1) out[oj] = (uint16_t)(wv[j >> 1] >> (16 * (j & 1)));
          }
        }
      }
    }
  }
}

// ============================================================ launch helpers

struct DeviceInfo {
  int sms = 0;
  bool configured = false;
};

std::mutex g_mu;
DeviceInfo g_dev[64];

df11_status device_info(int *dev, int *sms) {
  if (cudaGetDevice(dev) != cudaSuccess) {
    cudaGetLastError();
    return DF11_ERR_NO_DEVICE;
  }
  if (*dev < 0 || *dev >= 64) return DF11_ERR_NO_DEVICE;
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceInfo &d = g_dev[*dev];
  if (!d.configured) {
    if (cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, *dev) != cudaSuccess)
      return DF11_ERR_CUDA;
    if (cudaFuncSetAttribute(hist_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kHistSmem) != cudaSuccess)
      return DF11_ERR_CUDA;
    if (cudaFuncSetAttribute(decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem_layout(16384 + 16).total) != cudaSuccess)
      return DF11_ERR_CUDA;
    d.configured = true;
  }
  *sms = d.sms;
  return DF11_OK;
}

inline bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }
inline uint64_t cdiv(uint64_t a, uint64_t b) { return (a + b - 1) / b; }

df11_status launch_status() {
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? DF11_OK : DF11_ERR_CUDA;
}

}  // namespace

// ============================================================ C ABI

extern "C" df11_status df11_histogram(const uint16_t *d_w, uint64_t n, uint64_t *d_hist256,
                                      df11_stream_t stream) {
  if (!d_hist256 || (n && !d_w) || (n && !aligned16(d_w))) return DF11_ERR_INVALID_ARG;
  int dev, sms;
  df11_status st = device_info(&dev, &sms);
  if (st != DF11_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  auto *h = reinterpret_cast<unsigned long long *>(d_hist256);
  hist_clear_kernel<<<1, 256, 0, s>>>(h);
  if (n) {
    const uint64_t vec_warps = cdiv(n >> 3, 128);
    uint64_t grid = (uint64_t)sms * 3;
    grid = vec_warps ? std::min<uint64_t>(grid, cdiv(vec_warps, kHistWarps)) : 1;
    if (grid < 1) grid = 1;
    hist_kernel<<<(unsigned)grid, kHistThreads, kHistSmem, s>>>(d_w, n, h);
  }
  return launch_status();
}

extern "C" df11_status df11_encode(const uint16_t *d_w, uint64_t n, const df11_codebook *cb,
                                   uint64_t total_bits, const df11_encoded *out, void *d_workspace,
                                   size_t workspace_bytes, uint32_t *d_status,
                                   df11_stream_t stream) {
  if (!cb || !out || !d_status) return DF11_ERR_INVALID_ARG;
  if (n > DF11_MAX_N) return DF11_ERR_TOO_LARGE;
  if ((n && (!d_w || !aligned16(d_w))) || !out->stream || !out->gaps || !out->block_pos ||
      !out->sign_mantissa || !d_workspace)
    return DF11_ERR_INVALID_ARG;
  if (!aligned16(out->stream) || !aligned16(out->gaps) || !aligned16(out->block_pos) ||
      !aligned16(out->sign_mantissa) || !aligned16(d_workspace))
    return DF11_ERR_INVALID_ARG;
  if (total_bits > n * (uint64_t)DF11_MAX_CODE_LEN || (n && total_bits < n))
    return DF11_ERR_INVALID_ARG;
  const uint64_t n_tiles = cdiv(n, df11i::kEncTile);
  if (workspace_bytes < 8 * (n_tiles + 1)) return DF11_ERR_INVALID_ARG;
  int dev, sms;
  df11_status st = device_info(&dev, &sms);
  if (st != DF11_OK) return st;
  EncCodebook ecb;
  for (int i = 0; i < 256; ++i) {
    ecb.code[i] = cb->code[i];
    ecb.len[i] = cb->len[i];
  }
  const uint64_t C = cdiv(total_bits, 64);
  const uint64_t B = cdiv(C, kT);
  const uint64_t stream_alloc = 8 * kT * B + 16;
  const uint64_t gaps_alloc = kGapStage * B + 16;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  auto *ws = reinterpret_cast<uint64_t *>(d_workspace);
  const uint64_t grid1 = std::max<uint64_t>(n_tiles, 1);
  enc_sum_kernel<<<(unsigned)grid1, df11i::kEncThreads, 0, s>>>(
      d_w, n, ecb, ws, n_tiles, reinterpret_cast<uint4 *>(out->stream), stream_alloc / 16,
      reinterpret_cast<uint4 *>(out->gaps), gaps_alloc / 16, d_status);
  enc_scan_kernel<<<1, kScanThreads, 0, s>>>(ws, n_tiles, total_bits, out->block_pos, B, n,
                                            d_status);
  if (n_tiles)
    enc_pack_kernel<<<(unsigned)n_tiles, df11i::kEncThreads, 0, s>>>(
        d_w, n, ecb, ws, total_bits, out->stream, stream_alloc, out->gaps, gaps_alloc,
        out->block_pos, B, out->sign_mantissa);
  return launch_status();
}

extern "C" df11_status df11_decode_block_batch(const df11_matrix *ms, uint32_t count,
                                               uint16_t *const *d_outs, uint32_t *d_status,
                                               df11_stream_t stream) {
  if (count == 0) return DF11_OK;
  if (!ms || !d_outs) return DF11_ERR_INVALID_ARG;
  int dev, sms;
  df11_status st = device_info(&dev, &sms);
  if (st != DF11_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  for (uint32_t first = 0; first < count; first += DF11_MAX_BATCH) {
    const uint32_t k = std::min<uint32_t>(DF11_MAX_BATCH, count - first);
    DecParams P;
    P.count = 0;
    P.status = d_status;
    P.block_start[0] = 0;
    uint32_t min_len = DF11_MAX_CODE_LEN;
    for (uint32_t i = 0; i < k; ++i) {
      const df11_matrix &m = ms[first + i];
      if (m.n > DF11_MAX_N) return DF11_ERR_TOO_LARGE;
      if (m.n == 0) continue;
      if (!m.stream || !m.gaps || !m.block_pos || !m.sign_mantissa || !m.tables ||
          !d_outs[first + i])
        return DF11_ERR_INVALID_ARG;
      if (!aligned16(m.stream) || !aligned16(m.gaps) || !aligned16(m.sign_mantissa) ||
          !aligned16(m.tables) || !aligned16(d_outs[first + i]) || ((uintptr_t)m.block_pos & 3u))
        return DF11_ERR_INVALID_ARG;
      if (m.min_len < 1 || m.min_len > DF11_MAX_CODE_LEN) return DF11_ERR_INVALID_ARG;
      if (m.total_bits < m.n * (uint64_t)m.min_len || m.total_bits > m.n * 32ull)
        return DF11_ERR_INVALID_ARG;
      const uint64_t C = cdiv(m.total_bits, 64);
      const uint64_t B = cdiv(C, kT);
      DecMat &d = P.m[P.count];
      d.stream = m.stream;
      d.gaps = m.gaps;
      d.pos = m.block_pos;
      d.sm = m.sign_mantissa;
      d.tables = reinterpret_cast<const DecodeTables *>(m.tables);
      d.out = d_outs[first + i];
      d.n = m.n;
      d.total_bits = m.total_bits;
      d.n_chunks = C;
      P.block_start[P.count + 1] = P.block_start[P.count] + B;
      min_len = std::min(min_len, m.min_len);
      ++P.count;
    }
    if (P.count == 0) continue;
    for (uint32_t i = P.count + 1; i <= DF11_MAX_BATCH; ++i) P.block_start[i] = P.block_start[P.count];
    // at most ceil(64/min_len) codes start in a chunk
    const uint32_t per_block = (uint32_t)cdiv(64, min_len) * kT;
    P.stage_cap = (per_block + 15u) & ~15u;
    const uint32_t smem = smem_layout(P.stage_cap).total;
    int occ = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, decode_kernel, kT, smem) != cudaSuccess)
      return DF11_ERR_CUDA;
    if (occ < 1) return DF11_ERR_CUDA;
    const uint64_t blocks = P.block_start[P.count];
    const uint64_t grid = std::min<uint64_t>(blocks, (uint64_t)sms * occ);
    decode_kernel<<<(unsigned)grid, kT, smem, s>>>(P);
    st = launch_status();
    if (st != DF11_OK) return st;
  }
  return DF11_OK;
}

extern "C" df11_status df11_decode(const df11_matrix *m, uint16_t *d_out, uint32_t *d_status,
                                   df11_stream_t stream) {
  if (!m) return DF11_ERR_INVALID_ARG;
  return df11_decode_block_batch(m, 1, &d_out, d_status, stream);
}
