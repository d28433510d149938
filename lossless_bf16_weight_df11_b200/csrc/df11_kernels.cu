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
//   enc_block_max_kernel  most codes starting in one block (sizes the
//                       decoder's staging)
//   decode_kernel       persistent CTAs over the (matrix, unit) list of a
//                       batch; a unit is two blocks of 256 chunks, fetched
//                       with bulk copies (TMA, no multicast) one unit ahead;
//                       each thread decodes two consecutive chunks with a
//                       12-bit shared-memory table into warp-interleaved
//                       private rows; a CTA prefix sum of the per-thread
//                       code counts places the exponents, which are merged
//                       with the sign/mantissa bytes and stored as 16-byte
//                       BF16 rows
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>
#include <vector>
#include <cstddef>
#include <mutex>

#include "df11.h"
#include "df11_codebook.h"
#include "df11_internal.h"

using df11i::DecodeTables;

namespace {

constexpr int kT = 256;  // threads per decode group (a CTA holds up to four)
// Bounded mbarrier polls before a wait gives up (DF11_ERR_TIMEOUT).  The test
// build (DF11_TEST_HOOKS) compiles with a small limit.
#ifndef DF11_WAIT_LIMIT
#define DF11_WAIT_LIMIT (1u << 22)
#endif
constexpr uint32_t kWaitLimit = DF11_WAIT_LIMIT;

__device__ __forceinline__ void set_status(uint32_t *st, uint32_t code) {
  if (st) atomicCAS(st, 0u, code);
}

__device__ __forceinline__ uint32_t bswap32(uint32_t x) { return __byte_perm(x, 0, 0x0123); }


// ============================================================ histogram

constexpr int kHistWarps = 4;
constexpr int kHistThreads = kHistWarps * 32;
constexpr size_t kHistSmem = (size_t)kHistWarps * 128 * 32 * 4;  // 64 KiB
constexpr int kHistUnroll = 8;              // 16-byte vectors per lane per step
constexpr uint32_t kHistFlushEvery = 8000;  // vectors per lane: < 65535 / 8 increments
static_assert(kHistFlushEvery % kHistUnroll == 0, "flush exactly at the limit");

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
  // warp-uniform loop: each step a warp reads kHistUnroll x 32 consecutive
  // 16-byte vectors; the next step's vectors are requested before this
  // step's counting (its chain of shared-memory read-modify-writes) starts
  const uint64_t step = warps_total * (kHistUnroll * 32);
  uint64_t base = gwarp * (kHistUnroll * 32);
  uint4 q[kHistUnroll];
  auto load = [&](uint64_t b) {
#pragma unroll
    for (int u = 0; u < kHistUnroll; ++u) {
      const uint64_t i = b + u * 32 + lane;
      q[u] = i < nvec ? __ldg(wv + i) : make_uint4(0, 0, 0, 0);
    }
  };
  if (base < nvec) load(base);
  uint32_t since = 0;
  for (; base < nvec; base += step) {
    uint4 cur[kHistUnroll];
#pragma unroll
    for (int u = 0; u < kHistUnroll; ++u) cur[u] = q[u];
    if (base + step < nvec) load(base + step);
#pragma unroll
    for (int u = 0; u < kHistUnroll; ++u) {
      const uint64_t i = base + u * 32 + lane;
      if (i < nvec) {
        add2(cur[u].x);
        add2(cur[u].y);
        add2(cur[u].z);
        add2(cur[u].w);
      }
    }
    since += kHistUnroll;
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

// Entry t of the encoder's codebook: {length, code left-justified in 32 bits},
// from the launch parameters, or from a device codebook (df11_codebook) when
// dcb is given.  A device length above 32 counts as 32; a code's bits above
// its length fall off.
__device__ __forceinline__ uint2 enc_entry(const EncCodebook &cb, const df11_codebook *dcb, int t) {
  if (dcb) {
    uint32_t L = dcb->len[t];
    L = L > DF11_MAX_CODE_LEN ? DF11_MAX_CODE_LEN : L;
    return make_uint2(L, L ? dcb->code[t] << (32 - L) : 0u);
  }
  return make_uint2(cb.len[t], cb.code[t]);
}

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
    const uint16_t *__restrict__ w, uint64_t n, EncCodebook cb, const df11_codebook *dcb,
    uint64_t *__restrict__ tile_sum, uint64_t n_tiles, uint4 *__restrict__ stream,
    uint64_t stream_vecs, uint4 *__restrict__ gaps, uint64_t gap_vecs, uint32_t *status) {
  __shared__ uint8_t s_len[256];
  __shared__ uint32_t s_warp[df11i::kEncThreads / 32];
  const int t = threadIdx.x;
  s_len[t] = (uint8_t)enc_entry(cb, dcb, t).x;
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
    uint64_t n_blocks, uint64_t n, uint32_t *status, uint32_t *block_max) {
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
    if (block_max) *block_max = 0u;
  }
}

// Pack the codes of one tile.  Each thread appends its 16 codes to a pair of
// 32-bit registers (the word being filled and the next, most significant bit
// first) and ORs every word it completes into a shared bit buffer covering
// the tile's bit range (a thread's first and last words may hold a
// neighbouring thread's bits).  The thread that owns the first code starting
// in a chunk records that chunk's gap in a shared byte per chunk; the one
// that owns the first code starting in a block of 256 chunks writes the
// block's output position.  The buffer is then written out as 32-bit words
// (byte-swapped to the MSB-first byte order), and the tile's gaps as packed
// 5-bit fields; words shared with the neighbouring tiles are OR-ed
// atomically into the cleared stream and gap buffers.  Codes arrive
// left-justified (code << (32 - length)).
__device__ __forceinline__ void red_or_shared_if(uint32_t *p, uint32_t v, bool c) {
  asm volatile("{\n .reg .pred q;\n setp.ne.u32 q, %2, 0;\n @q red.shared.or.b32 [%0], %1;\n}\n" ::"r"(
                   (uint32_t)__cvta_generic_to_shared(p)),
               "r"(v), "r"((uint32_t)c)
               : "memory");
}

__global__ void __launch_bounds__(df11i::kEncThreads) enc_pack_kernel(
    const uint16_t *__restrict__ w, uint64_t n, EncCodebook cb, const df11_codebook *dcb,
    const uint64_t *__restrict__ tile_start, uint64_t total_bits, uint8_t *__restrict__ stream,
    uint64_t stream_alloc, uint8_t *__restrict__ gaps, uint64_t gaps_alloc,
    uint32_t *__restrict__ block_pos, uint64_t n_blocks, uint8_t *__restrict__ sign_mantissa) {
  constexpr int kWords = df11i::kEncTile * DF11_MAX_CODE_LEN / 32 + 2;
  __shared__ uint32_t s_bits[kWords];
  __shared__ uint2 s_lc[256];  // {length, left-justified code}
  __shared__ uint32_t s_warp[df11i::kEncThreads / 32];
  __shared__ uint32_t s_lastlen[df11i::kEncThreads / 32];  // each warp's last code length
  // gap of each chunk from chunk S0/64 on; 0xFF: the chunk's first code is
  // not in this tile
  constexpr int kGapChunks = df11i::kEncTile * DF11_MAX_CODE_LEN / DF11_CHUNK_BITS + 2;
  __shared__ uint8_t s_gap[kGapChunks];
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  s_lc[t] = enc_entry(cb, dcb, t);
  for (int k = t; k < kGapChunks; k += df11i::kEncThreads) s_gap[k] = 0xFFu;
  const uint64_t tile = blockIdx.x;
  const uint64_t S = tile_start[tile], E = tile_start[tile + 1];
  const uint64_t S0 = S & ~31ull;
  const uint32_t nwords = (uint32_t)((E - S0 + 31) >> 5);
  for (uint32_t k = t; k < nwords + 1 && k < (uint32_t)kWords; k += df11i::kEncThreads) s_bits[k] = 0u;
  // the value before the tile (its length is the first code's predecessor)
  const uint16_t before = (t == 0 && tile > 0) ? w[tile * df11i::kEncTile - 1] : (uint16_t)0;

  uint16_t v[16];
  const uint64_t i0 = tile * df11i::kEncTile + (uint64_t)t * df11i::kEncPerThread;
  load_tile_values(w, n, i0, v);
  const uint32_t nk = i0 < n ? (n - i0 < 16 ? (uint32_t)(n - i0) : 16u) : 0u;  // values of this thread
  // every thread reads the whole code table (and later the cleared bit and
  // gap buffers): the fills above must be complete first
  __syncthreads();
  // code-length sum, and the length of this thread's last value (the
  // value before the next thread's first)
  uint32_t sum = 0, my_last = 0;
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    const uint32_t Lk = (uint32_t)k < nk ? s_lc[(v[k] >> 7) & 0xFFu].x : 0u;
    sum += Lk;
    my_last = (uint32_t)k < nk ? Lk : my_last;
  }
  uint32_t incl = sum;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    uint32_t o = __shfl_up_sync(0xffffffffu, incl, d);
    if (lane >= d) incl += o;
  }
  if (lane == 31) {
    s_warp[warp] = incl;
    s_lastlen[warp] = my_last;
  }
  __syncthreads();
  uint32_t wpre = 0;
  for (int i = 0; i < warp; ++i) wpre += s_warp[i];
  const uint32_t rel = (uint32_t)(S - S0) + wpre + incl - sum;  // bit offset in s_bits
  const uint64_t start0 = S + wpre + incl - sum;                // absolute offset of the first code
  // length of the value before this thread's first one: the previous
  // thread's last (a value of the previous tile for thread 0)
  const uint32_t up = __shfl_up_sync(0xffffffffu, my_last, 1);
  uint32_t prev_len = lane ? up : (warp ? s_lastlen[warp - 1] : s_lc[(before >> 7) & 0xFFu].x);
  if (i0 == 0 || !nk) prev_len = 0;
  const uint32_t cb0 = (uint32_t)(S0 & 63u);  // S0's offset in its chunk
  // Bounds of the shared indices below: codes are at most 32 bits (checked
  // by the launcher), so the tile's bits E - S <= 4096 * 32 and every bit
  // offset rel + off <= 31 + 131072: word index wi <= 4096 < kWords, chunk
  // index pos / 64 <= 2049 < kGapChunks.
  uint32_t hi = 0, lo = 0;                 // the word being filled (word wi) and the next
  uint32_t nb = rel & 31u, wi = rel >> 5;  // bits of word wi already taken
  uint32_t off = 0;                        // bits of this thread's codes so far
  uint32_t last_len = 0;
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    if ((uint32_t)k >= nk) break;
    const uint2 lc = s_lc[(v[k] >> 7) & 0xFFu];
    const uint32_t L = lc.x;
    hi |= lc.y >> nb;                     // nb < 32
    lo |= __funnelshift_r(0u, lc.y, nb);  // the code's bits past word wi
    nb += L;
    const bool full = nb >= 32;
    red_or_shared_if(&s_bits[wi], hi, full);
    wi += full ? 1u : 0u;
    hi = full ? lo : hi;
    lo = full ? 0u : lo;
    nb -= full ? 32u : 0u;
    // the code starts a chunk (block) when its offset in that chunk (block)
    // is below the previous code's length; the very first code starts both
    const uint32_t pos = cb0 + rel + off;  // bit offset from chunk S0/64
    if ((k == 0 && i0 == 0) || (pos & 63u) < prev_len) {
      s_gap[pos >> 6] = (uint8_t)(pos & 63u);
      if ((k == 0 && i0 == 0) || (((uint32_t)start0 + off) & 16383u) < prev_len) {
        const uint64_t b = (start0 + off) >> 14;
        if (b < n_blocks) block_pos[b] = (uint32_t)(i0 + k);
      }
    }
    prev_len = L;
    last_len = L;
    off += L;
  }
  if (nb) atomicOr(&s_bits[wi], hi);
  if (nk && i0 + nk == n) {
    // the last chunk / block may begin inside the final code: its gap points
    // at the end of the stream
    const uint64_t C = (total_bits + 63) >> 6;
    const uint64_t s64 = start0 + off - last_len;  // the final code's start
    if (C > 0 && (s64 >> 6) < C - 1) {
      const uint64_t lc = (C - 1) - (S0 >> 6);
      if (lc < (uint64_t)kGapChunks) s_gap[lc] = (uint8_t)(total_bits - 64 * (C - 1));
    }
    if (n_blocks > 0 && (s64 >> 14) < n_blocks - 1) block_pos[n_blocks - 1] = (uint32_t)n;
  }
  // sign/mantissa plane ([Format]: kept verbatim, one byte per value).  Two
  // values per 32-bit word: the sign (bit 15 of a value) moved down to bit 7,
  // the mantissa (bits 6..0) kept, both values at once; then the two low
  // bytes of two such words packed into one word of four plane bytes
  if (i0 + 16 <= n) {
    uint32_t pk[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint32_t w0 = (uint32_t)v[4 * q] | ((uint32_t)v[4 * q + 1] << 16);
      const uint32_t w1 = (uint32_t)v[4 * q + 2] | ((uint32_t)v[4 * q + 3] << 16);
      const uint32_t t0 = (w0 & 0x007F007Fu) | ((w0 >> 8) & 0x00800080u);
      const uint32_t t1 = (w1 & 0x007F007Fu) | ((w1 >> 8) & 0x00800080u);
      pk[q] = __byte_perm(t0, t1, 0x6420);
    }
    *reinterpret_cast<uint4 *>(sign_mantissa + i0) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
  } else {
#pragma unroll
    for (int k = 0; k < 16; ++k)
      if ((uint32_t)k < nk) sign_mantissa[i0 + k] = (uint8_t)(((v[k] >> 8) & 0x80u) | (v[k] & 0x7Fu));
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
  // gaps: chunk c's five bits are bits 5c..5c+4 of the gap stream.  The
  // chunks this tile may own are local 0 .. nch-1 (chunk S0/64 on); a word
  // holding a chunk the tile does not own is OR-ed in, others are stored
  if (E > S) {
    const uint64_t c_base = S0 >> 6;
    const uint32_t nch = ((cb0 + (uint32_t)(E - S0) - 1) >> 6) + 1;
    const uint64_t w_lo = (5 * c_base) >> 5, w_hi = (5 * (c_base + nch) - 1) >> 5;
    uint32_t *gaps32 = reinterpret_cast<uint32_t *>(gaps);
    const uint64_t gap_words = gaps_alloc >> 2;
    for (uint64_t gw = w_lo + t; gw <= w_hi; gw += df11i::kEncThreads) {
      if (gw >= gap_words) break;
      // 64-bit window: bit 63 is gap-stream bit 32 gw - 4
      uint64_t acc = 0;
      bool owned = true;
      // the chunks touching the word: cf .. cf + 7 (cf's field begins at
      // most 4 bits before the word)
      const uint64_t cf = (32 * gw) / 5;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int64_t c = (int64_t)cf + j;
        const int64_t rb = 5 * c - (int64_t)(32 * gw) + 4;  // chunk's first bit in the window
        if (rb > 35) continue;                              // begins after the word
        const int64_t lc = c - (int64_t)c_base;
        const uint32_t gv = (lc >= 0 && lc < (int64_t)nch) ? s_gap[lc] : 0xFFu;
        if (gv == 0xFFu) {
          owned = false;
          continue;
        }
        acc |= (uint64_t)(gv & 31u) << (59 - rb);
      }
      const uint32_t val = bswap32((uint32_t)(acc >> 28));
      if (owned) gaps32[gw] = val;
      else if (val) atomicOr(&gaps32[gw], val);
    }
  }
}

// Most codes starting in any one block: max over b of pos[b+1] - pos[b].
__global__ void __launch_bounds__(256) enc_block_max_kernel(const uint32_t *__restrict__ pos,
                                                            uint64_t n_blocks, uint32_t *out) {
  uint32_t best = 0;
  for (uint64_t b = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; b < n_blocks;
       b += (uint64_t)gridDim.x * blockDim.x)
    best = max(best, pos[b + 1] - pos[b]);
#pragma unroll
  for (int d = 16; d > 0; d >>= 1) best = max(best, __shfl_down_sync(0xffffffffu, best, d));
  if ((threadIdx.x & 31) == 0 && best) atomicMax(out, best);
}

// ============================================================ codebook on the device

// One CTA of 256 threads, thread t standing for exponent t.  The ranks, the
// normalised lengths, the canonical codes, the encoded size and the lookup
// table are computed in parallel; the two tree constructions (Huffman, and
// package-merge when the cap binds) run on thread 0.  Every step is the
// shared implementation df11_build_codebook uses on the host.
constexpr int kCbThreads = 256;

__global__ void __launch_bounds__(kCbThreads) codebook_kernel(
    const uint64_t *__restrict__ hist, uint32_t cap, df11_codebook *__restrict__ cb_out,
    DecodeTables *__restrict__ t_out, uint64_t *__restrict__ total_bits, uint32_t *status) {
  __shared__ df11cb::Scratch sc;
  __shared__ df11cb::TableAux aux;
  __shared__ df11_codebook cb;
  __shared__ uint64_t h[256];
  __shared__ uint32_t len_count[DF11_MAX_CODE_LEN + 1];
  __shared__ uint64_t next[DF11_MAX_CODE_LEN + 1];
  __shared__ uint64_t s_bits[kCbThreads / 32];
  __shared__ int s_ok;
  const int t = threadIdx.x;
  h[t] = hist[t];
  if (t <= (int)DF11_MAX_CODE_LEN) len_count[t] = 0;
  __syncthreads();
  const bool present = h[t] != 0;
  if (present) sc.hist_sorted[df11cb::ascending_rank(h, t)] = h[t];
  const int m = __syncthreads_count(present);
  if (t == 0) {
    int longest = m ? df11cb::huffman_depths(m, sc) : 0;
    if (longest > (int)cap) longest = df11cb::package_merge_depths(m, (int)cap, sc);
    s_ok = longest >= 0;
    if (s_ok) {
      for (int i = 0; i < m; ++i) ++len_count[sc.depth[i]];
      df11cb::first_codes(len_count, next);
    }
  }
  __syncthreads();
  if (!s_ok) {
    if (t == 0) set_status(status, DF11_ERR_INVALID_ARG);
    return;
  }
  uint32_t *tz = reinterpret_cast<uint32_t *>(t_out);  // padding included
  for (uint32_t i = t; i < sizeof(DecodeTables) / 4; i += kCbThreads) tz[i] = 0u;
  cb.len[t] = df11cb::normalised_length(h, len_count, t);
  __syncthreads();
  cb.code[t] = df11cb::canonical_code(cb.len, next, t);
  uint64_t bits = h[t] * cb.len[t];
#pragma unroll
  for (int d = 16; d > 0; d >>= 1) bits += __shfl_down_sync(0xffffffffu, bits, d);
  if ((t & 31) == 0) s_bits[t >> 5] = bits;
  __syncthreads();
  if (t == 0) {
    uint64_t tot = 0;
    uint32_t mx = 0, mn = m ? DF11_MAX_CODE_LEN : 0u;
    for (int i = 0; i < kCbThreads / 32; ++i) tot += s_bits[i];
    for (int i = 0; i < 256; ++i)
      if (cb.len[i]) {
        mx = cb.len[i] > mx ? cb.len[i] : mx;
        mn = cb.len[i] < mn ? cb.len[i] : mn;
      }
    cb.max_len = mx;
    cb.min_len = mn;
    cb.n_symbols = (uint32_t)m;
    cb.cap = cap;
    *total_bits = tot;
    s_ok = df11cb::table_lengths(&cb, t_out, aux) == DF11_OK;
  }
  __syncthreads();
  if (!s_ok) {  // cannot happen for a codebook built here
    if (t == 0) set_status(status, DF11_ERR_INVALID_ARG);
    return;
  }
  df11cb::table_value(&cb, t_out, t);
  __syncthreads();
  for (uint32_t v = t; v < (uint32_t)df11i::kLutSize; v += kCbThreads)
    t_out->lut[v] = df11cb::lut_entry_for(*t_out, aux, cb.max_len, v);
  cb_out->len[t] = cb.len[t];
  cb_out->code[t] = cb.code[t];
  if (t == 0) {
    cb_out->max_len = cb.max_len;
    cb_out->min_len = cb.min_len;
    cb_out->n_symbols = cb.n_symbols;
    cb_out->cap = cb.cap;
  }
}

// ============================================================ decode
//
// Work unit: kUnitChunks = 512 consecutive chunks of one matrix (two of the
// format's 256-chunk blocks; the last unit of a matrix may hold one).  A group
// of 256 threads decodes a unit, each thread two consecutive chunks: it starts
// at the first chunk's gap and decodes straight on through the second, because
// the first code starting in the second chunk begins exactly where the last
// code starting in the first one ends.  The unit's first output is pos[2u] and
// its outputs end at pos[min(2u + 2, B)].
//
// A CTA (one per SM) holds up to kMaxGroups such groups.  They share one copy
// of the current matrix's decode tables in shared memory; everything else (the
// stages the unit's bytes are copied into, the staging rows, the mbarriers) is
// the group's own, and a group synchronises with a named barrier of its own.
// The CTA as a whole synchronises only where the tables change: its share of
// the batch's (matrix, unit) list is split at matrix boundaries, and within
// one matrix the units are dealt out to the groups in turn.

constexpr int kMaxGroups = 4;
constexpr int kCPT = 2;                                       // chunks per thread
constexpr uint32_t kUnitChunks = kT * kCPT;                   // 512
constexpr uint32_t kUnitBlocks = kUnitChunks / DF11_BLOCK_CHUNKS;  // 2
constexpr uint32_t kBlockStreamBytes = 8 * DF11_BLOCK_CHUNKS;      // 2048
constexpr uint32_t kBlockGapBytes = DF11_GAP_BITS * DF11_BLOCK_CHUNKS / 8;  // 160
static_assert(kUnitBlocks == 2, "a unit is two blocks (its middle position is checked)");
// warps whose threads decode the unit's first block
constexpr int kFirstBlockWarps = DF11_BLOCK_CHUNKS / kCPT / 32;  // 4

struct DecMat {
  const uint8_t *stream;
  const uint8_t *gaps;
  const uint32_t *pos;
  const uint8_t *sm;
  const uint16_t *run_index;  // indexed decoder only
  const uint32_t *seg;        // segment decoder only: the segment index
  const DecodeTables *tables;
  uint16_t *out;
  uint64_t n;
  uint64_t total_bits;
  uint32_t n_chunks;  // C = ceil(total_bits / 64) (< 2^31 for n < 2^32)
  uint32_t n_blocks;  // B = ceil(C / 256); pos holds B + 1 entries
  uint32_t n_segs;    // segment decoder: S = ceil(n / 64); seg holds S + 1 entries
  // fused matmul only: the matrix is rows x cols (row-major), x holds
  // `batch` rows of cols BF16 activations, y `batch` rows of rows FP32 sums
  uint32_t rows, cols;
  const uint16_t *x;
  float *y;
};

struct DecParams {
  DecMat m[DF11_MAX_BATCH];
  uint64_t unit_start[DF11_MAX_BATCH + 1];  // prefix sums of units per matrix
  uint32_t count;
  uint32_t stage_cap;  // bytes: max codes per unit, rounded up to 16
  uint32_t min_len;    // shortest code of the batch (regions are sized by it)
  uint32_t batch;      // fused matmul: activation rows (<= the kernel's NB)
  uint32_t *status;
#ifdef DF11_TEST_HOOKS
  // test build only: bytes every stream-stage barrier expects beyond what its
  // bulk copies deliver, so that the copies land but the waits run out
  uint32_t starve_tx;
#endif
};

constexpr uint32_t kStreamStage = 8 * kUnitChunks + 16;         // a unit of chunks + the next word
constexpr uint32_t kGapStage = DF11_GAP_BITS * kUnitChunks / 8;  // 320 B
constexpr uint32_t kStageBytes = kStreamStage + kGapStage + 16;
constexpr uint32_t kTablesSmem = (uint32_t)((sizeof(DecodeTables) + 127) & ~(size_t)127);
static_assert(kStageBytes % 16 == 0 && sizeof(DecodeTables) % 16 == 0, "stage alignment");

__host__ __device__ constexpr uint32_t round16(uint32_t x) { return (x + 15u) & ~15u; }

// Rows of the fused matmul's per-unit accumulators: a unit's outputs span at
// most (cols - 8 + units's codes + 15) / cols + 1 rows; with cols >= 256 and
// at most 32768 codes per unit that is below 136.
constexpr uint32_t kAccRows = 136;
constexpr uint32_t kMinMatmulCols = DF11_MATMUL_MIN_COLS;

// One group's shared memory, as offsets from the group's base (every section
// on a 16-byte boundary: bulk-copy destinations, 16-byte accesses, mbarriers):
//   stage0/1  a unit's stream bytes (+ the next 16) and gap bytes, each
//   sm        the sign/mantissa bytes of outputs P0 & ~15 .. P1 (<= cap + 32)
//   linear    the unit's exponents in output order, byte j for output
//             (P0 & ~15) + j; the merge reads it in 16-byte groups up to
//             round16(15 + cap) and relocation writes up to 15 + cap
//   priv      the threads' private rows (region_bytes per thread)
//   bars      mbarriers of stage 0, stage 1 and the sign/mantissa copy
//   meta      per stage: P0, P1, matrix, unit, PM (+ row, col for the matmul)
//   warp      per-warp code totals
//   acc       fused matmul row sums [NB][kAccRows]
struct GroupLayout {
  uint32_t stage0, stage1, sm, linear, priv, bars, meta, warp, acc, size;
};

__host__ __device__ inline GroupLayout group_layout(uint32_t cap, uint32_t region_bytes,
                                                    uint32_t nb) {
  GroupLayout G;
  G.stage0 = 0;
  G.stage1 = kStageBytes;
  G.sm = 2 * kStageBytes;
  G.linear = round16(G.sm + cap + 32);
  G.priv = round16(G.linear + cap + 32);
  G.bars = round16(G.priv + kT * region_bytes);
  G.meta = G.bars + 32;
  G.warp = G.meta + 64;
  G.acc = G.warp + 32;
  G.size = (G.acc + 4 * kAccRows * nb + 127u) & ~127u;
  return G;
}

// Per-thread private region, in 32-bit rows: the codes that can start in a
// thread's two chunks (ceil(128/min_len)), three codes of overshoot from the
// last table entry; rounded to an odd number of rows.
__host__ __device__ constexpr uint32_t region_words_even(uint32_t min_len) {
  return ((64 * kCPT + min_len - 1) / min_len + 3 + 4) / 4;
}
__host__ __device__ constexpr uint32_t region_bytes_for(uint32_t min_len) {
  return 4 * (region_words_even(min_len) + (region_words_even(min_len) % 2 == 0 ? 1 : 0));
}

// ---- shared memory through 32-bit shared-window addresses
__device__ __forceinline__ uint32_t smem_addr(const void *p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

// The checked build (DF11_CHECKED): every access of the decode path through
// the helpers below is checked against the CTA's dynamic shared memory (range
// and alignment), every global store and bulk-copy source against its buffer;
// a failed check skips the access and sets DF11_ERR_BOUNDS in the launch's
// status word, so an indexing error shows as a status, not a fault.  The
// product build compiles the checks away.
#ifdef DF11_CHECKED
// Set by each checked kernel before its first checked access: the status word
// and the shared-space address of its own dynamic shared memory (an extern
// shared array declared outside the kernel was found not to start there).
__shared__ uint32_t *s_check_status;
__shared__ uint32_t s_dyn_base;
__device__ __forceinline__ void check_failed() {
  if (s_check_status) atomicCAS(s_check_status, 0u, (uint32_t)DF11_ERR_BOUNDS);
}
__device__ __forceinline__ bool smem_ok(uint32_t a, uint32_t bytes) {
  uint32_t size;
  asm("mov.u32 %0, %%dynamic_smem_size;" : "=r"(size));
  const uint32_t lo = s_dyn_base;
  const bool ok = a >= lo && a - lo <= size && bytes <= size - (a - lo) && (a & (bytes - 1)) == 0;
  if (!ok) check_failed();
  return ok;
}
#define DF11_SMEM_CHECK(a, bytes, on_fail) \
  if (!smem_ok((a), (bytes))) on_fail;
#define DF11_GLOBAL_CHECK(cond, on_fail) \
  if (!(cond)) {                         \
    check_failed();                      \
    on_fail;                             \
  }
#else
#define DF11_SMEM_CHECK(a, bytes, on_fail)
#define DF11_GLOBAL_CHECK(cond, on_fail)
#endif

// (A failed check in the checked build skips the access.  A load then
// returns a value whose top four bits are set: read as a table entry's
// control word it consumes 15 bits and decodes nothing, so every decode loop
// still advances to its end.)
#ifdef DF11_CHECKED
constexpr uint32_t kCheckFailValue = 0xF0000000u;
#endif
__device__ __forceinline__ uint32_t lds32(uint32_t a) {
  DF11_SMEM_CHECK(a, 4, return kCheckFailValue)
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a) : "memory");
  return v;
}
__device__ __forceinline__ uint32_t lds8(uint32_t a) {
  DF11_SMEM_CHECK(a, 1, return 0u)
  uint32_t v;
  asm volatile("ld.shared.u8 %0, [%1];" : "=r"(v) : "r"(a) : "memory");
  return v;
}
__device__ __forceinline__ uint2 lds64(uint32_t a) {
  DF11_SMEM_CHECK(a, 8, return make_uint2(0u, kCheckFailValue))
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(a) : "memory");
  return v;
}
__device__ __forceinline__ uint4 lds128(uint32_t a) {
  DF11_SMEM_CHECK(a, 16, return make_uint4(0u, 0u, 0u, 0u))
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(a)
               : "memory");
  return v;
}
__device__ __forceinline__ void sts32(uint32_t a, uint32_t v) {
  DF11_SMEM_CHECK(a, 4, return)
  asm volatile("st.shared.u32 [%0], %1;" ::"r"(a), "r"(v) : "memory");
}
__device__ __forceinline__ void sts64(uint32_t a, uint32_t x, uint32_t y) {
  DF11_SMEM_CHECK(a, 8, return)
  asm volatile("st.shared.v2.u32 [%0], {%1, %2};" ::"r"(a), "r"(x), "r"(y) : "memory");
}
__device__ __forceinline__ void sts128_zero(uint32_t a) {
  DF11_SMEM_CHECK(a, 16, return)
  asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(a), "r"(0u) : "memory");
}
__device__ __forceinline__ void red_or32(uint32_t a, uint32_t v) {
  DF11_SMEM_CHECK(a, 4, return)
  asm volatile("red.shared.or.b32 [%0], %1;" ::"r"(a), "r"(v) : "memory");
}
// (a * b) >> 32 + c: field extraction on the multiply pipe
__device__ __forceinline__ uint32_t madhi(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t r;
  asm("mad.hi.u32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(c));
  return r;
}

// Barrier of one decode group (named barrier id, the group's 256 threads).
__device__ __forceinline__ void group_sync(uint32_t id) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(kT) : "memory");
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

// Bulk copy global -> shared (TMA, CTA-local, no multicast).  Both addresses
// 16-byte aligned, size a multiple of 16.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t phase) {
  for (uint32_t it = 0; it < kWaitLimit; ++it) {
    uint32_t done;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, "
        "p;\n}\n"
        : "=r"(done)
        : "r"(bar), "r"(phase)
        : "memory");
    if (done) return true;
  }
  return false;
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

// The control word of a code decoded by the length search: one code, no
// further starts, no bits counted (the trim after the loop then keeps it).
constexpr uint32_t kLongCodeCtrl =
    df11i::lut_ctrl(1, df11i::kCtrlNoStart, df11i::kCtrlNoStart, df11i::kCtrlNoStart, 0);

// Appending decoded exponents to a thread's private bytes.  The private
// regions of a warp are interleaved by 32-bit word: word j of lane l is
// shared word 32 j + l of the warp's region, so any access in which every
// lane touches one word of its own falls in 32 different banks.  The word
// being filled is kept in a register (cur) and written through on every
// step with one 32-bit store at row_a.  nb counts the bits appended (8 per
// exponent) in its bits 0..10; a table entry's control word is added to it
// whole (its bits 0..10 are 8 x its count, its higher bits land above the
// count and are never read).  xs holds the step's exponents from the low byte
// up (absent slots zero).
#define DF11_APPEND(xs, add)                                                \
  {                                                                         \
    const uint32_t lo = cur | __funnelshift_l(0u, (xs), nb);                \
    const uint32_t hi = __funnelshift_l((xs), 0u, nb);                      \
    sts32(row_a, lo);                                                       \
    const uint32_t nb2 = nb + (add);                                        \
    row_a = col_a + ((nb2 & 0x7E0u) << 2);                                  \
    cur = ((nb ^ nb2) & 32u) ? hi : lo;                                     \
    nb = nb2;                                                               \
  }

// One table step on the window of stream words hw:lw at bit p: the entry's
// exponents are appended and p advances by the bits they use.
#define DF11_STEP(hw, lw)                                                   \
  {                                                                         \
    const uint32_t w = __funnelshift_l((lw), (hw), p);                      \
    const uint2 e = lds64(lut_a + ((w >> (32 - df11i::kLutBits)) << 3));    \
    ctrl = e.y;                                                             \
    DF11_APPEND(e.x, ctrl)                                                  \
    p = madhi(ctrl, 1u << (32 - df11i::kCtrlUsedShift), p);                 \
  }

// 4 rotated exponents + 4 sign/mantissa bytes -> 4 BF16 words (two 32-bit
// halves).  Byte i of r4 is ror8(e_i): its bits 0..6 are the exponent's high
// seven bits (the BF16 high byte's bits 0..6), bit 7 its low bit (the low
// byte's bit 7); the sign/mantissa byte supplies the other bit of each.
__device__ __forceinline__ void merge4(uint32_t r4, uint32_t s4, uint32_t &w01, uint32_t &w23) {
  const uint32_t hi4 = (s4 & 0x80808080u) | (r4 & 0x7F7F7F7Fu);
  const uint32_t lo4 = (r4 & 0x80808080u) | (s4 & 0x7F7F7F7Fu);
  w01 = __byte_perm(lo4, hi4, 0x5140);
  w23 = __byte_perm(lo4, hi4, 0x7362);
}

// A decoded unit waiting for its merge: positions, output, staging.
struct Pending {
  uint32_t P0, P1;
  uint16_t *out;
  bool ok;
  uint32_t m;               // matrix of the batch
  uint32_t row_lo, col_lo;  // fused matmul: row and column of output P0 & ~7
  uint32_t n;               // values of the matrix (bounds of out)
};

// Merge a decoded unit: exponents in the linear row, sign/mantissa bytes in
// the sm stage, both indexed from output P0 & ~15 (so byte j of either is
// output (P0 & ~15) + j).  Thread t takes the whole 8-output groups t, t+256,
// ... from output P0 & ~7 on: each is one 16-byte store, and a warp's 32
// stores fill 512 contiguous bytes.  The ragged first and last groups are
// written element by element by threads 0 and 1.  The row is cleared behind
// the reads (relocation ORs the words shared by two threads into it).
__device__ __forceinline__ void merge_group8(uint32_t lin_a, uint32_t smb, uint32_t k, uint4 &r) {
  const uint2 e8 = lds64(lin_a + 8 * k);
  sts64(lin_a + 8 * k, 0u, 0u);
  const uint2 s8 = lds64(smb + 8 * k);
  merge4(e8.x, s8.x, r.x, r.y);
  merge4(e8.y, s8.y, r.z, r.w);
}

__device__ __forceinline__ void merge_unit(const Pending &q, uint32_t lin_a, uint32_t sm_a, int t) {
  const uint32_t base8 = q.P0 & ~7u;
  const uint32_t off8 = base8 - (q.P0 & ~15u);  // 0 or 8: where base8 sits in the rows
  const uint32_t lin8 = lin_a + off8, smb = sm_a + off8;
  const uint32_t head = q.P0 & 7u;         // outputs of group 0 before the unit
  const uint32_t span8 = q.P1 - base8;     // outputs from base8 to the unit's end
  const uint32_t full0 = head ? 1u : 0u;
  const uint32_t full1 = span8 >> 3;
  uint4 *out4 = reinterpret_cast<uint4 *>(q.out + base8);
  // four independent groups per thread and pass: their shared-memory reads
  // overlap
  for (uint32_t k0 = full0 + t; k0 < full1; k0 += 4 * kT) {
#pragma unroll
    for (uint32_t j = 0; j < 4; ++j) {
      const uint32_t k = k0 + j * kT;
      if (k < full1) {
        uint4 r;
        merge_group8(lin8, smb, k, r);
        DF11_GLOBAL_CHECK(base8 + 8 * k + 8 <= q.n, continue)
        out4[k] = r;
      }
    }
  }
  // ragged first group (thread 0) and last group (thread 1, unless it is the
  // first one); element j of group k is output base8 + 8k + j
  const bool last_edge = (span8 & 7u) != 0 && !(head && full1 == 0);
  if ((t == 0 && head) || (t == 1 && last_edge)) {
    const uint32_t k = t == 0 ? 0u : full1;
    const uint32_t lo = t == 0 ? head : 0u;
    const uint32_t hi = min(8u, span8 - 8 * k);
    uint4 r;
    merge_group8(lin8, smb, k, r);
    const uint32_t wv[4] = {r.x, r.y, r.z, r.w};
    uint16_t *o = q.out + base8 + 8 * k;
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if ((uint32_t)j >= lo && (uint32_t)j < hi) {
        DF11_GLOBAL_CHECK(base8 + 8 * k + j < q.n, continue)
        o[j] = (uint16_t)(wv[j >> 1] >> (16 * (j & 1)));
      }
  }
  // (the linear row's words before base8 were never written: relocation
  // starts at byte P0 & 15 >= base8 - (P0 & ~15))
}

// The same merge with the whole 8-output groups claimed by warps,
// kMergeClaim groups at a time (four per lane), from a shared counter (*ctr,
// zero before the first claim): a warp that finished its decoding early
// merges more of the unit, so the group barrier after the merge waits less
// for the slowest decoder, and each lane's four groups are independent work.
// (Measured on a Llama-3-70B-shaped block of 855 M weights: claims of 32 /
// 64 / 96 / 128 / 160 / 256 groups gave 0.662 / 0.627 / 0.635 / 0.608 /
// 0.608 / 0.628 ms per launch.)
constexpr uint32_t kMergeClaim = 128;
__device__ __forceinline__ void merge_unit_claimed(const Pending &q, uint32_t lin_a, uint32_t sm_a,
                                                   int t, uint32_t *ctr) {
  const uint32_t base8 = q.P0 & ~7u;
  const uint32_t off8 = base8 - (q.P0 & ~15u);
  const uint32_t lin8 = lin_a + off8, smb = sm_a + off8;
  const uint32_t head = q.P0 & 7u;
  const uint32_t span8 = q.P1 - base8;
  const uint32_t full0 = head ? 1u : 0u;
  const uint32_t full1 = span8 >> 3;
  uint4 *out4 = reinterpret_cast<uint4 *>(q.out + base8);
  const uint32_t lane = (uint32_t)t & 31u;
  while (true) {
    uint32_t c = 0;
    if (lane == 0) c = atomicAdd(ctr, kMergeClaim);
    c = __shfl_sync(0xffffffffu, c, 0);
    if (full0 + c >= full1) break;  // (the same for the whole warp)
    // kMergeClaim / 32 independent groups per lane: their shared-memory
    // reads overlap
#pragma unroll
    for (uint32_t j = 0; j < kMergeClaim; j += 32) {
      const uint32_t k = full0 + c + j + lane;
      if (k < full1) {
        uint4 r;
        merge_group8(lin8, smb, k, r);
        DF11_GLOBAL_CHECK(base8 + 8 * k + 8 <= q.n, continue)
        out4[k] = r;
      }
    }
  }
  const bool last_edge = (span8 & 7u) != 0 && !(head && full1 == 0);
  if ((t == 0 && head) || (t == 1 && last_edge)) {
    const uint32_t k = t == 0 ? 0u : full1;
    const uint32_t lo = t == 0 ? head : 0u;
    const uint32_t hi = min(8u, span8 - 8 * k);
    uint4 r;
    merge_group8(lin8, smb, k, r);
    const uint32_t wv[4] = {r.x, r.y, r.z, r.w};
    uint16_t *o = q.out + base8 + 8 * k;
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if ((uint32_t)j >= lo && (uint32_t)j < hi) {
        DF11_GLOBAL_CHECK(base8 + 8 * k + j < q.n, continue)
        o[j] = (uint16_t)(wv[j >> 1] >> (16 * (j & 1)));
      }
  }
}

// Fused matmul merge: the unit's decoded weights are multiplied with the
// activations instead of being stored.  Lane l of warp w takes 8-weight
// groups w*32 + l, + 256, ... (flat index base8 + 8k, masked to the unit's
// outputs); each group's dot products with the NB activation rows are reduced
// over the warp per output row (32 consecutive groups span at most two rows
// since cols >= 256) and added into the group's per-row accumulators (row
// offsets from row_lo).  The staging row is cleared behind the reads, as in
// the plain merge.
__device__ __forceinline__ void bf16x2_to_f32(uint32_t v, float &a, float &b) {
  a = __uint_as_float(v << 16);
  b = __uint_as_float(v & 0xFFFF0000u);
}

template <int NB>
__device__ __forceinline__ void merge_unit_matmul(const Pending &q, uint32_t lin_a, uint32_t sm_a,
                                                  int t, float *acc, const DecMat &M,
                                                  uint32_t batch) {
  const int lane = t & 31, warp = t >> 5;
  const uint32_t base8 = q.P0 & ~7u;
  const uint32_t off8 = base8 - (q.P0 & ~15u);  // 0 or 8: where base8 sits in the rows
  const uint32_t lin8 = lin_a + off8, smb = sm_a + off8;
  const uint32_t head = q.P0 & 7u;
  const uint32_t span8 = q.P1 - base8;
  const uint32_t ngroups = (span8 + 7) >> 3;
  const uint32_t cols = M.cols;
  // the activations of a group: its 8 columns of each of the batch rows
  // (rows past the batch read as zero)
  auto load_x = [&](uint32_t k, uint32_t col, uint4 (&xv)[NB]) {
#pragma unroll
    for (int j = 0; j < NB; ++j) {
      bool use = k < ngroups && (uint32_t)j < batch;
      DF11_GLOBAL_CHECK(!use || col + 8 <= cols, use = false)
      xv[j] = use ? __ldg(reinterpret_cast<const uint4 *>(M.x + (size_t)j * cols + col))
                  : make_uint4(0u, 0u, 0u, 0u);
    }
  };
  // row offset and column of this lane's first group
  uint32_t col = q.col_lo + 8u * (uint32_t)(warp * 32 + lane), row = 0;
  while (col >= cols) {
    col -= cols;
    ++row;
  }
  // with one or two activation rows the next group's activations are
  // requested before this group is merged (their latency is otherwise
  // exposed once per group); with more, the registers are not spared
  constexpr bool kPrefetch = NB <= 2;
  uint4 xn[NB];
  if (kPrefetch) load_x((uint32_t)warp * 32 + lane, col, xn);
  for (uint32_t kb = (uint32_t)warp * 32; kb < ngroups; kb += kT) {
    const uint32_t k = kb + lane;
    uint32_t ncol = col + 8u * kT, nrow = row;
    while (ncol >= cols) {
      ncol -= cols;
      ++nrow;
    }
    uint4 xv[NB];
    if (kPrefetch) {
#pragma unroll
      for (int j = 0; j < NB; ++j) xv[j] = xn[j];
      load_x(k + kT, ncol, xn);
    } else {
      load_x(k, col, xv);
    }
    float d[NB];
#pragma unroll
    for (int j = 0; j < NB; ++j) d[j] = 0.f;
    if (k < ngroups) {
      uint4 r;
      merge_group8(lin8, smb, k, r);
      float w[8];
      bf16x2_to_f32(r.x, w[0], w[1]);
      bf16x2_to_f32(r.y, w[2], w[3]);
      bf16x2_to_f32(r.z, w[4], w[5]);
      bf16x2_to_f32(r.w, w[6], w[7]);
      const uint32_t lo = k == 0 ? head : 0u, hi = min(8u, span8 - 8 * k);
      if (lo != 0 || hi != 8) {
        // the unit's ragged first or last group: weights outside it are zero
#pragma unroll
        for (int i = 0; i < 8; ++i) w[i] = ((uint32_t)i >= lo && (uint32_t)i < hi) ? w[i] : 0.f;
      }
#pragma unroll
      for (int j = 0; j < NB; ++j) {
        float xf[8];
        bf16x2_to_f32(xv[j].x, xf[0], xf[1]);
        bf16x2_to_f32(xv[j].y, xf[2], xf[3]);
        bf16x2_to_f32(xv[j].z, xf[4], xf[5]);
        bf16x2_to_f32(xv[j].w, xf[6], xf[7]);
        float sdot = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) sdot = fmaf(w[i], xf[i], sdot);
        d[j] = sdot;
      }
    }
    // per-row sums over the warp: lane 0's row and the next
    const uint32_t row0 = __shfl_sync(0xffffffffu, row, 0);
    const bool second = __any_sync(0xffffffffu, k < ngroups && row != row0);
#pragma unroll
    for (int j = 0; j < NB; ++j) {
      float a = row == row0 ? d[j] : 0.f;
      float b = d[j] - a;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        a += __shfl_xor_sync(0xffffffffu, a, o);
        b += __shfl_xor_sync(0xffffffffu, b, o);
      }
      if (lane == 0 && (uint32_t)j < batch) {
        if (row0 < kAccRows) atomicAdd(acc + j * kAccRows + row0, a);
        if (second && row0 + 1 < kAccRows) atomicAdd(acc + j * kAccRows + row0 + 1, b);
      }
    }
    col = ncol;
    row = nrow;
  }
  // the linear row's words before base8 were never written: nothing to clear
}

// Add a merged unit's row sums to y and clear the accumulators (after a group
// barrier that follows the merge).
template <int NB>
__device__ __forceinline__ void flush_matmul(const Pending &q, float *acc, const DecMat &M,
                                             uint32_t batch, int t) {
  const uint32_t base8 = q.P0 & ~7u;
  const uint32_t nrows = min((q.col_lo + (q.P1 - base8) - 1) / M.cols + 1, kAccRows);
#pragma unroll
  for (int j = 0; j < NB; ++j) {
    for (uint32_t r = t; r < nrows; r += kT) {
      const float v = acc[j * kAccRows + r];
      if ((uint32_t)j < batch && v != 0.f && q.row_lo + r < M.rows)
        atomicAdd(M.y + (size_t)j * M.rows + q.row_lo + r, v);
      DF11_GLOBAL_CHECK(j * kAccRows + r < NB * kAccRows, continue)
      acc[j * kAccRows + r] = 0.f;
    }
  }
}

// Whether a lookup-table entry could take the decoder outside its private
// region.  A valid entry has its reserved control bits clear and either one
// to four codes, each at least min_len bits long (start fields increasing by
// at least min_len, the last code ending by `used` <= the window; absent
// codes' fields 15), or the long-code flag with no codes, no starts and the
// whole window consumed.  With every code at least min_len bits, at most
// ceil(128 / min_len) codes start in a thread's two chunks, plus three more
// from the last entry: the region holds them.
__device__ __forceinline__ bool lut_entry_bad(uint32_t c, uint32_t min_len) {
  const uint32_t n = (c >> df11i::kCtrlCountShift) & 7u, used = c >> df11i::kCtrlUsedShift;
  const uint32_t starts = (c >> df11i::kCtrlStartShift) & 0xFFFu;
  if (c & df11i::kCtrlReserved) return true;
  if (c & df11i::kCtrlLongFlag) return n != 0 || used != (uint32_t)df11i::kLutBits || starts != 0xFFFu;
  if (n == 0 || n > df11i::kLutMaxCodes || used > (uint32_t)df11i::kLutBits) return true;
  bool bad = false;
  uint32_t prev = 0;
#pragma unroll
  for (uint32_t j = 1; j < df11i::kLutMaxCodes; ++j) {
    const uint32_t sj = (starts >> (4 * (j - 1))) & 15u;
    if (j < n) {
      bad |= sj < prev + min_len;
      prev = sj;
    } else {
      bad |= sj != df11i::kCtrlNoStart;
    }
  }
  return bad || used < prev + min_len;
}

// MAXW: 32-bit words of a thread's private region.  NB: 0 for the plain
// decode (BF16 stored to out); 1, 2, 4 or 8 for the fused matmul with up to
// NB activation rows (P.batch of them used).  blockDim.x = 256 x groups.
template <int MAXW, int NB>
__global__ void __launch_bounds__(kT *kMaxGroups, 1) decode_kernel(const __grid_constant__ DecParams P) {
  extern __shared__ __align__(128) uint8_t smem[];
  const uint32_t ngroups = blockDim.x / kT;
  const uint32_t grp = threadIdx.x / kT;
  const int t = (int)(threadIdx.x % kT), lane = t & 31, warp = t >> 5;
  const uint32_t cap = P.stage_cap;
  const GroupLayout GL = group_layout(cap, 4 * MAXW, NB);
  const uint32_t sbase = smem_addr(smem);
  const uint32_t gofs = kTablesSmem + grp * GL.size;
  const uint32_t gbase = sbase + gofs;
  const DecodeTables &tab = *reinterpret_cast<const DecodeTables *>(smem);
  const uint32_t lut_a = sbase;  // lut is the first member of the tables
  float *acc = reinterpret_cast<float *>(smem + gofs + GL.acc);  // [NB][kAccRows] row sums
  const uint32_t bar_stage = gbase + GL.bars, bar_sm = gbase + GL.bars + 16;
  uint32_t *meta = reinterpret_cast<uint32_t *>(smem + gofs + GL.meta);
  uint32_t *warp_tot = reinterpret_cast<uint32_t *>(smem + gofs + GL.warp);
  const uint32_t lin_a = gbase + GL.linear;
  const uint32_t sm_a = gbase + GL.sm;
  // this lane's column of its warp's interleaved private region
  const uint32_t col_a = gbase + GL.priv + (uint32_t)warp * (MAXW * 128u) + 4u * lane;
  const uint32_t bar_id = 1 + grp;

  const uint64_t total = P.unit_start[P.count];
  const uint64_t g0 = (uint64_t)blockIdx.x * total / gridDim.x;
  const uint64_t g1 = (uint64_t)(blockIdx.x + 1) * total / gridDim.x;
  if (g0 >= g1) return;  // the same for every thread of the CTA
#ifdef DF11_CHECKED
  if (threadIdx.x == 0) {
    s_check_status = P.status;
    s_dyn_base = smem_addr(smem);
  }
  __syncthreads();
#endif

  // the linear rows start zeroed (the words two threads share are OR-ed into)
  for (uint32_t k = t; k < (GL.priv - GL.linear) / 16; k += kT) sts128_zero(lin_a + 16 * k);
  if (t == 0) {
    mbar_init(bar_stage, 1);
    mbar_init(bar_stage + 8, 1);
    mbar_init(bar_sm, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if constexpr (NB > 0)
    for (uint32_t k = t; k < NB * kAccRows; k += kT) acc[k] = 0.f;

  uint32_t it = 0;  // units this group has started: stage it & 1, phases from it
  bool timed_out = false;
  uint32_t m = 0;
  while (m + 1 < P.count && g0 >= P.unit_start[m + 1]) ++m;
  for (; m < P.count && P.unit_start[m] < g1; ++m) {
    // every group is past the previous matrix (and a timeout anywhere ends
    // the CTA here, with nothing of its own in flight)
    if (__syncthreads_or(timed_out)) return;
    const uint64_t s0 = max(g0, P.unit_start[m]), s1 = min(g1, P.unit_start[m + 1]);
    if (s0 >= s1) continue;
    const DecMat &M = P.m[m];
    {
      const uint4 *src = reinterpret_cast<const uint4 *>(M.tables);
      uint4 *dst = reinterpret_cast<uint4 *>(smem);
      for (uint32_t k = threadIdx.x; k < sizeof(DecodeTables) / 16; k += blockDim.x)
        dst[k] = __ldg(src + k);
    }
    __syncthreads();
    bool tbad = false;
    for (uint32_t k = threadIdx.x; k < (uint32_t)df11i::kLutSize; k += blockDim.x)
      tbad |= lut_entry_bad(tab.lut[k].y, P.min_len);
    // a table that could take a decoder past its region is not used: the
    // matrix's units decode nothing and are reported as corrupt
    const bool table_ok = !__syncthreads_or(tbad);
    // every code fits the table: the decode loop needs no long-code test
    const bool table_short = tab.max_len <= (uint32_t)df11i::kLutBits;

    const uint64_t first = s0 + grp;
    if (first >= s1) continue;
    // thread 0 fetches the positions of the unit after next one iteration
    // early: its first output P0, the first output of its second block PM
    // (P1 if it has one block) and the end of its outputs P1
    uint32_t nxt_p0 = 0, nxt_p1 = 0, nxt_pm = 0;
    auto fetch_pos = [&](uint64_t g) {
      const uint32_t b0 = kUnitBlocks * (uint32_t)(g - P.unit_start[m]);
      DF11_GLOBAL_CHECK(b0 < M.n_blocks, return)
      nxt_p0 = __ldg(M.pos + b0);
      nxt_p1 = __ldg(M.pos + min(b0 + kUnitBlocks, M.n_blocks));
      nxt_pm = b0 + 1 < M.n_blocks ? __ldg(M.pos + b0 + 1) : nxt_p1;
    };
    auto issue_stream = [&](uint64_t g, uint32_t stage) {
      const uint32_t u = (uint32_t)(g - P.unit_start[m]);
      // the unit's blocks (the last unit of a matrix may hold one) and the
      // 16 bytes after them; nothing beyond the stream's and gaps' allocations
      const uint32_t nb = min(kUnitBlocks, M.n_blocks - kUnitBlocks * u);
      const uint32_t sbytes = nb * kBlockStreamBytes + 16, gbytes = nb * kBlockGapBytes;
      const uint32_t st = gbase + (stage ? GL.stage1 : GL.stage0);
      uint32_t *mt = meta + stage * 8;
      mt[0] = nxt_p0;
      mt[1] = nxt_p1;
      mt[2] = u;
      mt[3] = nxt_pm;
      if (NB > 0) {
        // fused matmul: row and column of output p0 & ~7
        const uint32_t base8 = nxt_p0 & ~7u;
        mt[4] = base8 / M.cols;
        mt[5] = base8 % M.cols;
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      // (checked build: both sources inside the stream's and gaps' allocations)
      DF11_GLOBAL_CHECK((uint64_t)u * (8 * kUnitChunks) + sbytes <=
                                (uint64_t)kBlockStreamBytes * M.n_blocks + 16 &&
                            (uint64_t)u * kGapStage + gbytes <=
                                (uint64_t)kBlockGapBytes * M.n_blocks + 16,
                        {
                          mbar_expect_tx(bar_stage + 8 * stage, 0);
                          return;
                        })
#ifdef DF11_TEST_HOOKS
      mbar_expect_tx(bar_stage + 8 * stage, sbytes + gbytes + P.starve_tx);
#else
      mbar_expect_tx(bar_stage + 8 * stage, sbytes + gbytes);
#endif
      bulk_g2s(st, M.stream + (uint64_t)u * (8 * kUnitChunks), sbytes, bar_stage + 8 * stage);
      bulk_g2s(st + kStreamStage, M.gaps + (uint64_t)u * kGapStage, gbytes, bar_stage + 8 * stage);
    };
    if (t == 0) {
      fetch_pos(first);
      issue_stream(first, it & 1);
      if (first + ngroups < s1) fetch_pos(first + ngroups);
    }
    group_sync(bar_id);

    Pending prev{0, 0, nullptr, false, 0, 0, 0, 0};
    bool have_prev = false;
    for (uint64_t g = first; g < s1; g += ngroups, ++it) {
      const uint32_t s = it & 1;
      // [A] the previous unit is relocated into the linear row
      if (have_prev) group_sync(bar_id);
      const uint32_t *mt = meta + s * 8;
      const uint32_t P0 = mt[0], P1 = mt[1], u = mt[2], PM = mt[3];
      const uint32_t RL = NB > 0 ? mt[4] : 0u, CL = NB > 0 ? mt[5] : 0u;
      // positions are trusted only as far as they stay inside the matrix and
      // the staging row; anything else is flagged as corrupt after the count
      const bool sane = P1 >= P0 && P1 <= M.n && P1 - P0 <= cap;
      if (t == 0 && g + ngroups < s1) {
        issue_stream(g + ngroups, s ^ 1);
        if (g + 2 * ngroups < s1) fetch_pos(g + 2 * ngroups);
      }
      bool tmo = !mbar_wait(bar_stage + 8 * s, (it >> 1) & 1);

      // ---- this thread's two chunks: decoded once into the private region
      const uint32_t c0 = u * kUnitChunks + kCPT * t;
      uint32_t cnt = 0;
      bool bad = false;
      if (table_ok && c0 < M.n_chunks) {
        const uint32_t st = gbase + (s ? GL.stage1 : GL.stage0);
        // stream words W0..W3 of the two chunks and the next chunk's first, W4
        const uint4 a4 = lds128(st + 16 * t);
        const uint32_t W0 = bswap32(a4.x), W1 = bswap32(a4.y), W2 = bswap32(a4.z),
                       W3 = bswap32(a4.w), W4 = bswap32(lds32(st + 16 * t + 16));
        const uint64_t avail = M.total_bits - 64ull * c0;
        const uint32_t lim = avail < 64u * kCPT ? (uint32_t)avail : 64u * kCPT;
        // the first chunk's 5-bit gap
        const uint32_t q = DF11_GAP_BITS * kCPT * t;
        const uint32_t ga = st + kStreamStage + (q >> 3);
        const uint32_t two = (lds8(ga) << 8) | lds8(ga + 1);
        const uint32_t gap = (two >> (11 - (q & 7u))) & 31u;
        uint32_t p = gap, nb = 0, cur = 0, row_a = col_a, ctrl = 0;
        if (table_short) {
          // one loop per 32-bit word in which codes start (each loop's window
          // needs no select): while p < 32(k+1) the window is Wk:Wk+1 << p % 32
          const uint32_t l1 = min(lim, 32u), l2 = min(lim, 64u), l3 = min(lim, 96u);
#pragma unroll 1
          while (p < l1) DF11_STEP(W0, W1)
#pragma unroll 1
          while (p < l2) DF11_STEP(W1, W2)
#pragma unroll 1
          while (p < l3) DF11_STEP(W2, W3)
#pragma unroll 1
          while (p < lim) DF11_STEP(W3, W4)
        } else {
          // codes longer than the table's reach: per word a table loop; a
          // flagged entry leaves it, the code is decoded by the length search
          // (its 32-bit window lies inside Wk:Wk+1 too), and the loop resumes
#pragma unroll 1
          while (p < lim) {
            const uint32_t k = p >> 5;
            const uint32_t hw = k == 0 ? W0 : k == 1 ? W1 : k == 2 ? W2 : W3;
            const uint32_t lw = k == 0 ? W1 : k == 1 ? W2 : k == 2 ? W3 : W4;
            const uint32_t seg = min(lim, 32u * (k + 1));
            bool flagged = false;
#pragma unroll 1
            while (p < seg) {
              const uint32_t w = __funnelshift_l(lw, hw, p);
              const uint2 e = lds64(lut_a + ((w >> (32 - df11i::kLutBits)) << 3));
              if (e.y & df11i::kCtrlLongFlag) {
                flagged = true;
                break;
              }
              ctrl = e.y;
              DF11_APPEND(e.x, ctrl)
              p = madhi(ctrl, 1u << (32 - df11i::kCtrlUsedShift), p);
            }
            if (!flagged) continue;
            const uint32_t w = __funnelshift_l(lw, hw, p);
            const uint32_t L = long_code_len(w, tab);
            if (L == 0) {
              bad = true;
              break;
            }
            const uint32_t x = tab.sym[((w >> (32 - L)) + tab.base[L]) & 0xFFu];
            ctrl = kLongCodeCtrl;
            DF11_APPEND(x, ctrl)
            p += L;
          }
        }
        sts32(row_a, cur);  // the word being filled (it may have just begun)
        uint32_t d = (nb & 0x7FFu) >> 3;
        const uint32_t ncodes = (ctrl >> df11i::kCtrlCountShift) & 7u;
        if (p > lim && ncodes) {
          // the last entry ran past the end of the thread's chunks: its codes
          // that start at or after lim belong to the next thread (an absent
          // code's start field, 15, is past lim too, as lim - pl < 11)
          const uint32_t pl = p - (ctrl >> df11i::kCtrlUsedShift);
          const uint32_t past = (uint32_t)(pl + ((ctrl >> 12) & 15u) >= lim) +
                                (uint32_t)(pl + ((ctrl >> 16) & 15u) >= lim) +
                                (uint32_t)(pl + ((ctrl >> 20) & 15u) >= lim);
          d -= past - (df11i::kLutMaxCodes - ncodes);
        }
        cnt = d;
      }
      // ---- the previous unit's merge (between decode and the count barrier);
      // its sign/mantissa phase is waited for even if the unit was rejected,
      // so that the barrier is never re-armed with a copy in flight
      if (have_prev) {
        if (!mbar_wait(bar_sm, (it - 1) & 1)) tmo = true;
        else if (prev.ok) {
          if constexpr (NB == 0) merge_unit(prev, lin_a, sm_a, t);
          else merge_unit_matmul<NB>(prev, lin_a, sm_a, t, acc, P.m[prev.m], P.batch);
        }
      }
      // ---- [B] group prefix sum of the counts
      uint32_t incl = cnt;
#pragma unroll
      for (int dd = 1; dd < 32; dd <<= 1) {
        const uint32_t o = __shfl_up_sync(0xffffffffu, incl, dd);
        if (lane >= dd) incl += o;
      }
      const uint32_t wflags = __ballot_sync(0xffffffffu, bad) ? 0x80000000u : 0u;
      const uint32_t wtime = __ballot_sync(0xffffffffu, tmo) ? 0x40000000u : 0u;
      if (lane == 31) warp_tot[warp] = incl | wflags | wtime;
      group_sync(bar_id);
      // lane i < 8 holds warp i's total: the group total, the totals of the
      // warps before this one and of the first block's warps, and the flags,
      // each one warp reduction
      const uint32_t xw = lane < kT / 32 ? warp_tot[lane] : 0u;
      const uint32_t vw = xw & 0x3FFFFFFFu;
      const uint32_t flagbits = __reduce_or_sync(0xffffffffu, xw);
      const uint32_t tot = __reduce_add_sync(0xffffffffu, vw);
      const uint32_t wpre = __reduce_add_sync(0xffffffffu, lane < warp ? vw : 0u);
      const uint32_t tot_first = __reduce_add_sync(0xffffffffu, lane < kFirstBlockWarps ? vw : 0u);
      if (flagbits & 0x40000000u) {
        // a bounded wait ran out: the group stops (uniformly) with the status
        // set, after a bounded wait for the next unit's copy issued at the top
        if (t == 0) {
          set_status(P.status, DF11_ERR_TIMEOUT);
          if (g + ngroups < s1) mbar_wait(bar_stage + 8 * (s ^ 1), ((it + 1) >> 1) & 1);
        }
        timed_out = true;
        break;
      }
      // the codes of the whole unit and of its first block must match the
      // block positions (every stored position is checked)
      const bool ok =
          table_ok && sane && !(flagbits >> 31) && tot == P1 - P0 && tot_first == PM - P0;
      // fused matmul: the previous unit's row sums (merged before the barrier)
      if constexpr (NB > 0) {
        if (have_prev && prev.ok) flush_matmul<NB>(prev, acc, P.m[prev.m], P.batch, t);
      }
      if (t == 0) {
        if (!ok) set_status(P.status, DF11_ERR_CORRUPT);
        // this unit's sign/mantissa bytes (the previous unit's merge is done),
        // rounded out to 16 B
        const uint32_t sm_lo = P0 & ~15u;
        uint32_t sm_bytes = sane ? (uint32_t)((((uint64_t)P1 + 15u) & ~15ull) - sm_lo) : 0u;
        DF11_GLOBAL_CHECK((uint64_t)sm_lo + sm_bytes <= ((M.n + 15) & ~15ull) + 16, sm_bytes = 0)
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        mbar_expect_tx(bar_sm, sm_bytes);
        if (sm_bytes) bulk_g2s(sm_a, M.sm + sm_lo, sm_bytes, bar_sm);
      }
      // ---- move this thread's exponents to its place in the linear row:
      // destination word i (from D / 4 on) is source words i-1 and i of the
      // private row, realigned with a funnel shift.  The first and the last
      // word may hold a neighbour's bytes too: they are OR-ed in (the row is
      // zero there); the words between belong to this thread alone and are
      // stored.  Bytes past the thread's count (codes trimmed above) are
      // masked off the last word.
      if (cnt && ok) {
        const uint32_t D = (P0 & 15u) + wpre + incl - cnt;
        const uint32_t sh = (D & 3u) * 8;
        const uint32_t la = lin_a + (D & ~3u);
        const uint32_t ndw = ((D + cnt - 1) >> 2) - (D >> 2) + 1;  // destination words
        const uint32_t nsw = (cnt + 3) >> 2;                        // source words
        const uint32_t lastmask = 0xFFFFFFFFu >> (8 * (3 - ((D + cnt - 1) & 3u)));
        uint32_t prevw = lds32(col_a);
        const uint32_t v0 = __funnelshift_l(0u, prevw, sh);
        red_or32(la, ndw == 1 ? (v0 & lastmask) : v0);
        uint32_t i = 1;
#pragma unroll 4
        for (; i + 1 < ndw; ++i) {
          const uint32_t cw = lds32(col_a + 128 * i);
          sts32(la + 4 * i, __funnelshift_l(prevw, cw, sh));
          prevw = cw;
        }
        if (ndw > 1) {
          const uint32_t cw = i < nsw ? lds32(col_a + 128 * i) : 0u;
          red_or32(la + 4 * i, __funnelshift_l(prevw, cw, sh) & lastmask);
        }
      }
      prev = Pending{P0, P1, M.out, ok, m, RL, CL, (uint32_t)M.n};
      have_prev = true;
    }
    // the group's last unit of this matrix
    if (!timed_out && have_prev) {
      group_sync(bar_id);
      const bool got = mbar_wait(bar_sm, (it - 1) & 1);
      if (!got) {
        if (lane == 0) set_status(P.status, DF11_ERR_TIMEOUT);
        timed_out = true;
      }
      if constexpr (NB == 0) {
        if (got && prev.ok) merge_unit(prev, lin_a, sm_a, t);
      } else {
        if (got && prev.ok) merge_unit_matmul<NB>(prev, lin_a, sm_a, t, acc, P.m[prev.m], P.batch);
        group_sync(bar_id);
        if (got && prev.ok) flush_matmul<NB>(prev, acc, P.m[prev.m], P.batch, t);
      }
    }
  }
}

#undef DF11_APPEND
#undef DF11_STEP

// ============================================================ decode with a run index
//
// The same work unit, group and pipeline as decode_kernel, with the run index
// (df11_build_run_index) fetched with the unit's stream bytes: thread t of a
// unit reads the first output of its run within its block, so it knows where
// its exponents go before it decodes them.  It decodes straight into the
// group's linear row at that place: the write-through store of each step is an
// OR (the row is zero where nothing was written, a word that only gains bits
// can be OR-ed again, and the words at a thread's two ends, shared with its
// neighbours, come out right in any order).  The steps whose codes may start
// past the thread's chunks (the last 11 bits of them) keep only the codes that
// start inside.  No private rows, no prefix sum and no relocation; two linear
// rows let the previous unit's merge overlap this unit's decode.

constexpr uint32_t kRunIndexStage = 2 * kUnitChunks / kCPT;          // 512 B: 256 uint16
constexpr uint32_t kStageBytesIdx = kStreamStage + kGapStage + kRunIndexStage + 16;
static_assert(kStageBytesIdx % 16 == 0, "stage alignment");
// a thread can write this far past its first output: 128 codes (1-bit codes
// over 128 bits) and the word holding the last of them
constexpr uint32_t kIdxRowSlack = 128 + 48;

// One group's shared memory for the indexed decoder (offsets from the group's
// base): two stages (stream + gaps + run index), the sign/mantissa bytes, two
// linear rows, mbarriers, positions, per-warp flags.
struct GroupLayoutIdx {
  uint32_t stage0, stage1, sm, lin0, lin1, bars, meta, flags, size;
};

__host__ __device__ inline GroupLayoutIdx group_layout_idx(uint32_t cap) {
  GroupLayoutIdx G;
  G.stage0 = 0;
  G.stage1 = kStageBytesIdx;
  G.sm = 2 * kStageBytesIdx;
  G.lin0 = round16(G.sm + cap + 32);
  G.lin1 = round16(G.lin0 + cap + kIdxRowSlack);
  G.bars = round16(G.lin1 + cap + kIdxRowSlack);
  G.meta = G.bars + 32;
  G.flags = G.meta + 64;
  G.size = (G.flags + 64 + 127u) & ~127u;
  return G;
}

// a * b + c (low word), kept on the multiply pipe
__device__ __forceinline__ uint32_t madlo(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t r;
  asm("mad.lo.u32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(c));
  return r;
}

// Append to the linear row through OR-ed write-through stores (see
// DF11_APPEND for the register side; here the row is contiguous).  The
// word's address, (nb2 bits 5..10) * 4 past row0, and the table address are
// computed with multiply-adds: the integer logic pipe is this loop's busiest.
#define DF11_APPEND_OR(xs, add)                                             \
  {                                                                         \
    const uint32_t lo = cur | __funnelshift_l(0u, (xs), nb);                \
    const uint32_t hi = __funnelshift_l((xs), 0u, nb);                      \
    red_or32(row_a, lo);                                                    \
    const uint32_t nb2 = nb + (add);                                        \
    row_a = madlo(madhi(nb2 << 21, 1u << 6, 0u), 4u, row0);                 \
    cur = ((nb ^ nb2) & 32u) ? hi : lo;                                     \
    nb = nb2;                                                               \
  }

#define DF11_LUT_ADDR(w) madlo(madhi((w), 1u << df11i::kLutBits, 0u), 8u, lut_a)

#define DF11_STEP_OR(hw, lw)                                                \
  {                                                                         \
    const uint32_t w = __funnelshift_l((lw), (hw), p);                      \
    const uint2 e = lds64(DF11_LUT_ADDR(w));                                \
    DF11_APPEND_OR(e.x, e.y)                                                \
    p = madhi(e.y, 1u << (32 - df11i::kCtrlUsedShift), p);                  \
  }

// A table step that keeps only the entry's codes starting before lim (room =
// lim - p <= kLutBits bits ahead): the first code always, each further one if
// its start field is below room (an absent code's field, 15, never is).
#define DF11_STEP_MASKED(hw, lw)                                            \
  {                                                                         \
    const uint32_t w = __funnelshift_l((lw), (hw), p);                      \
    const uint2 e = lds64(DF11_LUT_ADDR(w));                                \
    const uint32_t room = lim - p;                                          \
    const uint32_t nc = (e.y >> df11i::kCtrlCountShift) & 7u;               \
    uint32_t keep = 1u + (((e.y >> 12) & 15u) < room) +                     \
                    (((e.y >> 16) & 15u) < room) + (((e.y >> 20) & 15u) < room); \
    keep = min(keep, nc);                                                   \
    const uint32_t mask = keep >= 4u ? 0xFFFFFFFFu : ((1u << (8u * keep)) - 1u); \
    DF11_APPEND_OR(e.x & mask, 8u * keep)                                   \
    p = madhi(e.y, 1u << (32 - df11i::kCtrlUsedShift), p);                  \
  }

__global__ void __launch_bounds__(kT *kMaxGroups, 1) decode_idx_kernel(const __grid_constant__ DecParams P) {
  extern __shared__ __align__(128) uint8_t smem[];
  const uint32_t ngroups = blockDim.x / kT;
  const uint32_t grp = threadIdx.x / kT;
  const int t = (int)(threadIdx.x % kT), lane = t & 31, warp = t >> 5;
  const uint32_t cap = P.stage_cap;
  const GroupLayoutIdx GL = group_layout_idx(cap);
  const uint32_t sbase = smem_addr(smem);
  const uint32_t gofs = kTablesSmem + grp * GL.size;
  const uint32_t gbase = sbase + gofs;
  const DecodeTables &tab = *reinterpret_cast<const DecodeTables *>(smem);
  const uint32_t lut_a = sbase;  // lut is the first member of the tables
  const uint32_t bar_stage = gbase + GL.bars, bar_sm = gbase + GL.bars + 16;
  uint32_t *meta = reinterpret_cast<uint32_t *>(smem + gofs + GL.meta);
  uint32_t *wflags = reinterpret_cast<uint32_t *>(smem + gofs + GL.flags);
  const uint32_t sm_a = gbase + GL.sm;
  const uint32_t bar_id = 1 + grp;

  const uint64_t total = P.unit_start[P.count];
  const uint64_t g0 = (uint64_t)blockIdx.x * total / gridDim.x;
  const uint64_t g1 = (uint64_t)(blockIdx.x + 1) * total / gridDim.x;
  if (g0 >= g1) return;  // the same for every thread of the CTA
#ifdef DF11_CHECKED
  if (threadIdx.x == 0) {
    s_check_status = P.status;
    s_dyn_base = smem_addr(smem);
  }
  __syncthreads();
#endif

  // both linear rows start zeroed
  for (uint32_t k = t; k < (GL.bars - GL.lin0) / 16; k += kT) sts128_zero(gbase + GL.lin0 + 16 * k);
  if (t == 0) {
    mbar_init(bar_stage, 1);
    mbar_init(bar_stage + 8, 1);
    mbar_init(bar_sm, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }

  uint32_t it = 0;
  bool timed_out = false;
  uint32_t m = 0;
  while (m + 1 < P.count && g0 >= P.unit_start[m + 1]) ++m;
  for (; m < P.count && P.unit_start[m] < g1; ++m) {
    if (__syncthreads_or(timed_out)) return;
    if (t == 0) meta[4] = meta[12] = 0u;  // the two merge counters (used after a group barrier)
    const uint64_t s0 = max(g0, P.unit_start[m]), s1 = min(g1, P.unit_start[m + 1]);
    if (s0 >= s1) continue;
    const DecMat &M = P.m[m];
    {
      const uint4 *src = reinterpret_cast<const uint4 *>(M.tables);
      uint4 *dst = reinterpret_cast<uint4 *>(smem);
      for (uint32_t k = threadIdx.x; k < sizeof(DecodeTables) / 16; k += blockDim.x)
        dst[k] = __ldg(src + k);
    }
    __syncthreads();
    bool tbad = false;
    for (uint32_t k = threadIdx.x; k < (uint32_t)df11i::kLutSize; k += blockDim.x)
      tbad |= lut_entry_bad(tab.lut[k].y, P.min_len);
    const bool table_ok = !__syncthreads_or(tbad);
    const bool table_short = tab.max_len <= (uint32_t)df11i::kLutBits;

    const uint64_t first = s0 + grp;
    if (first >= s1) continue;
    uint32_t nxt_p0 = 0, nxt_p1 = 0, nxt_pm = 0;
    auto fetch_pos = [&](uint64_t g) {
      const uint32_t b0 = kUnitBlocks * (uint32_t)(g - P.unit_start[m]);
      DF11_GLOBAL_CHECK(b0 < M.n_blocks, return)
      nxt_p0 = __ldg(M.pos + b0);
      nxt_p1 = __ldg(M.pos + min(b0 + kUnitBlocks, M.n_blocks));
      nxt_pm = b0 + 1 < M.n_blocks ? __ldg(M.pos + b0 + 1) : nxt_p1;
    };
    auto issue_stream = [&](uint64_t g, uint32_t stage) {
      const uint32_t u = (uint32_t)(g - P.unit_start[m]);
      const uint32_t nb = min(kUnitBlocks, M.n_blocks - kUnitBlocks * u);
      const uint32_t sbytes = nb * kBlockStreamBytes + 16, gbytes = nb * kBlockGapBytes;
      const uint32_t ibytes = nb * (kRunIndexStage / kUnitBlocks);
      const uint32_t st = gbase + (stage ? GL.stage1 : GL.stage0);
      uint32_t *mt = meta + stage * 8;
      mt[0] = nxt_p0;
      mt[1] = nxt_p1;
      mt[2] = u;
      mt[3] = nxt_pm;
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      DF11_GLOBAL_CHECK((uint64_t)u * (8 * kUnitChunks) + sbytes <=
                                (uint64_t)kBlockStreamBytes * M.n_blocks + 16 &&
                            (uint64_t)u * kGapStage + gbytes <=
                                (uint64_t)kBlockGapBytes * M.n_blocks + 16,
                        {
                          mbar_expect_tx(bar_stage + 8 * stage, 0);
                          return;
                        })
#ifdef DF11_TEST_HOOKS
      mbar_expect_tx(bar_stage + 8 * stage, sbytes + gbytes + ibytes + P.starve_tx);
#else
      mbar_expect_tx(bar_stage + 8 * stage, sbytes + gbytes + ibytes);
#endif
      bulk_g2s(st, M.stream + (uint64_t)u * (8 * kUnitChunks), sbytes, bar_stage + 8 * stage);
      bulk_g2s(st + kStreamStage, M.gaps + (uint64_t)u * kGapStage, gbytes, bar_stage + 8 * stage);
      bulk_g2s(st + kStreamStage + kGapStage, M.run_index + (uint64_t)u * (kRunIndexStage / 2),
               ibytes, bar_stage + 8 * stage);
    };
    if (t == 0) {
      fetch_pos(first);
      issue_stream(first, it & 1);
      if (first + ngroups < s1) fetch_pos(first + ngroups);
    }
    group_sync(bar_id);

    // One group barrier per unit, at its end ([B]).  Everything a unit
    // reuses was last touched before the previous [B]: the stage and meta
    // slot the next copy goes to (read while decoding the unit before),
    // the linear row this unit decodes into (merged and cleared in the
    // previous iteration, or cleared after its [B] when rejected), and the
    // flag words (two sets, by the stage's parity).
    Pending prev{0, 0, nullptr, false, 0, 0, 0, 0};
    bool have_prev = false;
    for (uint64_t g = first; g < s1; g += ngroups, ++it) {
      const uint32_t s = it & 1;
      const uint32_t *mt = meta + s * 8;
      const uint32_t P0 = mt[0], P1 = mt[1], u = mt[2], PM = mt[3];
      const bool sane = P1 >= P0 && P1 <= M.n && P1 - P0 <= cap && PM >= P0 && PM <= P1;
      if (t == 0 && g + ngroups < s1) {
        issue_stream(g + ngroups, s ^ 1);
        if (g + 2 * ngroups < s1) fetch_pos(g + 2 * ngroups);
      }
      bool tmo = !mbar_wait(bar_stage + 8 * s, (it >> 1) & 1);
      const uint32_t lin_s = gbase + (s ? GL.lin1 : GL.lin0);

      // ---- this thread's two chunks, decoded straight into the linear row
      const uint32_t c0 = u * kUnitChunks + kCPT * t;
      bool bad = false;
      if (table_ok && sane && c0 < M.n_chunks) {
        const uint32_t st = gbase + (s ? GL.stage1 : GL.stage0);
        // the run's first output within its block and the next run's (or the
        // block's total after its last run)
        const uint32_t ia = st + kStreamStage + kGapStage + 2 * t;
        const uint32_t r = (uint32_t)t & 127u;
        const uint32_t btot = t < 128 ? PM - P0 : P1 - PM;
        const uint32_t two_idx = lds32(ia & ~3u);
        const uint32_t off = (t & 1) ? two_idx >> 16 : two_idx & 0xFFFFu;
        const uint32_t nxt = r == 127u ? btot : ((t & 1) ? lds32(ia + 2) & 0xFFFFu : two_idx >> 16);
        bad = off > nxt || nxt > btot || (r == 0u && off != 0u);
        if (!bad) {
          const uint32_t D = (P0 & 15u) + (t < 128 ? 0u : PM - P0) + off;
          const uint4 a4 = lds128(st + 16 * t);
          const uint32_t W0 = bswap32(a4.x), W1 = bswap32(a4.y), W2 = bswap32(a4.z),
                         W3 = bswap32(a4.w), W4 = bswap32(lds32(st + 16 * t + 16));
          const uint64_t avail = M.total_bits - 64ull * c0;
          const uint32_t lim = avail < 64u * kCPT ? (uint32_t)avail : 64u * kCPT;
          const uint32_t q = DF11_GAP_BITS * kCPT * t;
          const uint32_t ga = st + kStreamStage + (q >> 3);
          const uint32_t two = (lds8(ga) << 8) | lds8(ga + 1);
          const uint32_t gap = (two >> (11 - (q & 7u))) & 31u;
          const uint32_t row0 = lin_s + (D & ~3u);
          const uint32_t nb0 = 8u * (D & 3u);
          uint32_t p = gap, nb = nb0, cur = 0, row_a = row0;
          if (table_short) {
            // steps whose codes all start before lim, one loop per word; then
            // the last few steps, masked
            const uint32_t safe = lim > (uint32_t)df11i::kLutBits ? lim - df11i::kLutBits : 0u;
            const uint32_t l1 = min(safe, 32u), l2 = min(safe, 64u), l3 = min(safe, 96u);
#pragma unroll 1
            while (p < l1) DF11_STEP_OR(W0, W1)
#pragma unroll 1
            while (p < l2) DF11_STEP_OR(W1, W2)
#pragma unroll 1
            while (p < l3) DF11_STEP_OR(W2, W3)
#pragma unroll 1
            while (p < safe) DF11_STEP_OR(W3, W4)
#pragma unroll 1
            while (p < lim) {
              const uint32_t k = p >> 5;
              const uint32_t hw = k == 0 ? W0 : k == 1 ? W1 : k == 2 ? W2 : W3;
              const uint32_t lw = k == 0 ? W1 : k == 1 ? W2 : k == 2 ? W3 : W4;
              DF11_STEP_MASKED(hw, lw)
            }
          } else {
            // codes longer than the table's reach: per word a table loop that
            // leaves on a flagged entry, whose code the length search decodes
            // (a code starting before lim is the thread's whatever its
            // length); the last steps masked as above
            const uint32_t safe = lim > (uint32_t)df11i::kLutBits ? lim - df11i::kLutBits : 0u;
#pragma unroll 1
            while (p < lim) {
              const uint32_t k = p >> 5;
              const uint32_t hw = k == 0 ? W0 : k == 1 ? W1 : k == 2 ? W2 : W3;
              const uint32_t lw = k == 0 ? W1 : k == 1 ? W2 : k == 2 ? W3 : W4;
              if (p < safe) {
                // steps of word k whose codes all start before lim
                const uint32_t seg = min(safe, 32u * (k + 1));
                bool flagged = false;
#pragma unroll 1
                while (p < seg) {
                  const uint32_t w = __funnelshift_l(lw, hw, p);
                  const uint2 e = lds64(DF11_LUT_ADDR(w));
                  if (e.y & df11i::kCtrlLongFlag) {
                    flagged = true;
                    break;
                  }
                  DF11_APPEND_OR(e.x, e.y)
                  p = madhi(e.y, 1u << (32 - df11i::kCtrlUsedShift), p);
                }
                if (!flagged) continue;  // the next word's loop (words re-picked)
              } else {
                // p in [safe, lim): a table entry may hold the next thread's codes
                const uint32_t w = __funnelshift_l(lw, hw, p);
                const uint32_t ey = lds32(DF11_LUT_ADDR(w) + 4);
                if (!(ey & df11i::kCtrlLongFlag)) {
                  DF11_STEP_MASKED(hw, lw)
                  continue;
                }
              }
              // a flagged entry at p (inside word k): the length search
              const uint32_t w = __funnelshift_l(lw, hw, p);
              const uint32_t L = long_code_len(w, tab);
              if (L == 0) {
                bad = true;
                break;
              }
              const uint32_t x = tab.sym[((w >> (32 - L)) + tab.base[L]) & 0xFFu];
              DF11_APPEND_OR(x, 8u)
              p += L;
            }
          }
          red_or32(row_a, cur);  // the word being filled
          const uint32_t d = ((nb & 0x7FFu) - nb0) >> 3;
          bad |= d != nxt - off;
        }
      }
      // ---- the previous unit's merge (its row is the other one)
      if (have_prev) {
        // (warp-uniform: the claimed merge shuffles across the whole warp)
        if (!__all_sync(0xffffffffu, mbar_wait(bar_sm, (it - 1) & 1))) tmo = true;
        else if (prev.ok)
          merge_unit_claimed(prev, gbase + (s ? GL.lin0 : GL.lin1), sm_a, t, meta + (s ^ 1u) * 8 + 4);
      }
      // ---- [B] the group's flags
      const uint32_t wf = (__ballot_sync(0xffffffffu, bad) ? 1u : 0u) |
                          (__ballot_sync(0xffffffffu, tmo) ? 2u : 0u);
      uint32_t *wfl = wflags + 8 * s;
      if (lane == 0) wfl[warp] = wf;
      group_sync(bar_id);
      if (t == 0) meta[(s ^ 1u) * 8 + 4] = 0u;  // the merge counter of the unit just merged
      const uint32_t flagbits = __reduce_or_sync(0xffffffffu, lane < kT / 32 ? wfl[lane] : 0u);
      if (flagbits & 2u) {
        if (t == 0) {
          set_status(P.status, DF11_ERR_TIMEOUT);
          if (g + ngroups < s1) mbar_wait(bar_stage + 8 * (s ^ 1), ((it + 1) >> 1) & 1);
        }
        timed_out = true;
        break;
      }
      // every thread's count matched its run's share of the block positions
      const bool ok = table_ok && sane && !(flagbits & 1u);
      if (t == 0) {
        if (!ok) set_status(P.status, DF11_ERR_CORRUPT);
        const uint32_t sm_lo = P0 & ~15u;
        uint32_t sm_bytes = sane ? (uint32_t)((((uint64_t)P1 + 15u) & ~15ull) - sm_lo) : 0u;
        DF11_GLOBAL_CHECK((uint64_t)sm_lo + sm_bytes <= ((M.n + 15) & ~15ull) + 16, sm_bytes = 0)
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        mbar_expect_tx(bar_sm, sm_bytes);
        if (sm_bytes) bulk_g2s(sm_a, M.sm + sm_lo, sm_bytes, bar_sm);
      }
      // a rejected unit is not merged: its row is cleared here instead
      if (!ok)
        for (uint32_t k = t; k < (cap + kIdxRowSlack) / 16; k += kT) sts128_zero(lin_s + 16 * k);
      prev = Pending{P0, P1, M.out, ok, m, 0, 0, (uint32_t)M.n};
      have_prev = true;
    }
    if (!timed_out && have_prev) {
      group_sync(bar_id);
      const bool got = __all_sync(0xffffffffu, mbar_wait(bar_sm, (it - 1) & 1));
      if (!got) {
        if (lane == 0) set_status(P.status, DF11_ERR_TIMEOUT);
        timed_out = true;
      }
      if (got && prev.ok)
        merge_unit_claimed(prev, gbase + (((it - 1) & 1) ? GL.lin1 : GL.lin0), sm_a, t,
                           meta + ((it - 1) & 1u) * 8 + 4);
    }
  }
}

#undef DF11_APPEND_OR
#undef DF11_LUT_ADDR
#undef DF11_STEP_OR
#undef DF11_STEP_MASKED

// ============================================================ run index
//
// One CTA of 128 threads per block of 256 chunks at a time (persistent over a
// contiguous range of blocks, decode tables loaded once): thread r counts the
// codes that start in chunks 2r and 2r+1 (the decode steps without appends,
// the last entry trimmed at the end of the run), the CTA's exclusive prefix
// sum gives each run's first output within the block, and the block's total
// is checked against its stored positions.
constexpr int kRiThreads = DF11_BLOCK_CHUNKS / kCPT;  // 128
constexpr uint32_t kSegOut = DF11_SEGMENT;  // outputs per segment of the segment index
static_assert(kSegOut == 64, "segment index: code index >> 6 is its segment");

// kSeg = false: the run index (one uint16 per run).  kSeg = true: the
// segment index instead -- after the count pass and the block's scan each
// thread knows the output index of its run's first code, and a second pass
// over the run records the start bit of every code whose index is a
// multiple of 64 (the start of a segment).
template <bool kSeg>
__global__ void __launch_bounds__(kRiThreads) run_index_kernel(const __grid_constant__ DecParams P,
                                                              uint16_t *__restrict__ out,
                                                              uint32_t *__restrict__ seg) {
  __shared__ __align__(16) DecodeTables tab;
  __shared__ uint32_t s_warp[kRiThreads / 32];
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const DecMat &M = P.m[0];
  const uint32_t B = M.n_blocks;
  const uint32_t b0 = (uint32_t)((uint64_t)blockIdx.x * B / gridDim.x);
  const uint32_t b1 = (uint32_t)((uint64_t)(blockIdx.x + 1) * B / gridDim.x);
  if (b0 >= b1) return;
  {
    const uint4 *src = reinterpret_cast<const uint4 *>(M.tables);
    uint4 *dst = reinterpret_cast<uint4 *>(&tab);
    for (uint32_t k = t; k < sizeof(DecodeTables) / 16; k += kRiThreads) dst[k] = __ldg(src + k);
  }
  __syncthreads();
  bool tbad = false;
  for (uint32_t k = t; k < (uint32_t)df11i::kLutSize; k += kRiThreads)
    tbad |= lut_entry_bad(tab.lut[k].y, P.min_len);
  if (__syncthreads_or(tbad)) {
    if (t == 0) set_status(P.status, DF11_ERR_CORRUPT);
    return;
  }
  const bool table_short = tab.max_len <= (uint32_t)df11i::kLutBits;
  const uint64_t n_segs = (M.n + kSegOut - 1) / kSegOut;
  if (kSeg && blockIdx.x == 0 && t == 0) seg[n_segs] = (uint32_t)M.total_bits;
  for (uint32_t b = b0; b < b1; ++b) {
    const uint32_t c0 = b * DF11_BLOCK_CHUNKS + kCPT * t;
    uint32_t cnt = 0;
    bool bad = false;
    uint32_t W0 = 0, W1 = 0, W2 = 0, W3 = 0, W4 = 0, lim = 0, gap = 0;
    if (c0 < M.n_chunks) {
      // the run's 16 stream bytes and the next 4 (inside the stream's
      // allocation: whole blocks plus 16 bytes)
      const uint4 a4 = __ldg(reinterpret_cast<const uint4 *>(M.stream + 8ull * c0));
      W0 = bswap32(a4.x), W1 = bswap32(a4.y), W2 = bswap32(a4.z), W3 = bswap32(a4.w);
      W4 = bswap32(__ldg(reinterpret_cast<const uint32_t *>(M.stream + 8ull * c0 + 16)));
      const uint64_t avail = M.total_bits - 64ull * c0;
      lim = avail < 64u * kCPT ? (uint32_t)avail : 64u * kCPT;
      const uint64_t q = (uint64_t)DF11_GAP_BITS * c0;
      const uint32_t two = ((uint32_t)__ldg(M.gaps + (q >> 3)) << 8) | __ldg(M.gaps + (q >> 3) + 1);
      gap = (two >> (11 - (q & 7u))) & 31u;
      uint32_t p = gap, acc = 0, ctrl = 0;
#pragma unroll 1
      while (p < lim) {
        const uint32_t k = p >> 5;
        const uint32_t hw = k == 0 ? W0 : k == 1 ? W1 : k == 2 ? W2 : W3;
        const uint32_t lw = k == 0 ? W1 : k == 1 ? W2 : k == 2 ? W3 : W4;
        const uint32_t w = __funnelshift_l(lw, hw, p);
        const uint32_t ey = tab.lut[w >> (32 - df11i::kLutBits)].y;  // (static shared memory)
        if (!table_short && (ey & df11i::kCtrlLongFlag)) {
          const uint32_t L = long_code_len(w, tab);
          if (L == 0) {
            bad = true;
            break;
          }
          acc += 8u;
          ctrl = kLongCodeCtrl;
          p += L;
        } else {
          acc += ey;  // bits 0..10: 8 x the codes (the rest is never read)
          ctrl = ey;
          p = madhi(ey, 1u << (32 - df11i::kCtrlUsedShift), p);
        }
      }
      cnt = (acc & 0x7FFu) >> 3;
      const uint32_t ncodes = (ctrl >> df11i::kCtrlCountShift) & 7u;
      if (p > lim && ncodes) {
        const uint32_t pl = p - (ctrl >> df11i::kCtrlUsedShift);
        const uint32_t past = (uint32_t)(pl + ((ctrl >> 12) & 15u) >= lim) +
                              (uint32_t)(pl + ((ctrl >> 16) & 15u) >= lim) +
                              (uint32_t)(pl + ((ctrl >> 20) & 15u) >= lim);
        cnt -= past - (df11i::kLutMaxCodes - ncodes);
      }
    }
    uint32_t incl = cnt;
#pragma unroll
    for (int dd = 1; dd < 32; dd <<= 1) {
      const uint32_t o = __shfl_up_sync(0xffffffffu, incl, dd);
      if (lane >= dd) incl += o;
    }
    if (lane == 31) s_warp[warp] = incl;
    const bool any_bad = __syncthreads_or(bad);
    uint32_t pre = 0, tot = 0;
#pragma unroll
    for (int i = 0; i < kRiThreads / 32; ++i) {
      pre += i < warp ? s_warp[i] : 0u;
      tot += s_warp[i];
    }
    const uint32_t excl = pre + incl - cnt;
    const uint32_t pb = __ldg(M.pos + b);
    const bool block_bad = any_bad || tot != __ldg(M.pos + b + 1) - pb || tot > 0xFFFFu;
    if (!kSeg) out[(uint64_t)b * kRiThreads + t] = (uint16_t)excl;
    if (t == 0 && block_bad) set_status(P.status, DF11_ERR_CORRUPT);
    if (kSeg && !block_bad && c0 < M.n_chunks) {
      // second pass: the codes that start in this run, with their output
      // indices; a LUT entry holds at most 4 codes, so at most one of them
      // starts a segment
      uint64_t i = (uint64_t)pb + excl;
      uint32_t p = gap;
#pragma unroll 1
      while (p < lim) {
        const uint32_t k = p >> 5;
        const uint32_t hw = k == 0 ? W0 : k == 1 ? W1 : k == 2 ? W2 : W3;
        const uint32_t lw = k == 0 ? W1 : k == 1 ? W2 : k == 2 ? W3 : W4;
        const uint32_t w = __funnelshift_l(lw, hw, p);
        const uint32_t ey = tab.lut[w >> (32 - df11i::kLutBits)].y;
        uint32_t nc, adv;
        if (!table_short && (ey & df11i::kCtrlLongFlag)) {
          nc = 1u;
          adv = long_code_len(w, tab);
          if (adv == 0) break;  // reported by the count pass
        } else {
          nc = (ey >> df11i::kCtrlCountShift) & 7u;
          adv = ey >> df11i::kCtrlUsedShift;
        }
        const uint32_t j = (uint32_t)(-i) & (kSegOut - 1);  // first code here at a multiple of 64
        if (j < nc) {
          const uint32_t st = j == 0 ? 0u : (ey >> (8 + 4 * j)) & 15u;  // its start in the window
          if (p + st < lim && ((i + j) >> 6) < n_segs)
            seg[(i + j) >> 6] = (uint32_t)(64ull * c0) + p + st;
        }
        i += nc;
        p += adv;
      }
    }
    __syncthreads();  // s_warp is reused by the next block
  }
}

// ============================================================ segment decoder
//
// With the segment index (the stream bit at which every 64th code starts),
// each lane of a warp decodes one segment -- exactly 64 codes, or the
// matrix's last few -- into its own exponent row, checks that it ended
// where the next segment begins, and merges the row with the segment's
// sign/mantissa bytes into 128 bytes of BF16.  A warp takes a unit of 32
// consecutive segments (2048 outputs): their stream bits are one contiguous
// range, copied into the warp's shared memory (cp.async) while the warp
// decodes the unit before; the unit's sign/mantissa bytes are copied while
// it decodes.  Nothing is counted, scanned or relocated, and the warps of a
// CTA meet only when the CTA moves on to another matrix (its tables).
constexpr uint32_t kSegWarps = 32;
constexpr uint32_t kSegThreads = 32 * kSegWarps;
constexpr uint32_t kSegUnit = 32 * kSegOut;          // outputs per warp unit
constexpr uint32_t kSegRowWords = kSegOut / 4;       // exponent words per lane
constexpr uint32_t kSegStage = 1024;                 // stream bytes per stage
constexpr uint32_t kSegWarpBytes = 128 * kSegRowWords + kSegUnit + 2 * kSegStage;
constexpr uint32_t kSegSmem = kTablesSmem + kSegWarps * kSegWarpBytes;
static_assert(kSegWarpBytes % 16 == 0, "segment decoder layout");

__device__ __forceinline__ void seg_cp16(uint32_t dst, const void *src) {
  DF11_SMEM_CHECK(dst, 16, return)
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void seg_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void seg_wait_prev() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }
__device__ __forceinline__ void seg_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

#define DF11_LUT_ADDR(w) madlo(madhi((w), 1u << df11i::kLutBits, 0u), 8u, lut_a)

// Append `add` bits (whole exponent bytes, low byte first) of xs at bit nb of
// the lane's exponent row (word w at row_a + row_stride * w); the word being
// filled is kept in cur and stored whole at every step.
#define DF11_SEG_APPEND(xs, add)                                            \
  {                                                                         \
    const uint32_t lo4 = cur | __funnelshift_l(0u, (xs), nb);               \
    const uint32_t hi4 = __funnelshift_l((xs), 0u, nb);                     \
    sts32(row_a + (nb >> 5) * row_stride, lo4);                             \
    const uint32_t nb2 = nb + (add);                                        \
    cur = ((nb ^ nb2) & 32u) ? hi4 : lo4;                                   \
    nb = nb2;                                                               \
  }

// Advance the window to bit pn; a step moves at most 32 bits, so at most one
// word boundary is crossed.
#define DF11_SEG_ADVANCE(pn)                                                \
  {                                                                         \
    if (((pn) >> 5) != (p >> 5)) {                                          \
      hw = lw;                                                              \
      lw = nxt;                                                             \
      nxt = word(((pn) >> 5) + 2u);                                         \
    }                                                                       \
    p = (pn);                                                               \
  }

// One lane's segment: cnt (<= 64) codes from stream bit p (relative to the
// words word(k) returns, byte-swapped to MSB-first; hw, lw and nxt are words
// p/32, p/32 + 1 and p/32 + 2), exponents into the lane's row.  True when
// exactly cnt codes were decoded and the last one ended at pend (where the
// next segment starts).
template <class WordFn>
__device__ __forceinline__ bool seg_decode_lane(uint32_t p, uint32_t pend, uint32_t cnt,
                                                bool table_short, const DecodeTables &tab,
                                                uint32_t lut_a, uint32_t row_a, uint32_t row_stride,
                                                WordFn word, uint32_t hw, uint32_t lw,
                                                uint32_t nxt) {
  uint32_t nb = 0, cur = 0;
  const uint32_t nb_end = 8u * cnt;
  if (table_short) {
    // whole table entries while at least 4 codes remain
    const int32_t nb_fast = 8 * ((int32_t)cnt - 4);
#pragma unroll 1
    while ((int32_t)nb <= nb_fast && p < pend) {
      const uint32_t w = __funnelshift_l(lw, hw, p);
      const uint2 en = lds64(DF11_LUT_ADDR(w));
      DF11_SEG_APPEND(en.x, en.y & 0x38u)
      const uint32_t pn = madhi(en.y, 1u << (32 - df11i::kCtrlUsedShift), p);
      DF11_SEG_ADVANCE(pn)
    }
  }
  // the last codes (and codes longer than the table's reach): keep only as
  // many of an entry's codes as remain
#pragma unroll 1
  while (nb < nb_end && p < pend) {
    const uint32_t w = __funnelshift_l(lw, hw, p);
    const uint2 en = lds64(DF11_LUT_ADDR(w));
    uint32_t adv;
    if (!table_short && (en.y & df11i::kCtrlLongFlag)) {
      const uint32_t L = long_code_len(w, tab);
      if (L == 0) break;  // no code: reported (nb short of nb_end)
      const uint32_t x = tab.sym[((w >> (32 - L)) + tab.base[L]) & 0xFFu];
      DF11_SEG_APPEND(x, 8u)
      adv = L;
    } else {
      const uint32_t nc = (en.y >> df11i::kCtrlCountShift) & 7u;
      const uint32_t keep = min(nc, (nb_end - nb) >> 3);
      const uint32_t mask = keep >= 4u ? 0xFFFFFFFFu : ((1u << (8u * keep)) - 1u);
      DF11_SEG_APPEND(en.x & mask, 8u * keep)
      adv = keep < nc ? (en.y >> (8u + 4u * keep)) & 15u : en.y >> df11i::kCtrlUsedShift;
    }
    const uint32_t pn = p + adv;
    DF11_SEG_ADVANCE(pn)
  }
  if (nb & 31u) sts32(row_a + (nb >> 5) * row_stride, cur);  // the word being filled
  return nb == nb_end && p == pend;
}

__global__ void __launch_bounds__(kSegThreads, 1) decode_seg_kernel(const __grid_constant__ DecParams P) {
  extern __shared__ __align__(128) uint8_t smem[];
  const uint32_t warp = threadIdx.x >> 5, lane = threadIdx.x & 31u;
  const uint32_t sbase = smem_addr(smem);
  const DecodeTables &tab = *reinterpret_cast<const DecodeTables *>(smem);
  const uint32_t lut_a = sbase;  // lut is the first member of the tables
  const uint32_t wb = sbase + kTablesSmem + warp * kSegWarpBytes;
  const uint32_t row_a = wb + 4u * lane;                // exponent word w: row_a + 128 w
  const uint32_t sm_a = wb + 128u * kSegRowWords;       // sign/mantissa piece q of lane l:
                                                        // sm_a + 16 (32 q + l)
  const uint32_t stage_a = sm_a + kSegUnit;             // stream stages 0 and 1

  const uint64_t total = P.unit_start[P.count];
  const uint64_t g0 = (uint64_t)blockIdx.x * total / gridDim.x;
  const uint64_t g1 = (uint64_t)(blockIdx.x + 1) * total / gridDim.x;
  if (g0 >= g1) return;  // the same for every thread of the CTA
#ifdef DF11_CHECKED
  if (threadIdx.x == 0) {
    s_check_status = P.status;
    s_dyn_base = smem_addr(smem);
  }
  __syncthreads();
#endif
  uint32_t m = 0;
  while (m + 1 < P.count && g0 >= P.unit_start[m + 1]) ++m;
  for (; m < P.count && P.unit_start[m] < g1; ++m) {
    const uint64_t s0 = max(g0, P.unit_start[m]), s1 = min(g1, P.unit_start[m + 1]);
    __syncthreads();  // every warp is done with the previous matrix's tables
    if (s0 >= s1) continue;
    const DecMat &M = P.m[m];
    {
      const uint4 *src = reinterpret_cast<const uint4 *>(M.tables);
      uint4 *dst = reinterpret_cast<uint4 *>(smem);
      for (uint32_t k = threadIdx.x; k < sizeof(DecodeTables) / 16; k += blockDim.x)
        dst[k] = __ldg(src + k);
    }
    __syncthreads();
    bool tbad = false;
    for (uint32_t k = threadIdx.x; k < (uint32_t)df11i::kLutSize; k += blockDim.x)
      tbad |= lut_entry_bad(tab.lut[k].y, P.min_len);
    const bool table_ok = !__syncthreads_or(tbad);
    const bool table_short = tab.max_len <= (uint32_t)df11i::kLutBits;

    const uint64_t ubase = P.unit_start[m];
    const uint64_t first = s0 + warp;
    if (first >= s1) continue;
    const uint32_t S = M.n_segs;
    const uint64_t alloc = 2048ull * M.n_blocks + 16;  // the stream's allocation (bytes)
    // this lane's segment start and the unit's end (the next unit's first
    // segment start, or total_bits), as absolute stream bits
    auto bounds = [&](uint64_t g, uint32_t &a, uint32_t &E) {
      const uint64_t j0 = (uint64_t)kSegWarps * (g - ubase);
      a = __ldg(M.seg + min(j0 + lane, (uint64_t)S));
      E = __ldg(M.seg + min(j0 + 32, (uint64_t)S));
    };
    // the unit's stream bytes [lo, hi) into a stage, when they fit; staged
    // is false otherwise (the unit then reads the stream from global memory)
    auto stage_in = [&](uint32_t a, uint32_t E, uint32_t st, uint32_t &lo, bool &staged) {
      const uint32_t a0 = __shfl_sync(0xffffffffu, a, 0);
      const bool sane = a0 <= E && E <= M.total_bits;
      lo = sane ? (a0 >> 3) & ~15u : 0u;
      const uint64_t hi = min((uint64_t)((4ull * ((E >> 5) + 3u) + 15u) & ~15ull), alloc);
      const uint32_t size = sane && hi > lo ? (uint32_t)(hi - lo) : 0u;
      staged = size <= kSegStage;
      if (staged)
        for (uint32_t q = lane; 16u * q < size; q += 32u) seg_cp16(st + 16u * q, M.stream + lo + 16u * q);
    };

    uint64_t g = first;
    uint32_t a, E, lo;
    bool staged;
    bounds(g, a, E);
    stage_in(a, E, stage_a, lo, staged);
    seg_commit();
    uint32_t an = 0, En = 0;
    if (g + kSegWarps < s1) bounds(g + kSegWarps, an, En);
    for (uint32_t it = 0; g < s1; g += kSegWarps, ++it) {
      const uint64_t j = (uint64_t)kSegWarps * (g - ubase) + lane;  // this lane's segment
      const uint32_t cnt = j < S ? (uint32_t)min((uint64_t)kSegOut, M.n - kSegOut * j) : 0u;
      // this unit's sign/mantissa bytes and the next unit's stream
      for (uint32_t q = 0; q < 4u; ++q)
        if (16u * q < cnt) seg_cp16(sm_a + 16u * (32u * q + lane), M.sm + kSegOut * j + 16u * q);
      uint32_t lo_n = 0;
      bool staged_n = true;
      if (g + kSegWarps < s1) stage_in(an, En, stage_a + kSegStage * ((it + 1) & 1u), lo_n, staged_n);
      seg_commit();
      uint32_t an2 = 0, En2 = 0;
      if (g + 2 * kSegWarps < s1) bounds(g + 2 * kSegWarps, an2, En2);
      seg_wait_prev();  // this unit's stream
      __syncwarp();

      // ---- decode this lane's segment into its exponent row
      const uint32_t st = stage_a + kSegStage * (it & 1u);
      const uint32_t a_next = __shfl_down_sync(0xffffffffu, a, 1);  // every lane takes part
      const uint32_t e = lane < 31u ? a_next : E;
      const uint32_t lo_bits = 8u * lo;
      const uint64_t gl_words = (alloc - lo) / 4;  // global words from lo (lo < alloc)
      const uint32_t *gsrc = reinterpret_cast<const uint32_t *>(M.stream + lo);
      auto word = [&](uint32_t k) -> uint32_t {
        return bswap32(staged ? lds32(st + 4u * min(k, kSegStage / 4 - 1))
                              : __ldg(gsrc + min((uint64_t)k, gl_words - 1)));
      };
      bool ok = table_ok && a >= lo_bits && a <= e && e <= M.total_bits &&
                e - a <= (uint64_t)DF11_MAX_CODE_LEN * cnt;
      if (cnt && ok) {
        const uint32_t p = a - lo_bits;
        ok = seg_decode_lane(p, e - lo_bits, cnt, table_short, tab, lut_a, row_a, 128u, word,
                             word(p >> 5), word((p >> 5) + 1u), word((p >> 5) + 2u));
      }
      if (__ballot_sync(0xffffffffu, cnt && !ok) && lane == 0) set_status(P.status, DF11_ERR_CORRUPT);

      // ---- merge: exponents + sign/mantissa -> BF16, 16 outputs at a time
      seg_wait_all();  // this unit's sign/mantissa bytes (and the next unit's stream)
      if (cnt && ok) {
        uint16_t *o = M.out + kSegOut * j;
#pragma unroll
        for (uint32_t q = 0; q < 4u; ++q) {
          if (16u * q < cnt) {
            const uint4 sv = lds128(sm_a + 16u * (32u * q + lane));
            const uint32_t e0 = lds32(row_a + 128u * (4u * q)), e1 = lds32(row_a + 128u * (4u * q + 1u)),
                           e2 = lds32(row_a + 128u * (4u * q + 2u)),
                           e3 = lds32(row_a + 128u * (4u * q + 3u));
            uint4 r0, r1;
            merge4(e0, sv.x, r0.x, r0.y);
            merge4(e1, sv.y, r0.z, r0.w);
            merge4(e2, sv.z, r1.x, r1.y);
            merge4(e3, sv.w, r1.z, r1.w);
            if (16u * q + 16u <= cnt) {
              DF11_GLOBAL_CHECK(kSegOut * j + 16u * q + 16u <= M.n, continue)
              reinterpret_cast<uint4 *>(o + 16u * q)[0] = r0;
              reinterpret_cast<uint4 *>(o + 16u * q)[1] = r1;
            } else {
              const uint32_t wv[8] = {r0.x, r0.y, r0.z, r0.w, r1.x, r1.y, r1.z, r1.w};
#pragma unroll
              for (uint32_t i = 0; i < 16u; ++i)
                if (16u * q + i < cnt) o[16u * q + i] = (uint16_t)(wv[i >> 1] >> (16u * (i & 1u)));
            }
          }
        }
      }
      __syncwarp();  // the stage and the sign/mantissa pieces are refilled next
      a = an;
      E = En;
      lo = lo_n;
      staged = staged_n;
      an = an2;
      En = En2;
    }
    seg_wait_all();
  }
}

#undef DF11_SEG_APPEND
#undef DF11_SEG_ADVANCE
#undef DF11_LUT_ADDR

// ============================================================ launch helpers

// decode_kernel instantiations: regions of codes >= 2 bits and >= 1 bit
constexpr int kMaxWords2 = 17;  // region_bytes_for(2) / 4
constexpr int kMaxWords1 = 33;  // region_bytes_for(1) / 4
static_assert(region_bytes_for(2) == 4 * kMaxWords2 && region_bytes_for(1) == 4 * kMaxWords1,
              "private region sizes");

using DecodeKernel = void (*)(DecParams);

// The instantiation for a batch: regions for codes of >= 2 bits or of 1 bit
// (wide), and the epilogue (0: store BF16; NB: matmul with up to NB rows).
DecodeKernel decode_kernel_for(bool wide, uint32_t nb) {
  switch (nb) {
    case 0: return wide ? decode_kernel<kMaxWords1, 0> : decode_kernel<kMaxWords2, 0>;
    case 1: return wide ? decode_kernel<kMaxWords1, 1> : decode_kernel<kMaxWords2, 1>;
    case 2: return wide ? decode_kernel<kMaxWords1, 2> : decode_kernel<kMaxWords2, 2>;
    case 4: return wide ? decode_kernel<kMaxWords1, 4> : decode_kernel<kMaxWords2, 4>;
    default: return wide ? decode_kernel<kMaxWords1, 8> : decode_kernel<kMaxWords2, 8>;
  }
}

struct DeviceInfo {
  int sms = 0;
  int smem_optin = 0;  // largest dynamic shared memory per decode CTA
  bool configured = false;
};

std::mutex g_mu;
DeviceInfo g_dev[64];

df11_status device_info(int *dev, int *sms, int *smem_optin = nullptr) {
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
    if (cudaDeviceGetAttribute(&d.smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, *dev) !=
        cudaSuccess)
      return DF11_ERR_CUDA;
    // the decode kernels' static shared memory (the checked build has some)
    // comes out of the same per-CTA limit
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, decode_kernel_for(false, 0)) != cudaSuccess) return DF11_ERR_CUDA;
    d.smem_optin -= (int)fa.sharedSizeBytes;
    if (cudaFuncSetAttribute(hist_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kHistSmem) != cudaSuccess)
      return DF11_ERR_CUDA;
    for (int wide = 0; wide < 2; ++wide)
      for (uint32_t nb : {0u, 1u, 2u, 4u, 8u})
        if (cudaFuncSetAttribute(decode_kernel_for(wide != 0, nb),
                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 d.smem_optin) != cudaSuccess)
          return DF11_ERR_CUDA;
    if (cudaFuncSetAttribute(decode_idx_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             d.smem_optin) != cudaSuccess)
      return DF11_ERR_CUDA;
    if (d.smem_optin >= (int)kSegSmem &&
        cudaFuncSetAttribute(decode_seg_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kSegSmem) != cudaSuccess)
      return DF11_ERR_CUDA;
    d.configured = true;
  }
  *sms = d.sms;
  if (smem_optin) *smem_optin = d.smem_optin;
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
    const uint64_t vec_warps = cdiv(n >> 3, kHistUnroll * 32);
    uint64_t grid = (uint64_t)sms * 3;
    grid = vec_warps ? std::min<uint64_t>(grid, cdiv(vec_warps, kHistWarps)) : 1;
    if (grid < 1) grid = 1;
    hist_kernel<<<(unsigned)grid, kHistThreads, kHistSmem, s>>>(d_w, n, h);
  }
  return launch_status();
}

namespace {

// The codebook of the launch parameters: lengths up to the format's limit,
// codes that fit their length, left-justified in 32 bits for the packer.
df11_status host_enc_codebook(const df11_codebook *cb, EncCodebook *ecb) {
  for (int i = 0; i < 256; ++i) {
    const uint32_t L = cb->len[i];
    if (L > DF11_MAX_CODE_LEN || (L < 32 && (cb->code[i] >> L) != 0)) return DF11_ERR_INVALID_ARG;
    ecb->code[i] = L ? cb->code[i] << (32 - L) : 0u;
    ecb->len[i] = (uint8_t)L;
  }
  return DF11_OK;
}

df11_status check_encode_out(const uint16_t *d_w, uint64_t n, uint64_t total_bits,
                             const df11_encoded *out) {
  if ((n && (!d_w || !aligned16(d_w))) || !out->stream || !out->gaps || !out->block_pos ||
      !out->sign_mantissa)
    return DF11_ERR_INVALID_ARG;
  if (!aligned16(out->stream) || !aligned16(out->gaps) || !aligned16(out->block_pos) ||
      !aligned16(out->sign_mantissa))
    return DF11_ERR_INVALID_ARG;
  if (total_bits > n * (uint64_t)DF11_MAX_CODE_LEN || (n && total_bits < n))
    return DF11_ERR_INVALID_ARG;
  return DF11_OK;
}

// Length sums per tile (clearing the stream and gap buffers), their prefix
// sum, packing, and the largest block.  ws: n_tiles + 1 uint64 of scratch.
df11_status launch_encode(const uint16_t *d_w, uint64_t n, const EncCodebook &ecb,
                          const df11_codebook *dcb, uint64_t total_bits, const df11_encoded *out,
                          uint64_t *ws, uint32_t *d_status, cudaStream_t s) {
  const uint64_t n_tiles = cdiv(n, df11i::kEncTile);
  const uint64_t C = cdiv(total_bits, 64);
  const uint64_t B = cdiv(C, DF11_BLOCK_CHUNKS);
  // the stream and gap allocations of the format (df11_encoded_sizes)
  const uint64_t stream_alloc = (uint64_t)kBlockStreamBytes * B + 16;
  const uint64_t gaps_alloc = (uint64_t)kBlockGapBytes * B + 16;
  const uint64_t grid1 = std::max<uint64_t>(n_tiles, 1);
  enc_sum_kernel<<<(unsigned)grid1, df11i::kEncThreads, 0, s>>>(
      d_w, n, ecb, dcb, ws, n_tiles, reinterpret_cast<uint4 *>(out->stream), stream_alloc / 16,
      reinterpret_cast<uint4 *>(out->gaps), gaps_alloc / 16, d_status);
  enc_scan_kernel<<<1, kScanThreads, 0, s>>>(ws, n_tiles, total_bits, out->block_pos, B, n,
                                            d_status, out->block_max);
  if (n_tiles)
    enc_pack_kernel<<<(unsigned)n_tiles, df11i::kEncThreads, 0, s>>>(
        d_w, n, ecb, dcb, ws, total_bits, out->stream, stream_alloc, out->gaps, gaps_alloc,
        out->block_pos, B, out->sign_mantissa);
  if (out->block_max && B)
    enc_block_max_kernel<<<(unsigned)std::min<uint64_t>(cdiv(B, 256), 1024), 256, 0, s>>>(
        out->block_pos, B, out->block_max);
  return launch_status();
}

}  // namespace

extern "C" df11_status df11_encode(const uint16_t *d_w, uint64_t n, const df11_codebook *cb,
                                   uint64_t total_bits, const df11_encoded *out, void *d_workspace,
                                   size_t workspace_bytes, uint32_t *d_status,
                                   df11_stream_t stream) {
  if (!cb || !out || !d_status) return DF11_ERR_INVALID_ARG;
  if (n > DF11_MAX_N) return DF11_ERR_TOO_LARGE;
  df11_status st = check_encode_out(d_w, n, total_bits, out);
  if (st != DF11_OK) return st;
  if (!d_workspace || !aligned16(d_workspace)) return DF11_ERR_INVALID_ARG;
  if (workspace_bytes < 8 * (cdiv(n, df11i::kEncTile) + 1)) return DF11_ERR_INVALID_ARG;
  EncCodebook ecb;
  if ((st = host_enc_codebook(cb, &ecb)) != DF11_OK) return st;
  int dev, sms;
  if ((st = device_info(&dev, &sms)) != DF11_OK) return st;
  return launch_encode(d_w, n, ecb, nullptr, total_bits, out,
                       reinterpret_cast<uint64_t *>(d_workspace), d_status,
                       reinterpret_cast<cudaStream_t>(stream));
}

extern "C" df11_status df11_encode_device_codebook(const uint16_t *d_w, uint64_t n,
                                                   const df11_codebook *d_cb, uint64_t total_bits,
                                                   const df11_encoded *out, void *d_workspace,
                                                   size_t workspace_bytes, uint32_t *d_status,
                                                   df11_stream_t stream) {
  if (!d_cb || !out || !d_status || ((uintptr_t)d_cb & 3u)) return DF11_ERR_INVALID_ARG;
  if (n > DF11_MAX_N) return DF11_ERR_TOO_LARGE;
  df11_status st = check_encode_out(d_w, n, total_bits, out);
  if (st != DF11_OK) return st;
  if (!d_workspace || !aligned16(d_workspace)) return DF11_ERR_INVALID_ARG;
  if (workspace_bytes < 8 * (cdiv(n, df11i::kEncTile) + 1)) return DF11_ERR_INVALID_ARG;
  int dev, sms;
  if ((st = device_info(&dev, &sms)) != DF11_OK) return st;
  EncCodebook unused{};
  return launch_encode(d_w, n, unused, d_cb, total_bits, out,
                       reinterpret_cast<uint64_t *>(d_workspace), d_status,
                       reinterpret_cast<cudaStream_t>(stream));
}

extern "C" df11_status df11_build_codebook_device(const uint64_t *d_hist256, uint32_t cap,
                                                  df11_codebook *d_cb, void *d_tables,
                                                  uint64_t *d_total_bits, uint32_t *d_status,
                                                  df11_stream_t stream) {
  if (!d_hist256 || !d_cb || !d_tables || !d_total_bits || cap < 1 || cap > DF11_MAX_CODE_LEN)
    return DF11_ERR_INVALID_ARG;
  if (((uintptr_t)d_hist256 & 7u) || ((uintptr_t)d_cb & 3u) || !aligned16(d_tables) ||
      ((uintptr_t)d_total_bits & 7u))
    return DF11_ERR_INVALID_ARG;
  int dev, sms;
  df11_status st = device_info(&dev, &sms);
  if (st != DF11_OK) return st;
  codebook_kernel<<<1, kCbThreads, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      d_hist256, cap, d_cb, reinterpret_cast<DecodeTables *>(d_tables), d_total_bits, d_status);
  return launch_status();
}

namespace {

// Shared by df11_decode_block_batch (io == nullptr: BF16 stored to d_outs)
// and df11_decode_matmul_batch (d_outs == nullptr: products added to io[i].y).
df11_status launch_decode(const df11_matrix *ms, uint32_t count, uint16_t *const *d_outs,
                          const df11_matmul_io *io, uint32_t batch, uint32_t *d_status,
                          df11_stream_t stream, uint32_t starve_tx = 0) {
  if (count == 0) return DF11_OK;
  if (!ms || (!d_outs && !io)) return DF11_ERR_INVALID_ARG;
  const uint32_t nb = io ? (batch <= 1 ? 1u : batch <= 2 ? 2u : batch <= 4 ? 4u : 8u) : 0u;
  if (io && (batch < 1 || batch > DF11_MATMUL_MAX_BATCH)) return DF11_ERR_INVALID_ARG;
  int dev, sms, smem_optin;
  df11_status st = device_info(&dev, &sms, &smem_optin);
  if (st != DF11_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  for (uint32_t first = 0; first < count; first += DF11_MAX_BATCH) {
    const uint32_t k = std::min<uint32_t>(DF11_MAX_BATCH, count - first);
    DecParams P;
    P.count = 0;
    P.status = d_status;
    P.unit_start[0] = 0;
#ifdef DF11_TEST_HOOKS
    P.starve_tx = starve_tx;
#else
    (void)starve_tx;
#endif
    uint32_t min_len = DF11_MAX_CODE_LEN;
    uint32_t unit_codes = 0;  // staging size: most codes in one unit of the batch
    bool indexed = io == nullptr;  // every matrix has a run index (plain decode only)
    bool segmented = io == nullptr;  // every matrix has a segment index (plain decode only)
    for (uint32_t i = 0; i < k; ++i) {
      const df11_matrix &m = ms[first + i];
      if (m.n > DF11_MAX_N) return DF11_ERR_TOO_LARGE;
      if (m.n == 0) continue;
      if (!m.stream || !m.gaps || !m.block_pos || !m.sign_mantissa || !m.tables)
        return DF11_ERR_INVALID_ARG;
      if (!aligned16(m.stream) || !aligned16(m.gaps) || !aligned16(m.sign_mantissa) ||
          !aligned16(m.tables) || ((uintptr_t)m.block_pos & 3u) || !aligned16(m.run_index) ||
          ((uintptr_t)m.seg_index & 3u))
        return DF11_ERR_INVALID_ARG;
      indexed = indexed && m.run_index != nullptr;
      segmented = segmented && m.seg_index != nullptr && m.total_bits <= 0xFFFFFFFFull;
      if (io) {
        // the matrix is rows x cols; activations and sums 16-byte aligned
        const df11_matmul_io &q = io[first + i];
        if ((uint64_t)q.rows * q.cols != m.n || q.cols % 8 || q.cols < kMinMatmulCols || !q.x ||
            !q.y || !aligned16(q.x) || ((uintptr_t)q.y & 3u))
          return DF11_ERR_INVALID_ARG;
      } else if (!d_outs[first + i] || !aligned16(d_outs[first + i])) {
        return DF11_ERR_INVALID_ARG;
      }
      // a complete code over at most 256 values has a code of at most 8 bits
      if (m.min_len < 1 || m.min_len > 8) return DF11_ERR_INVALID_ARG;
      if (m.total_bits < m.n * (uint64_t)m.min_len || m.total_bits > m.n * 32ull)
        return DF11_ERR_INVALID_ARG;
      // codes that can start in one block / one unit
      const uint32_t worst_block = (uint32_t)cdiv(64, m.min_len) * DF11_BLOCK_CHUNKS;
      const uint32_t worst_unit = (uint32_t)cdiv(64 * kCPT, m.min_len) * kT;
      if (m.max_block_codes > worst_block) return DF11_ERR_INVALID_ARG;
      unit_codes = std::max(unit_codes, m.max_block_codes
                                            ? std::min(kUnitBlocks * m.max_block_codes, worst_unit)
                                            : worst_unit);
      const uint64_t C = cdiv(m.total_bits, 64);
      const uint64_t B = cdiv(C, DF11_BLOCK_CHUNKS);
      if (C >= (1ull << 31)) return DF11_ERR_TOO_LARGE;
      DecMat &d = P.m[P.count];
      d.stream = m.stream;
      d.gaps = m.gaps;
      d.pos = m.block_pos;
      d.sm = m.sign_mantissa;
      d.tables = reinterpret_cast<const DecodeTables *>(m.tables);
      d.run_index = m.run_index;
      d.seg = m.seg_index;
      d.n_segs = (uint32_t)cdiv(m.n, kSegOut);
      d.out = io ? nullptr : d_outs[first + i];
      d.rows = io ? io[first + i].rows : 0u;
      d.cols = io ? io[first + i].cols : 1u;
      d.x = io ? io[first + i].x : nullptr;
      d.y = io ? io[first + i].y : nullptr;
      d.n = m.n;
      d.total_bits = m.total_bits;
      d.n_chunks = (uint32_t)C;
      d.n_blocks = (uint32_t)B;
      P.unit_start[P.count + 1] = P.unit_start[P.count] + cdiv(B, kUnitBlocks);
      min_len = std::min(min_len, m.min_len);
      ++P.count;
    }
    if (P.count == 0) continue;
    // with both indices the run index wins: its decoder is the faster one
    if (segmented && !indexed && smem_optin >= (int)kSegSmem) {
      // the segment decoder: units of 32 segments, one CTA of 32 warps per SM
      for (uint32_t i = 0; i < P.count; ++i)
        P.unit_start[i + 1] = P.unit_start[i] + cdiv(P.m[i].n_segs, kSegWarps);
      for (uint32_t i = P.count + 1; i <= DF11_MAX_BATCH; ++i) P.unit_start[i] = P.unit_start[P.count];
      P.min_len = min_len;
      P.stage_cap = 0;
      P.batch = 0;
      const uint64_t units = P.unit_start[P.count];
      const uint64_t grid = std::min<uint64_t>(cdiv(units, kSegWarps), (uint64_t)sms);
      decode_seg_kernel<<<(unsigned)grid, kSegThreads, kSegSmem, s>>>(P);
      st = launch_status();
      if (st != DF11_OK) return st;
      continue;
    }
    for (uint32_t i = P.count + 1; i <= DF11_MAX_BATCH; ++i) P.unit_start[i] = P.unit_start[P.count];
    P.stage_cap = (unit_codes + 15u) & ~15u;
    P.min_len = min_len;
    P.batch = io ? batch : 0u;
    const uint32_t region = 4u * (min_len >= 2 ? kMaxWords2 : kMaxWords1);
    const uint32_t group_bytes =
        indexed ? group_layout_idx(P.stage_cap).size : group_layout(P.stage_cap, region, nb).size;
    const uint64_t units = P.unit_start[P.count];
    // groups per CTA: as many as one CTA's shared memory holds next to the
    // tables (one CTA per SM), but no more than there are units per SM
    if (smem_optin < (int)(kTablesSmem + group_bytes)) return DF11_ERR_INVALID_ARG;
    const uint32_t fit = (uint32_t)((smem_optin - (int)kTablesSmem) / (int)group_bytes);
    const uint32_t groups = (uint32_t)std::min<uint64_t>(
        std::min<uint32_t>(kMaxGroups, fit), std::max<uint64_t>(1, cdiv(units, (uint64_t)sms)));
    const uint32_t smem = kTablesSmem + groups * group_bytes;
    const DecodeKernel kern = indexed ? decode_idx_kernel : decode_kernel_for(min_len < 2, nb);
    int occ = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, (int)(groups * kT), smem) !=
        cudaSuccess)
      return DF11_ERR_CUDA;
    if (occ < 1) return DF11_ERR_CUDA;
    const uint64_t grid = std::min<uint64_t>(cdiv(units, groups), (uint64_t)sms * occ);
    kern<<<(unsigned)grid, groups * kT, smem, s>>>(P);
    st = launch_status();
    if (st != DF11_OK) return st;
  }
  return DF11_OK;
}

}  // namespace

extern "C" df11_status df11_decode_block_batch(const df11_matrix *ms, uint32_t count,
                                               uint16_t *const *d_outs, uint32_t *d_status,
                                               df11_stream_t stream) {
  if (count && !d_outs) return DF11_ERR_INVALID_ARG;
  return launch_decode(ms, count, d_outs, nullptr, 0, d_status, stream);
}

extern "C" df11_status df11_decode_matmul_batch(const df11_matrix *ms, const df11_matmul_io *io,
                                                uint32_t count, uint32_t batch, uint32_t *d_status,
                                                df11_stream_t stream) {
  if (count && !io) return DF11_ERR_INVALID_ARG;
  return launch_decode(ms, count, nullptr, io, batch, d_status, stream);
}

extern "C" df11_status df11_decode(const df11_matrix *m, uint16_t *d_out, uint32_t *d_status,
                                   df11_stream_t stream) {
  if (!m) return DF11_ERR_INVALID_ARG;
  return df11_decode_block_batch(m, 1, &d_out, d_status, stream);
}

extern "C" df11_status df11_build_run_index(const df11_matrix *m, uint16_t *d_run_index,
                                            uint32_t *d_status, df11_stream_t stream) {
  if (!m || !d_status) return DF11_ERR_INVALID_ARG;
  if (m->n > DF11_MAX_N) return DF11_ERR_TOO_LARGE;
  if (m->n == 0) return DF11_OK;
  if (!d_run_index || !aligned16(d_run_index) || !m->stream || !m->gaps || !m->block_pos ||
      !m->tables || !aligned16(m->stream) || !aligned16(m->tables) ||
      ((uintptr_t)m->block_pos & 3u))
    return DF11_ERR_INVALID_ARG;
  if (m->min_len < 1 || m->min_len > 8) return DF11_ERR_INVALID_ARG;
  if (m->total_bits < m->n * (uint64_t)m->min_len || m->total_bits > m->n * 32ull)
    return DF11_ERR_INVALID_ARG;
  int dev, sms;
  df11_status st = device_info(&dev, &sms);
  if (st != DF11_OK) return st;
  const uint64_t C = cdiv(m->total_bits, 64);
  const uint64_t B = cdiv(C, DF11_BLOCK_CHUNKS);
  if (C >= (1ull << 31)) return DF11_ERR_TOO_LARGE;
  DecParams P{};
  DecMat &d = P.m[0];
  d.stream = m->stream;
  d.gaps = m->gaps;
  d.pos = m->block_pos;
  d.tables = reinterpret_cast<const DecodeTables *>(m->tables);
  d.n = m->n;
  d.total_bits = m->total_bits;
  d.n_chunks = (uint32_t)C;
  d.n_blocks = (uint32_t)B;
  P.count = 1;
  P.min_len = m->min_len;
  P.status = d_status;
  const uint64_t grid = std::min<uint64_t>(B, (uint64_t)sms * 8);
  run_index_kernel<false><<<(unsigned)grid, kRiThreads, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      P, d_run_index, nullptr);
  return launch_status();
}

extern "C" df11_status df11_build_segment_index(const df11_matrix *m, uint32_t *d_seg_index,
                                                uint32_t *d_status, df11_stream_t stream) {
  if (!m || !d_status) return DF11_ERR_INVALID_ARG;
  if (m->n > DF11_MAX_N) return DF11_ERR_TOO_LARGE;
  if (!d_seg_index || ((uintptr_t)d_seg_index & 3u)) return DF11_ERR_INVALID_ARG;
  if (m->total_bits > 0xFFFFFFFFull) return DF11_ERR_TOO_LARGE;
  if (m->n == 0) {
    // one entry: total_bits (0)
    return cudaMemsetAsync(d_seg_index, 0, 4, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
               ? DF11_OK
               : DF11_ERR_CUDA;
  }
  if (!m->stream || !m->gaps || !m->block_pos || !m->tables || !aligned16(m->stream) ||
      !aligned16(m->tables) || ((uintptr_t)m->block_pos & 3u))
    return DF11_ERR_INVALID_ARG;
  if (m->min_len < 1 || m->min_len > 8) return DF11_ERR_INVALID_ARG;
  if (m->total_bits < m->n * (uint64_t)m->min_len || m->total_bits > m->n * 32ull)
    return DF11_ERR_INVALID_ARG;
  int dev, sms;
  df11_status st = device_info(&dev, &sms);
  if (st != DF11_OK) return st;
  const uint64_t C = cdiv(m->total_bits, 64);
  const uint64_t B = cdiv(C, DF11_BLOCK_CHUNKS);
  DecParams P{};
  DecMat &d = P.m[0];
  d.stream = m->stream;
  d.gaps = m->gaps;
  d.pos = m->block_pos;
  d.tables = reinterpret_cast<const DecodeTables *>(m->tables);
  d.n = m->n;
  d.total_bits = m->total_bits;
  d.n_chunks = (uint32_t)C;
  d.n_blocks = (uint32_t)B;
  P.count = 1;
  P.min_len = m->min_len;
  P.status = d_status;
  const uint64_t grid = std::min<uint64_t>(B, (uint64_t)sms * 8);
  run_index_kernel<true><<<(unsigned)grid, kRiThreads, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      P, nullptr, d_seg_index);
  return launch_status();
}

#ifdef DF11_TEST_HOOKS
// Test build only (not in the product library): df11_decode whose stream-stage
// barriers each expect 16 bytes more than their bulk copies deliver.  Every
// copy lands, but no stage barrier completes, so each bounded wait runs out
// and the kernel must end with DF11_ERR_TIMEOUT in *d_status, nothing of its
// own in flight and nothing written outside d_out.
extern "C" df11_status df11_test_decode_starved(const df11_matrix *m, uint16_t *d_out,
                                                uint32_t *d_status, df11_stream_t stream) {
  if (!m || !d_out) return DF11_ERR_INVALID_ARG;
  uint16_t *outs[1] = {d_out};
  // the decoders with bulk-copy barriers (the segment decoder has none)
  df11_matrix mm = *m;
  mm.seg_index = nullptr;
  return launch_decode(&mm, 1, outs, nullptr, 0, d_status, stream, 16u);
}
#endif

// ============================================================ encode without allocation
//
// df11_encode needs a scratch buffer from its caller (the per-tile bit
// offsets).  Some callers cannot hand one over: code running inside another
// framework's execution callback with no access to that framework's device
// allocator, or a process that has reserved all device memory up front and
// may not allocate afterwards.  For them this variant keeps its scratch in a
// fixed array in the library's own device memory, so a call allocates
// nothing.  Its cost: every GPU that loads the library holds the array
// (kStaticTiles * 8 bytes, 512 KiB) until the process exits, and matrices are
// limited to DF11_STATIC_WS_MAX_N values.

namespace {

constexpr uint64_t kStaticTiles = 1ull << 16;  // tile offsets the array holds (incl. the total)
static_assert((kStaticTiles - 1) * df11i::kEncTile == DF11_STATIC_WS_MAX_N,
              "header limit and array size agree");

// The scratch itself.  Host code must not pass this name to a kernel (on the
// host it names a stand-in, not device memory); it uses the device address
// obtained with cudaGetSymbolAddress below.
static __device__ __align__(256) uint64_t g_static_tile_offsets[kStaticTiles];

std::mutex g_static_mu;
uint64_t *g_static_ptr[64] = {nullptr};

// Device address of the array on the current device, looked up once per device
// and kept for the life of the process (a device reset after the first call
// is not supported: the address would belong to the destroyed context).
df11_status static_scratch(int dev, uint64_t **ptr) {
  std::lock_guard<std::mutex> lk(g_static_mu);
  if (!g_static_ptr[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_tile_offsets) != cudaSuccess || !p) {
      cudaGetLastError();
      return DF11_ERR_CUDA;
    }
    g_static_ptr[dev] = reinterpret_cast<uint64_t *>(p);
  }
  *ptr = g_static_ptr[dev];
  return DF11_OK;
}

}  // namespace

extern "C" df11_status df11_encode_static_ws(const uint16_t *d_w, uint64_t n,
                                             const df11_codebook *cb, uint64_t total_bits,
                                             const df11_encoded *out, uint32_t *d_status,
                                             df11_stream_t stream) {
  if (!cb || !out || !d_status) return DF11_ERR_INVALID_ARG;
  if (n > DF11_STATIC_WS_MAX_N) return DF11_ERR_TOO_LARGE;
  df11_status st = check_encode_out(d_w, n, total_bits, out);
  if (st != DF11_OK) return st;
  // (n <= DF11_STATIC_WS_MAX_N gives at most kStaticTiles - 1 tiles plus the
  // total: the static_assert next to the array ties the two limits together)
  EncCodebook ecb;
  if ((st = host_enc_codebook(cb, &ecb)) != DF11_OK) return st;
  int dev, sms;
  if ((st = device_info(&dev, &sms)) != DF11_OK) return st;
  uint64_t *ws = nullptr;
  if ((st = static_scratch(dev, &ws)) != DF11_OK) return st;
  // nothing in the array needs clearing: every tile offset a call reads is
  // written earlier in the same call
  return launch_encode(d_w, n, ecb, nullptr, total_bits, out, ws, d_status,
                       reinterpret_cast<cudaStream_t>(stream));
}

// ============================================================ fused decode -> tensor-core GEMM
//
// y[j][r] += sum_c W[r][c] x[j][c] for up to 256 activation rows at a time,
// with W decoded through its segment index straight into the B operand of
// tcgen05.mma and never written to device memory.  A CTA (one per SM) owns
// 256 rows of W (the MMA's N) and walks its columns in steps of 64: row r's
// columns [64k, 64k + 64) are exactly segment r * cols / 64 + k of the
// segment index, so decode lane t (eight warps) decodes that segment and
// writes its 64 BF16 weights as row t of the step's B tile (K-major,
// 128-byte rows, 128-byte swizzle).  Everything a step reads from global
// memory is requested a step ahead with cp.async: the lane's 64 stream bytes
// from its segment's start, its 64 sign/mantissa bytes, and the step's
// activation tiles (zero-filled past the batch) as A.  A ninth warp issues,
// per step and 128-row M tile, four 128 x 256 x 16 MMAs accumulating in TMEM
// and commits them to the stage's "empty" barrier; after the last step the
// decode warps read the accumulators out of TMEM and add them to y.  Every
// wait is bounded.
namespace {

constexpr uint32_t kGemmN = 256;        // W rows per CTA (MMA N)
constexpr uint32_t kGemmM = 128;        // activation rows per M tile (MMA M)
constexpr uint32_t kGemmK = kSegOut;    // columns per step: one segment per row
constexpr uint32_t kGemmStages = 2;
constexpr uint32_t kGemmLanes = kGemmN;  // decode lanes: one per W row of the tile
constexpr uint32_t kGemmThreads = kGemmLanes + 32;
constexpr uint32_t kGemmBTile = kGemmN * kGemmK * 2;  // 32 KiB
constexpr uint32_t kGemmATile = kGemmM * kGemmK * 2;  // 16 KiB
constexpr uint32_t kGemmWin = 64;       // stream bytes staged per lane and step
constexpr uint32_t kGemmChunk = 64;     // steps per work item: 4096 columns
constexpr uint32_t kGemmMaxMT = DF11_GEMM_MAX_BATCH / kGemmM;
static_assert(kGemmK * 2 == 128, "one 128-byte swizzle row per tile row");
static_assert(kGemmN * kGemmMaxMT <= 512, "accumulators fit the 512 TMEM columns");

struct GemmParams {
  DecMat m[DF11_MAX_BATCH];
  uint32_t item_start[DF11_MAX_BATCH + 1];  // prefix sums of work items per matrix
  uint32_t count;
  uint32_t batch;  // activation rows of this launch (<= 128 * mt)
  uint32_t mt;     // M tiles: 1 or 2
  uint32_t min_len;
  uint32_t *status;
};

__host__ __device__ constexpr uint32_t gemm_stage_bytes(uint32_t mt) {
  return kGemmBTile + mt * kGemmATile;
}
// stages, tables, exponent rows, two buffers each of sign/mantissa bytes and
// of stream bytes, barriers and the TMEM address (the stages start the
// dynamic shared memory, which the kernel declares 1024-byte aligned: the
// swizzle atom)
__host__ __device__ constexpr uint32_t gemm_smem_bytes(uint32_t mt) {
  return kGemmStages * gemm_stage_bytes(mt) + kTablesSmem + 4 * kSegRowWords * kGemmLanes +
         2 * kGemmK * kGemmLanes + 2 * kGemmWin * kGemmLanes + 64;
}
static_assert(8 * (2 * kGemmStages + 3) + 8 <= 64, "barriers and the TMEM address fit");

// Shared-memory operand descriptor: K-major, 128-byte swizzle, rows of 128
// bytes, 8-row groups 1024 bytes apart.
__device__ __forceinline__ uint64_t umma_desc_sw128(uint32_t saddr) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu)  // start address
         | ((uint64_t)1 << 16)               // leading byte offset (unused with swizzle)
         | ((uint64_t)(1024 >> 4) << 32)     // stride byte offset: 8 rows
         | ((uint64_t)1 << 46)               // descriptor version
         | ((uint64_t)2 << 61);              // 128-byte swizzle
}

// Instruction descriptor: BF16 A and B (both K-major), FP32 accumulator,
// M = 128, N = 256.
constexpr uint32_t kGemmIdesc = (1u << 4) | (1u << 7) | (1u << 10) | ((kGemmN >> 3) << 17) |
                                ((kGemmM >> 4) << 24);

__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t acc) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(kGemmIdesc), "r"(acc)
      : "memory");
}
__device__ __forceinline__ void umma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
               : "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void gemm_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void cp16_zfill(uint32_t dst, const void *src, uint32_t bytes) {
  DF11_SMEM_CHECK(dst, 16, return)
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void cp_wait2() { asm volatile("cp.async.wait_group 2;" ::: "memory"); }

__global__ void __launch_bounds__(kGemmThreads, 1) decode_gemm_tc_kernel(const __grid_constant__ GemmParams P) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  if (raw & 1023u) {  // the declared alignment was not honoured: nothing is done
    if (threadIdx.x == 0) set_status(P.status, DF11_ERR_CUDA);
    return;
  }
  const uint32_t base = raw;
  uint8_t *smem = smem_raw;
  const uint32_t MT = P.mt;
  const uint32_t stage_bytes = gemm_stage_bytes(MT);
  const uint32_t tab_off = kGemmStages * stage_bytes;
  const uint32_t rows_off = tab_off + kTablesSmem;
  const uint32_t smp_off = rows_off + 4 * kSegRowWords * kGemmLanes;
  const uint32_t win_off = smp_off + 2 * kGemmK * kGemmLanes;
  const uint32_t bar_off = win_off + 2 * kGemmWin * kGemmLanes;
  const DecodeTables &tab = *reinterpret_cast<const DecodeTables *>(smem + tab_off);
  const uint32_t lut_a = base + tab_off;
  const uint32_t bar_full = base + bar_off;               // per stage: decode lanes arrived
  const uint32_t bar_empty = bar_full + 8 * kGemmStages;  // per stage: its MMAs completed
  const uint32_t bar_done = bar_empty + 8 * kGemmStages;  // an item's MMAs completed
  const uint32_t bar_free = bar_done + 8;                 // an item's accumulators read out
  const uint32_t bar_last = bar_free + 8;                 // every MMA completed
  uint32_t *slot = reinterpret_cast<uint32_t *>(smem + bar_off + 8 * (2 * kGemmStages + 3));
  const uint32_t t = threadIdx.x, warp = t >> 5, lane = t & 31u;
  constexpr uint32_t kMmaWarp = kGemmLanes / 32;
#ifdef DF11_CHECKED
  if (t == 0) {
    s_check_status = P.status;
    s_dyn_base = raw;
  }
  __syncthreads();
#endif
  const uint32_t ncols = kGemmN * MT;  // TMEM columns: a power of two
  if (t == 0) {
    for (uint32_t s = 0; s < kGemmStages; ++s) {
      mbar_init(bar_full + 8 * s, kGemmLanes);
      mbar_init(bar_empty + 8 * s, 1);
    }
    mbar_init(bar_done, 1);
    mbar_init(bar_free, kGemmLanes);
    mbar_init(bar_last, 1);
    slot[1] = 0u;  // set when a bounded wait runs out
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == kMmaWarp) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     base + bar_off + 8 * (2 * kGemmStages + 3)),
                 "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(slot);
  volatile uint32_t *gave_up = slot + 1;

  // this CTA's work items: a contiguous share of the launch's (matrix, tile
  // of 256 rows, chunk of kGemmChunk steps) list
  const uint32_t total = P.item_start[P.count];
  const uint32_t i0 = (uint32_t)((uint64_t)blockIdx.x * total / gridDim.x);
  const uint32_t i1 = (uint32_t)((uint64_t)(blockIdx.x + 1) * total / gridDim.x);
  uint32_t gstep = 0;  // steps so far: stage gstep % 2, its use gstep / 2
  uint32_t nitems = 0;
  uint32_t mi = 0xFFFFFFFFu;
  bool table_ok = false, table_short = true;
  bool bad = false;
  for (uint32_t item = i0; item < i1; ++item) {
    uint32_t m = mi == 0xFFFFFFFFu ? 0 : mi;
    while (m + 1 < P.count && item >= P.item_start[m + 1]) ++m;
    const DecMat &M = P.m[m];
    if (m != mi) {
      // a new matrix: its tables (every thread is past the previous item's decode)
      __syncthreads();
      const uint4 *src = reinterpret_cast<const uint4 *>(M.tables);
      uint4 *dst = reinterpret_cast<uint4 *>(smem + tab_off);
      for (uint32_t k = t; k < sizeof(DecodeTables) / 16; k += blockDim.x) dst[k] = __ldg(src + k);
      __syncthreads();
      bool tbad = false;
      for (uint32_t k = t; k < (uint32_t)df11i::kLutSize; k += blockDim.x)
        tbad |= lut_entry_bad(tab.lut[k].y, P.min_len);
      table_ok = !__syncthreads_or(tbad);
      table_short = tab.max_len <= (uint32_t)df11i::kLutBits;
      mi = m;
    }
    const uint32_t ksteps = M.cols / kGemmK;
    const uint32_t chunks = (ksteps + kGemmChunk - 1) / kGemmChunk;
    const uint32_t local = item - P.item_start[m];
    const uint32_t n0 = (local / chunks) * kGemmN;
    const uint32_t k0 = (local % chunks) * kGemmChunk, k1 = min(k0 + kGemmChunk, ksteps);

    if (warp < kMmaWarp) {
      // ---- decode lane t: row n0 + t of W, one segment per step
      const uint32_t r = n0 + t;
      const bool row_ok = r < M.rows;
      const uint64_t seg0 = (uint64_t)r * ksteps;  // segment of (row r, step 0)
      const uint64_t alloc = 2048ull * M.n_blocks + 16;  // the stream's allocation (bytes)
      const uint32_t row_a = base + rows_off + 4 * t;    // exponent word w: row_a + 1024 w
      const uint32_t smp = base + smp_off;               // sign/mantissa: 2 buffers
      const uint32_t win = base + win_off;               // stream bytes: 2 buffers
      // step k's sign/mantissa bytes (piece q of lane t at 16 (256 q + t)) and
      // the 64 stream bytes from its start a, 16-byte aligned, into buffers k & 1
      auto fetch = [&](uint32_t k, uint32_t a) {
        if (!row_ok || k >= k1) return;
        const uint32_t bf = k & 1u;
        for (uint32_t q = 0; q < 4u; ++q)
          seg_cp16(smp + kGemmK * kGemmLanes * bf + 16u * (kGemmLanes * q + t),
                   M.sm + (seg0 + k) * kGemmK + 16u * q);
        const uint64_t lo = min((uint64_t)((a >> 3) & ~15u), alloc - kGemmWin);
        for (uint32_t q = 0; q < kGemmWin / 16; ++q)
          seg_cp16(win + kGemmWin * kGemmLanes * bf + 16u * (kGemmLanes * q + t),
                   M.stream + lo + 16u * q);
      };
      uint32_t a = row_ok ? __ldg(M.seg + seg0 + k0) : 0u;
      uint32_t e = row_ok ? __ldg(M.seg + seg0 + k0 + 1) : 0u;
      fetch(k0, a);
      seg_commit();
      for (uint32_t k = k0; k < k1; ++k, ++gstep) {
        const uint32_t s = gstep % kGemmStages, use = gstep / kGemmStages;
        // the stage is free once the MMAs of its previous step completed
        if (*gave_up || (gstep >= kGemmStages && !mbar_wait(bar_empty + 8 * s, (use - 1) & 1u))) {
          *gave_up = 1u;  // (a bounded wait ran out: the CTA skips the rest of its
          continue;       // work but keeps its loop structure, barriers included)
        }
        const uint32_t st = base + s * stage_bytes;
        // the step's activation tiles: row m, 16-byte chunk c at chunk c ^ (m & 7)
        for (uint32_t i = t; i < MT * kGemmM * 8; i += kGemmLanes) {
          const uint32_t mm = i >> 3, c = i & 7u;
          const bool in = mm < P.batch;
          const uint16_t *src = in ? M.x + (uint64_t)mm * M.cols + kGemmK * k + 8 * c : M.x;
          cp16_zfill(st + kGemmBTile + kGemmATile * (mm / kGemmM) + (mm % kGemmM) * 128 +
                         ((c ^ (mm & 7u)) << 4),
                     src, in ? 16u : 0u);
        }
        seg_commit();     // this step's tiles
        fetch(k + 1, e);  // the next step starts where this one ends
        seg_commit();
        const uint32_t e_next = row_ok && k + 1 < k1 ? __ldg(M.seg + seg0 + k + 2) : 0u;
        cp_wait2();  // this step's stream and sign/mantissa bytes
        // the staged words from lo (the lane's 16-byte pieces interleave with
        // the other lanes': piece q of lane t at 16 (256 q + t)); past them (a
        // segment longer than the staged bytes allow), global memory
        const uint32_t bf = k & 1u;
        const uint32_t lo = (uint32_t)min((uint64_t)((a >> 3) & ~15u), alloc - kGemmWin);
        const uint32_t *gsrc = reinterpret_cast<const uint32_t *>(M.stream + lo);
        const uint32_t wbuf = win + kGemmWin * kGemmLanes * bf + 16u * t;
        auto word = [&](uint32_t j) -> uint32_t {
          return bswap32(j < kGemmWin / 4 ? lds32(wbuf + 16u * kGemmLanes * (j >> 2) + 4u * (j & 3u))
                                          : __ldg(gsrc + min((uint64_t)j, (alloc - lo) / 4 - 1)));
        };
        bool ok = row_ok && table_ok && a <= e && e <= M.total_bits && a >= 8u * lo &&
                  e - a <= (uint32_t)DF11_MAX_CODE_LEN * kGemmK;
        if (ok) {
          const uint32_t p = a - 8u * lo;
          ok = seg_decode_lane(p, e - 8u * lo, kGemmK, table_short, tab, lut_a, row_a,
                               4u * kGemmLanes, word, word(p >> 5), word((p >> 5) + 1u),
                               word((p >> 5) + 2u));
        }
        bad |= row_ok && !ok;
        // row t of the B tile: 16-byte chunk c at chunk c ^ (t & 7)
        const uint32_t brow = st + 128u * t;
        const uint32_t smk = smp + kGemmK * kGemmLanes * bf;
#pragma unroll
        for (uint32_t q = 0; q < 4u; ++q) {
          uint4 r0 = make_uint4(0u, 0u, 0u, 0u), r1 = r0;
          if (ok) {
            const uint4 sv = lds128(smk + 16u * (kGemmLanes * q + t));
            const uint32_t stride = 4u * kGemmLanes;
            merge4(lds32(row_a + stride * (4u * q)), sv.x, r0.x, r0.y);
            merge4(lds32(row_a + stride * (4u * q + 1u)), sv.y, r0.z, r0.w);
            merge4(lds32(row_a + stride * (4u * q + 2u)), sv.z, r1.x, r1.y);
            merge4(lds32(row_a + stride * (4u * q + 3u)), sv.w, r1.z, r1.w);
          }
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(brow + (((2u * q) ^ (t & 7u)) << 4)),
                       "r"(r0.x), "r"(r0.y), "r"(r0.z), "r"(r0.w)
                       : "memory");
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(brow + (((2u * q + 1u) ^ (t & 7u)) << 4)),
                       "r"(r1.x), "r"(r1.y), "r"(r1.z), "r"(r1.w)
                       : "memory");
        }
        seg_wait_prev();  // this step's activation tiles (all but the next step's bytes)
        // the tiles, written through the generic proxy, are read by the MMA
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        gemm_arrive(bar_full + 8 * s);
        a = e;
        e = e_next;
      }
      seg_wait_all();
      // ---- the item's accumulators (TMEM lane = activation row) added to y.
      // Warps w and w + 4 share lanes 32 (w % 4).. and split the 256 columns;
      // other items add to the same sums, hence the atomic adds.
      if (*gave_up || !mbar_wait(bar_done, nitems & 1u)) *gave_up = 1u;
      tc_fence_after();
      const uint32_t quarter = warp & 3u, half = warp >> 2;
      // (the TMEM loads need the whole warp: it skips them together)
      const bool skip = __any_sync(0xffffffffu, *gave_up != 0u);
      for (uint32_t mt = 0; mt < (skip ? 0u : MT); ++mt) {
        const uint32_t j = kGemmM * mt + 32u * quarter + lane;  // activation row
#pragma unroll 1
        for (uint32_t c = kGemmN / 2 * half; c < kGemmN / 2 * (half + 1); c += 16) {
          uint32_t v[16];
          asm volatile(
              "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
              "%11, %12, %13, %14, %15}, [%16];"
              : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
                "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]),
                "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
              : "r"(tmem + ((32u * quarter) << 16) + kGemmN * mt + c));
          asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
          if (j < P.batch) {
            float *yr = M.y + (uint64_t)j * M.rows + n0 + c;
#pragma unroll
            for (uint32_t i = 0; i < 16; ++i)
              if (n0 + c + i < M.rows) atomicAdd(yr + i, __uint_as_float(v[i]));
          }
        }
      }
      tc_fence_before();
      gemm_arrive(bar_free);  // the next item's MMAs may overwrite the accumulators
    } else if (lane == 0) {
      // ---- the MMA issuer: the item's steps into the accumulators, once the
      // previous item's were read out
      if (*gave_up || (nitems > 0 && !mbar_wait(bar_free, (nitems - 1) & 1u))) *gave_up = 1u;
      tc_fence_after();
      for (uint32_t k = k0; k < k1; ++k, ++gstep) {
        const uint32_t s = gstep % kGemmStages, use = gstep / kGemmStages;
        if (*gave_up || !mbar_wait(bar_full + 8 * s, use & 1u)) {
          *gave_up = 1u;
          continue;
        }
        tc_fence_after();
        const uint32_t st = base + s * stage_bytes;
        for (uint32_t mt = 0; mt < MT; ++mt)
#pragma unroll
          for (uint32_t kk = 0; kk < kGemmK / 16; ++kk)
            umma_bf16(tmem + kGemmN * mt,
                      umma_desc_sw128(st + kGemmBTile + kGemmATile * mt + 32u * kk),
                      umma_desc_sw128(st + 32u * kk), (k != k0) || (kk != 0u));
        umma_commit(bar_empty + 8 * s);
      }
      umma_commit(bar_done);  // arrives once the item's MMAs have completed
    } else {
      // lanes 1..31 of the MMA warp follow the loop (for the table barriers)
      gstep += k1 - k0;
    }
    ++nitems;
  }
  if (bad) set_status(P.status, DF11_ERR_CORRUPT);
  // every MMA this CTA issued has completed before the accumulators go
  if (warp == kMmaWarp && lane == 0) umma_commit(bar_last);
  if (!mbar_wait(bar_last, 0)) *gave_up = 1u;
  tc_fence_before();
  __syncthreads();
  if (t == 0 && *gave_up) set_status(P.status, DF11_ERR_TIMEOUT);
  if (warp == kMmaWarp) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(ncols)
                 : "memory");
  }
}

}  // namespace

extern "C" df11_status df11_decode_gemm_batch(const df11_matrix *ms, const df11_matmul_io *io,
                                              uint32_t count, uint32_t batch, uint32_t *d_status,
                                              df11_stream_t stream) {
  if (count == 0) return DF11_OK;
  if (!ms || !io || !d_status || batch < 1) return DF11_ERR_INVALID_ARG;
  int dev, sms;
  df11_status st = device_info(&dev, &sms);
  if (st != DF11_OK) return st;
  // the dynamic shared memory this kernel may take: the device's per-CTA
  // limit less the kernel's own static shared variables
  static int avail[64] = {};
  static std::mutex mu;
  {
    std::lock_guard<std::mutex> lk(mu);
    if (!avail[dev]) {
      int optin = 0;
      cudaFuncAttributes fa;
      if (cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess ||
          cudaFuncGetAttributes(&fa, decode_gemm_tc_kernel) != cudaSuccess)
        return DF11_ERR_CUDA;
      const int a = optin - (int)fa.sharedSizeBytes;
      if (cudaFuncSetAttribute(decode_gemm_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               std::min(a, (int)gemm_smem_bytes(kGemmMaxMT))) != cudaSuccess)
        return DF11_ERR_CUDA;
      avail[dev] = a;
    }
  }
  if (avail[dev] < (int)gemm_smem_bytes(std::min<uint32_t>(kGemmMaxMT, (batch + kGemmM - 1) / kGemmM)))
    return DF11_ERR_INVALID_ARG;
  // check every matrix (the work items are then listed longest matrix first)
  std::vector<uint32_t> order;
  for (uint32_t i = 0; i < count; ++i) {
    const df11_matrix &m = ms[i];
    const df11_matmul_io &q = io[i];
    if (m.n == 0) continue;
    if (m.n > DF11_MAX_N || m.total_bits > 0xFFFFFFFFull) return DF11_ERR_TOO_LARGE;
    if (!m.stream || !m.sign_mantissa || !m.tables || !m.seg_index || !aligned16(m.stream) ||
        !aligned16(m.sign_mantissa) || !aligned16(m.tables) || ((uintptr_t)m.seg_index & 3u))
      return DF11_ERR_INVALID_ARG;
    if (m.min_len < 1 || m.min_len > 8 || m.total_bits < m.n * (uint64_t)m.min_len ||
        m.total_bits > m.n * 32ull)
      return DF11_ERR_INVALID_ARG;
    if ((uint64_t)q.rows * q.cols != m.n || q.cols % kGemmK || !q.x || !q.y || !aligned16(q.x) ||
        ((uintptr_t)q.y & 3u))
      return DF11_ERR_INVALID_ARG;
    order.push_back(i);
  }
  std::stable_sort(order.begin(), order.end(),
                   [&](uint32_t x, uint32_t y) { return io[x].cols > io[y].cols; });
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // batches above DF11_GEMM_MAX_BATCH rows: one pass per 256 rows (W decoded again)
  for (uint32_t j0 = 0; j0 < batch; j0 += DF11_GEMM_MAX_BATCH) {
    const uint32_t nb = std::min<uint32_t>(DF11_GEMM_MAX_BATCH, batch - j0);
    for (size_t first = 0; first < order.size(); first += DF11_MAX_BATCH) {
      const size_t k = std::min<size_t>(DF11_MAX_BATCH, order.size() - first);
      GemmParams P{};
      P.status = d_status;
      P.batch = nb;
      P.mt = (nb + kGemmM - 1) / kGemmM;
      P.min_len = DF11_MAX_CODE_LEN;
      for (size_t i = 0; i < k; ++i) {
        const df11_matrix &m = ms[order[first + i]];
        const df11_matmul_io &q = io[order[first + i]];
        DecMat &d = P.m[P.count];
        d.stream = m.stream;
        d.sm = m.sign_mantissa;
        d.seg = m.seg_index;
        d.tables = reinterpret_cast<const DecodeTables *>(m.tables);
        d.n = m.n;
        d.total_bits = m.total_bits;
        d.n_blocks = (uint32_t)cdiv(cdiv(m.total_bits, 64), DF11_BLOCK_CHUNKS);
        d.n_segs = (uint32_t)cdiv(m.n, kSegOut);
        d.rows = q.rows;
        d.cols = q.cols;
        d.x = q.x + (uint64_t)j0 * q.cols;
        d.y = q.y + (uint64_t)j0 * q.rows;
        P.item_start[P.count + 1] =
            P.item_start[P.count] +
            (uint32_t)(cdiv(q.rows, kGemmN) * cdiv(q.cols / kGemmK, kGemmChunk));
        P.min_len = std::min(P.min_len, m.min_len);
        ++P.count;
      }
      // one persistent CTA per SM, each with a contiguous share of the items
      const uint32_t items = P.item_start[P.count];
      const uint32_t grid = std::min<uint32_t>(items, (uint32_t)sms);
      decode_gemm_tc_kernel<<<grid, kGemmThreads, gemm_smem_bytes(P.mt), s>>>(P);
      st = launch_status();
      if (st != DF11_OK) return st;
    }
  }
  return DF11_OK;
}

// ============================================================ decode from host memory, pipelined
//
// Matrices held in host memory, decoded into host memory.  Each matrix is cut
// into pieces of whole decode units (kPieceBlocks blocks), and every piece is
// a matrix of its own to the kernels: its stored arrays are copied in, its
// block positions are made relative to its first output, its run index is
// built, it is decoded, and its BF16 words are copied out to their place in
// the matrix.  Pieces take turns in kHostSlots slots of the caller's device
// scratch, and three streams of the call's own carry the copies in, the
// kernels and the copies out, so that both copy directions and the kernels
// overlap from one piece to the next.
namespace {

constexpr uint64_t kHostAlign = 256;
constexpr uint32_t kHostSlots = 3;
#ifndef DF11_PIECE_BLOCKS
#define DF11_PIECE_BLOCKS 4096  // about 26 M values at 2.6 code bits per value
#endif
#ifndef DF11_FIRST_PIECE_BLOCKS
#define DF11_FIRST_PIECE_BLOCKS 256
#endif
constexpr uint64_t kPieceBlocks = DF11_PIECE_BLOCKS;
constexpr uint64_t kFirstPieceBlocks = DF11_FIRST_PIECE_BLOCKS;
static_assert(kPieceBlocks % kUnitBlocks == 0 && kFirstPieceBlocks % kUnitBlocks == 0 &&
                  kFirstPieceBlocks <= kPieceBlocks,
              "pieces are whole decode units");
constexpr uint64_t kBlockBits = 64ull * DF11_BLOCK_CHUNKS;

inline uint64_t up_to(uint64_t x, uint64_t a) { return (x + a - 1) / a * a; }

// The decode tables of a codebook, built on the device from the codebook
// itself (a kernel parameter), so the call queues no pageable copy.
__global__ void __launch_bounds__(kCbThreads) tables_kernel(const __grid_constant__ df11_codebook cb,
                                                            DecodeTables *__restrict__ t_out) {
  __shared__ df11cb::TableAux aux;
  const int t = threadIdx.x;
  uint32_t *tz = reinterpret_cast<uint32_t *>(t_out);
  for (uint32_t i = t; i < sizeof(DecodeTables) / 4; i += kCbThreads) tz[i] = 0u;
  __syncthreads();
  if (t == 0) df11cb::table_lengths(&cb, t_out, aux);  // checked on the host already
  __syncthreads();
  df11cb::table_value(&cb, t_out, t);
  __syncthreads();
  for (uint32_t v = t; v < (uint32_t)df11i::kLutSize; v += kCbThreads)
    t_out->lut[v] = df11cb::lut_entry_for(*t_out, aux, cb.max_len, v);
}

// Block positions of a piece, made relative to its first output.
__global__ void rebase_pos_kernel(uint32_t *__restrict__ pos, uint32_t count, uint32_t base) {
  for (uint32_t i = blockIdx.x * blockDim.x + threadIdx.x; i < count; i += gridDim.x * blockDim.x)
    pos[i] -= base;
}

// A piece: blocks [b0, b1) of matrix `mat`, outputs [p0, p1), code bits from
// the piece's first chunk to its end.
struct Piece {
  uint32_t mat;
  uint64_t b0, b1, p0, p1, bits;
};

// One piece's arrays in a slot (offsets from the slot).
struct HostSlot {
  uint64_t stream, gaps, pos, sm, run_index, out, bytes;
};
HostSlot host_slot(const df11_sizes &z) {
  HostSlot s{};
  uint64_t o = 0;
  s.stream = o, o = up_to(o + z.stream_alloc, kHostAlign);
  s.gaps = o, o = up_to(o + z.gaps_alloc, kHostAlign);
  s.pos = o, o = up_to(o + z.block_pos_alloc, kHostAlign);
  s.sm = o, o = up_to(o + z.sign_mantissa_alloc, kHostAlign);
  s.run_index = o, o = up_to(o + std::max<uint64_t>(16, z.run_index_bytes), kHostAlign);
  s.out = o, o = up_to(o + 2 * z.n, kHostAlign);
  s.bytes = o;
  return s;
}

uint32_t shortest_code(const uint8_t *len) {
  uint32_t m = 0;
  for (int s = 0; s < 256; ++s)
    if (len[s] && (!m || len[s] < m)) m = len[s];
  return m;
}

// Cuts every matrix into pieces and sizes the scratch: the decode tables of
// every matrix, then kHostSlots slots as large as the largest piece needs.
// The call's first piece is short (kFirstPieceBlocks), so the first copy out
// starts early; each piece after it may be twice as long as the one before,
// up to kPieceBlocks, so the copy in of the next piece still ends before the
// copy out of the current one.  Few long pieces suit the PCIe link: copies
// in and out running at once lose bandwidth with every extra pair.  A cut falls between two decode units, and only where the positions stored
// there are in order and leave the piece at least min_len bits per value
// (codes running over the cut can shorten a piece by a few bits; such a cut
// moves on by a unit).  A last piece of one block would hold no code start
// and joins the piece before it.
df11_status plan_pieces(const df11_host_matrix *ms, uint32_t count, std::vector<Piece> *pieces,
                        uint64_t *tables_bytes, uint64_t *slot_bytes) {
  *tables_bytes = up_to((uint64_t)count * up_to(sizeof(DecodeTables), 16), kHostAlign);
  *slot_bytes = 0;
  uint64_t limit = kFirstPieceBlocks;  // doubles with every piece up to kPieceBlocks
  for (uint32_t i = 0; i < count; ++i) {
    const df11_host_matrix &h = ms[i];
    df11_sizes z;
    df11_status st = df11_sizes_from_bits(h.n, h.total_bits, &z);
    if (st != DF11_OK) return st;
    if (!h.n) continue;
    if (!h.lengths || !h.block_pos || !h.gaps || !h.stream || !h.sign_mantissa)
      return DF11_ERR_INVALID_ARG;
    // the decoder's conditions on a matrix (a complete code over at most 256
    // values has a code of at most 8 bits)
    const uint32_t ml = shortest_code(h.lengths);
    if (ml < 1 || ml > 8) return DF11_ERR_INVALID_ARG;
    if (h.max_block_codes > (64 + ml - 1) / ml * DF11_BLOCK_CHUNKS) return DF11_ERR_INVALID_ARG;
    const uint64_t B = z.n_blocks;
    if (h.block_pos[0] != 0 || h.block_pos[B] != h.n) return DF11_ERR_CORRUPT;
    auto settle = [B](uint64_t b) { return B - b < kUnitBlocks ? B : b; };  // no 1-block tail
    for (uint64_t b0 = 0; b0 < B;) {
      auto fits = [&](uint64_t b1) {
        const uint64_t p1 = h.block_pos[b1], p0 = h.block_pos[b0];
        return p1 >= p0 && p1 <= h.n && (p1 - p0) * ml <= (b1 - b0) * kBlockBits;
      };
      uint64_t b1 = settle(std::min(B, b0 + limit));
      limit = std::min(2 * limit, kPieceBlocks);
      while (b1 < B && !fits(b1)) b1 = settle(b1 + kUnitBlocks);
      Piece pc{i, b0, b1, h.block_pos[b0], h.block_pos[b1],
               (b1 == B ? h.total_bits : b1 * kBlockBits) - b0 * kBlockBits};
      if (pc.p1 < pc.p0 || (pc.p1 - pc.p0) * ml > pc.bits) return DF11_ERR_CORRUPT;
      df11_sizes pz;
      if (df11_sizes_from_bits(pc.p1 - pc.p0, pc.bits, &pz) != DF11_OK) return DF11_ERR_CORRUPT;
      *slot_bytes = std::max(*slot_bytes, host_slot(pz).bytes);
      if (pieces) pieces->push_back(pc);
      b0 = b1;
    }
  }
  return DF11_OK;
}

}  // namespace

extern "C" uint64_t df11_decode_host_scratch_bytes(const df11_host_matrix *ms, uint32_t count) {
  if (!ms && count) return 0;
  uint64_t tb, sb;
  if (plan_pieces(ms, count, nullptr, &tb, &sb) != DF11_OK) return 0;
  return tb + kHostSlots * sb;
}

extern "C" df11_status df11_decode_host_batch(const df11_host_matrix *ms, uint32_t count,
                                              uint16_t *const *h_outs, void *d_scratch,
                                              uint64_t scratch_bytes, uint32_t *d_status,
                                              df11_stream_t stream) {
  if (count == 0) return DF11_OK;
  if (!ms || !h_outs || !d_scratch || !d_status || ((uintptr_t)d_scratch % kHostAlign))
    return DF11_ERR_INVALID_ARG;
  // host side first: every matrix's codebook (checked), its pieces, the sizes
  std::vector<df11_codebook> cbs(count);
  for (uint32_t i = 0; i < count; ++i) {
    const df11_host_matrix &h = ms[i];
    if (h.n > DF11_MAX_N) return DF11_ERR_TOO_LARGE;
    if (!h.n) continue;
    if (!h.lengths || !h_outs[i]) return DF11_ERR_INVALID_ARG;
    const uint32_t cap = h.cap >= 1 && h.cap <= DF11_MAX_CODE_LEN ? h.cap : DF11_MAX_CODE_LEN;
    df11_status st = df11_codebook_from_lengths(h.lengths, cap, &cbs[i]);
    if (st != DF11_OK) return st;
  }
  std::vector<Piece> pieces;
  uint64_t tb, sb;
  df11_status st = plan_pieces(ms, count, &pieces, &tb, &sb);
  if (st != DF11_OK) return st;
  if (scratch_bytes < tb + kHostSlots * sb) return DF11_ERR_INVALID_ARG;
  int dev, sms;
  if ((st = device_info(&dev, &sms)) != DF11_OK) return st;  // a usable device

  uint8_t *base = static_cast<uint8_t *>(d_scratch);
  const uint64_t tstride = up_to(sizeof(DecodeTables), 16);
  cudaStream_t caller = reinterpret_cast<cudaStream_t>(stream);
  cudaStream_t cs = nullptr, xs = nullptr, ds = nullptr;
  std::vector<cudaEvent_t> ev;  // every event made here, released at the end
  auto event = [&](cudaEvent_t *e) {
    if (cudaEventCreateWithFlags(e, cudaEventDisableTiming) != cudaSuccess) return false;
    ev.push_back(*e);
    return true;
  };
  cudaEvent_t start = nullptr, slot_free[kHostSlots] = {};
  bool ok = cudaStreamCreateWithFlags(&cs, cudaStreamNonBlocking) == cudaSuccess &&
            cudaStreamCreateWithFlags(&xs, cudaStreamNonBlocking) == cudaSuccess &&
            cudaStreamCreateWithFlags(&ds, cudaStreamNonBlocking) == cudaSuccess && event(&start);
  // everything starts after the work already queued on the caller's stream
  ok = ok && cudaEventRecord(start, caller) == cudaSuccess &&
       cudaStreamWaitEvent(cs, start, 0) == cudaSuccess &&
       cudaStreamWaitEvent(xs, start, 0) == cudaSuccess &&
       cudaStreamWaitEvent(ds, start, 0) == cudaSuccess;
  // every matrix's decode tables, on the kernel stream
  for (uint32_t i = 0; ok && i < count; ++i) {
    if (!ms[i].n) continue;
    tables_kernel<<<1, kCbThreads, 0, xs>>>(cbs[i], reinterpret_cast<DecodeTables *>(base + i * tstride));
    ok = cudaGetLastError() == cudaSuccess;
  }
  for (size_t k = 0; ok && k < pieces.size(); ++k) {
    const Piece &pc = pieces[k];
    const df11_host_matrix &h = ms[pc.mat];
    df11_sizes hz, z;
    df11_sizes_from_bits(h.n, h.total_bits, &hz);
    df11_sizes_from_bits(pc.p1 - pc.p0, pc.bits, &z);
    const HostSlot L = host_slot(z);
    const uint32_t slot = (uint32_t)(k % kHostSlots);
    uint8_t *sp = base + tb + slot * sb;
    // copy in, once the slot's previous piece has been copied out: the
    // piece's stream plus the next 16 bytes (read past its last run), its
    // gaps, positions and sign/mantissa bytes
    const uint64_t s_off = pc.b0 * (kBlockBits / 8), g_off = pc.b0 * (DF11_GAP_BITS * DF11_BLOCK_CHUNKS / 8);
    const uint64_t s_len = std::min<uint64_t>(z.stream_bytes + 16, hz.stream_bytes - s_off);
    const uint64_t g_len = std::min<uint64_t>(z.gaps_bytes + 1, hz.gaps_bytes - g_off);
    const uint64_t n = pc.p1 - pc.p0;
    cudaEvent_t in_done, dec_done, freed;
    ok = event(&in_done) && event(&dec_done) && event(&freed);
    if (ok && slot_free[slot]) ok = cudaStreamWaitEvent(cs, slot_free[slot], 0) == cudaSuccess;
    ok = ok &&
         cudaMemcpyAsync(sp + L.stream, h.stream + s_off, s_len, cudaMemcpyHostToDevice, cs) == cudaSuccess &&
         cudaMemcpyAsync(sp + L.gaps, h.gaps + g_off, g_len, cudaMemcpyHostToDevice, cs) == cudaSuccess &&
         cudaMemcpyAsync(sp + L.pos, h.block_pos + pc.b0, 4 * (pc.b1 - pc.b0 + 1), cudaMemcpyHostToDevice,
                         cs) == cudaSuccess &&
         cudaMemcpyAsync(sp + L.sm, h.sign_mantissa + pc.p0, n, cudaMemcpyHostToDevice, cs) == cudaSuccess &&
         cudaEventRecord(in_done, cs) == cudaSuccess;
    // positions relative to the piece, its run index, its decode
    df11_matrix m{};
    m.n = n;
    m.total_bits = pc.bits;
    m.stream = sp + L.stream;
    m.gaps = sp + L.gaps;
    m.block_pos = reinterpret_cast<const uint32_t *>(sp + L.pos);
    m.sign_mantissa = sp + L.sm;
    m.tables = base + pc.mat * tstride;
    m.min_len = cbs[pc.mat].min_len;
    m.max_block_codes = h.max_block_codes;
    uint16_t *d_out = reinterpret_cast<uint16_t *>(sp + L.out);
    ok = ok && cudaStreamWaitEvent(xs, in_done, 0) == cudaSuccess;
    if (ok && pc.p0) {
      const uint32_t cnt = (uint32_t)(pc.b1 - pc.b0 + 1);
      rebase_pos_kernel<<<(cnt + 255) / 256, 256, 0, xs>>>(reinterpret_cast<uint32_t *>(sp + L.pos), cnt,
                                                            (uint32_t)pc.p0);
      ok = cudaGetLastError() == cudaSuccess;
    }
    ok = ok && df11_build_run_index(&m, reinterpret_cast<uint16_t *>(sp + L.run_index), d_status,
                                    reinterpret_cast<df11_stream_t>(xs)) == DF11_OK;
    m.run_index = reinterpret_cast<const uint16_t *>(sp + L.run_index);
    ok = ok && launch_decode(&m, 1, &d_out, nullptr, 0, d_status, reinterpret_cast<df11_stream_t>(xs)) == DF11_OK;
    ok = ok && cudaEventRecord(dec_done, xs) == cudaSuccess;
    // copy out to the piece's place; the slot is free after it
    ok = ok && cudaStreamWaitEvent(ds, dec_done, 0) == cudaSuccess &&
         cudaMemcpyAsync(h_outs[pc.mat] + pc.p0, d_out, 2 * n, cudaMemcpyDeviceToHost, ds) == cudaSuccess &&
         cudaEventRecord(freed, ds) == cudaSuccess;
    if (ok) slot_free[slot] = freed;
  }
  // the caller's stream waits for all three streams (after a failure too,
  // for whatever was queued before it uses the scratch)
  for (cudaStream_t q : {cs, xs, ds}) {
    cudaEvent_t done;
    if (!q || !event(&done) || cudaEventRecord(done, q) != cudaSuccess ||
        cudaStreamWaitEvent(caller, done, 0) != cudaSuccess)
      ok = false;
  }
  // streams and events are released by CUDA once their work completes
  for (cudaEvent_t e : ev) cudaEventDestroy(e);
  if (cs) cudaStreamDestroy(cs);
  if (xs) cudaStreamDestroy(xs);
  if (ds) cudaStreamDestroy(ds);
  if (ok) return DF11_OK;
  cudaGetLastError();
  return DF11_ERR_CUDA;
}
