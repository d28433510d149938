// rans_kernels.cu -- sm_100a kernels of the rANS exponent-codec variant
// (include/df11_rans.h) and their C-ABI launchers.
//
// Source: "DFloat11: Nén suy luận GPU không mất dữ liệu, giảm LLM xuống còn 70%
// kích thước" (vi.news.hada.io/topic?id=20542); its Hacker News discussion
// names rANS as the SIMD-friendlier alternative to the Huffman exponent code.
// The coding step is range ANS (J. Duda, "Asymmetric numeral systems", 2013).
//
// Kernels:
//   rans_encode_kernel<false>  one warp per 16384-value unit runs the 32
//                      interleaved encoders backwards and counts the unit's
//                      words
//   rans_scan_kernel   unit sizes -> 16-byte unit offsets (one CTA)
//   rans_encode_kernel<true>   the same pass again, now storing each word at
//                      its decoding-order index, the final states, segment
//                      word starts, padding and the sign/mantissa plane
//   rans_decode_kernel persistent CTAs over a contiguous share of the batch's
//                      units; the slot table of the current matrix sits in
//                      shared memory; each warp decodes one unit at a time,
//                      its 32 states in lockstep.  A ballot gives the lanes
//                      that renormalise and each one's word index.  The next
//                      segment's words are copied to shared memory
//                      (cp.async) while the current segment decodes.
//                      Exponents are staged per segment and merged with the
//                      sign/mantissa bytes into 16-byte BF16 stores.
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "df11_rans.h"

namespace {

constexpr uint32_t kM = 1u << DF11_RANS_PROB_BITS;  // 4096
constexpr uint32_t kL = 1u << 16;                   // lower end of the state range
constexpr uint32_t kUnit = DF11_RANS_UNIT;          // 16384 values
constexpr uint32_t kSegSteps = DF11_RANS_STEPS / DF11_RANS_SEGMENTS;  // 64
constexpr uint32_t kSegVals = 32 * kSegSteps;       // 2048 values per segment
constexpr uint32_t kHeader = DF11_RANS_HEADER_BYTES;
static_assert(kUnit == 32 * DF11_RANS_STEPS && DF11_RANS_LANES == 32, "a warp per unit");
static_assert(DF11_RANS_TABLES_BYTES == 4 * (kM + 256), "table layout");

__device__ __forceinline__ void set_status(uint32_t *st, uint32_t code) {
  if (st) atomicCAS(st, 0u, code);
}

__device__ __forceinline__ uint32_t lanemask_lt() {
  uint32_t m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

// ============================================================ encode

constexpr int kEncWarps = 8;
constexpr int kEncThreads = 32 * kEncWarps;

// One warp per unit.  The encoder of state l runs steps k = 511..0 over values
// v0 + 32k + l; the decoder reads the words in the reverse order, so a word
// emitted at step k by lane l has decoding index
//   (words of steps < k) + (lanes < l that emit at step k)
//   = W - (words of steps > k) - (words of step k) + popc(mask & lanes < l).
// Both passes make the same decisions; kEmit also stores.
template <bool kEmit>
__global__ void __launch_bounds__(kEncThreads)
rans_encode_kernel(const uint16_t *__restrict__ w, uint64_t n, const uint32_t *__restrict__ tables,
                   uint32_t units, uint32_t *__restrict__ unit_words,
                   const uint32_t *__restrict__ off16, uint8_t *__restrict__ stream,
                   uint8_t *__restrict__ sign_mantissa, uint32_t *status) {
  __shared__ uint32_t enc_s[256];
  for (int i = threadIdx.x; i < 256; i += kEncThreads) enc_s[i] = tables[kM + i];
  __syncthreads();
  const uint32_t lane = threadIdx.x & 31;
  const uint32_t lt = lanemask_lt();
  for (uint32_t u = blockIdx.x * kEncWarps + (threadIdx.x >> 5); u < units;
       u += gridDim.x * kEncWarps) {
    const uint64_t v0 = (uint64_t)u * kUnit;
    const uint32_t nv = (n - v0) < kUnit ? (uint32_t)(n - v0) : kUnit;
    const uint32_t W = kEmit ? unit_words[u] : 0u;
    uint8_t *base = kEmit ? stream + (uint64_t)off16[u] * 16 : nullptr;
    uint16_t *words = kEmit ? reinterpret_cast<uint16_t *>(base + kHeader) : nullptr;
    const uint64_t unit_bytes = kEmit ? (uint64_t)(off16[u + 1] - off16[u]) * 16 : 0;
    if (kEmit && (off16[u + 1] < off16[u] || unit_bytes < kHeader + 2ull * W ||
                  unit_bytes >= kHeader + 2ull * W + 16)) {
      if (lane == 0) set_status(status, DF11_ERR_CORRUPT);  // layout disagrees with the counts
      continue;
    }
    uint32_t x = kL, after = 0;
    uint32_t seg[DF11_RANS_SEGMENTS];
    bool bad_symbol = false;
#pragma unroll
    for (int g = DF11_RANS_SEGMENTS - 1; g >= 0; --g) {
      seg[g] = 0;
#pragma unroll 8
      for (int kk = kSegSteps - 1; kk >= 0; --kk) {
        const uint32_t i = (g * kSegSteps + kk) * 32 + lane;
        const bool in = i < nv;
        const uint32_t v = in ? w[v0 + i] : 0u;
        const uint32_t ent = enc_s[(v >> 7) & 0xFF];
        const uint32_t f = ent & 0xFFFF, cum = ent >> 16;
        bad_symbol |= in && f == 0;
        const bool act = in && f != 0;
        const bool emit = act && (x >> 20) >= f;  // x >= f * 2^20, without overflow
        const uint32_t mask = __ballot_sync(~0u, emit);
        const uint32_t c = __popc(mask);
        if constexpr (kEmit) {
          const uint32_t idx = W - after - c + __popc(mask & lt);
          if (emit && idx < W) words[idx] = (uint16_t)(x & 0xFFFF);
        }
        if (emit) x >>= 16;
        if (act) x = (x / f) * kM + x % f + cum;
        after += c;
        seg[g] += c;
        if (kEmit && in) sign_mantissa[v0 + i] = (uint8_t)(((v >> 8) & 0x80) | (v & 0x7F));
      }
    }
    if (__any_sync(~0u, bad_symbol) && lane == 0) set_status(status, DF11_ERR_SYMBOL_NOT_IN_CODEBOOK);
    if (!kEmit) {
      if (lane == 0) unit_words[u] = after;
      continue;
    }
    if (after != W) {
      if (lane == 0) set_status(status, DF11_ERR_CORRUPT);
      continue;
    }
    reinterpret_cast<uint32_t *>(base)[lane] = x;
    uint32_t start = 0;
#pragma unroll
    for (int g = 0; g < (int)DF11_RANS_SEGMENTS; ++g) start += (uint32_t)g < lane ? seg[g] : 0u;
    if (lane < DF11_RANS_SEGMENTS) reinterpret_cast<uint16_t *>(base + 128)[lane] = (uint16_t)start;
    const uint32_t pad_words = (uint32_t)(unit_bytes - kHeader - 2ull * W) / 2;  // < 8, checked above
    if (lane < pad_words) words[W + lane] = 0;
  }
}

// off16[u] = sum over units before u of ceil((144 + 2 W) / 16); off16[U] = total.
constexpr int kScanThreads = 1024;

__global__ void __launch_bounds__(kScanThreads)
rans_scan_kernel(const uint32_t *__restrict__ unit_words, uint32_t units, uint32_t *__restrict__ off16) {
  __shared__ uint32_t warp_sum[32];
  const uint32_t t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const uint32_t per = (units + kScanThreads - 1) / kScanThreads;
  const uint32_t lo = t * per < units ? t * per : units;
  const uint32_t hi = lo + per < units ? lo + per : units;
  auto size16 = [&](uint32_t u) { return (kHeader + 2 * unit_words[u] + 15) / 16; };
  uint32_t sum = 0;
  for (uint32_t u = lo; u < hi; ++u) sum += size16(u);
  uint32_t inc = sum;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const uint32_t y = __shfl_up_sync(~0u, inc, d);
    if (lane >= (uint32_t)d) inc += y;
  }
  if (lane == 31) warp_sum[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    uint32_t s = warp_sum[lane];
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const uint32_t y = __shfl_up_sync(~0u, s, d);
      if (lane >= (uint32_t)d) s += y;
    }
    warp_sum[lane] = s;
  }
  __syncthreads();
  uint32_t run = inc - sum + (warp ? warp_sum[warp - 1] : 0u);
  for (uint32_t u = lo; u < hi; ++u) {
    off16[u] = run;
    run += size16(u);
  }
  if (t == kScanThreads - 1) off16[units] = run;
}

// ============================================================ decode

constexpr int kDecWarps = 16;
constexpr int kDecThreads = 32 * kDecWarps;
constexpr uint32_t kWordBuf = 512;  // words per staging buffer (two per warp)
// per warp: two word buffers, then the segment's exponents
constexpr uint32_t kWarpSmem = 2 * kWordBuf * 2 + kSegVals;
constexpr uint32_t kDecSmem = kM * 4 + kDecWarps * kWarpSmem;
static_assert(kDecSmem <= 227 * 1024, "shared memory");

struct RansMat {
  const uint8_t *stream;
  const uint32_t *off16;
  const uint8_t *sm;
  const uint32_t *tables;
  uint16_t *out;
  uint64_t n;
  uint32_t units;
  uint32_t unit0;  // index of the matrix's first unit in the batch
};

struct RansDecParams {
  RansMat m[DF11_RANS_MAX_BATCH];
  uint32_t count;
  uint32_t total_units;
  uint32_t *status;
};

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all_but_one() {
  asm volatile("cp.async.wait_group 1;\n" ::: "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;\n" ::: "memory"); }

__device__ __forceinline__ uint4 ldg_stream(const void *p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

__device__ __forceinline__ void stg_stream(void *p, uint4 v) {
  asm volatile("st.global.cs.v4.u32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z),
               "r"(v.w)
               : "memory");
}

// 4 exponents + 4 sign/mantissa bytes -> 4 BF16 words (two 32-bit halves).
__device__ __forceinline__ void merge4(uint32_t e4, uint32_t s4, uint32_t &w01, uint32_t &w23) {
  const uint32_t hi4 = (s4 & 0x80808080u) | ((e4 >> 1) & 0x7F7F7F7Fu);
  const uint32_t lo4 = (s4 & 0x7F7F7F7Fu) | ((e4 << 7) & 0x80808080u);
  w01 = __byte_perm(lo4, hi4, 0x5140);
  w23 = __byte_perm(lo4, hi4, 0x7362);
}

// The segment's word range [s0, s1) widened to 16-byte boundaries; staged in
// shared memory when it fits a buffer.
struct SegRange {
  uint32_t a0, span;
};

__device__ __forceinline__ SegRange seg_range(uint32_t starts, int g, uint32_t navail) {
  uint32_t s1 = __shfl_sync(~0u, starts, g + 1);
  uint32_t s0 = __shfl_sync(~0u, starts, g);
  s1 = s1 < navail ? s1 : navail;
  s0 = s0 < s1 ? s0 : s1;
  SegRange r;
  r.a0 = s0 & ~7u;
  r.span = ((s1 + 7u) & ~7u) - r.a0;  // navail is a multiple of 8: stays inside the unit
  return r;
}

__device__ __forceinline__ void stage_words(const uint16_t *words, SegRange r, uint32_t buf_addr,
                                            uint32_t lane) {
  if (r.span <= kWordBuf)
    for (uint32_t c = lane; c < r.span / 8; c += 32) cp_async16(buf_addr + 16 * c, words + r.a0 + 8 * c);
  cp_async_commit();
}

// 64 steps of the unit's 32 states.  kFull: every value of the segment exists
// (else lane values at or past nv are skipped, as the encoder skipped them).
// kStaged: the segment's words are in shared memory at wb (word a0 first);
// otherwise they are read from global memory with a bounds check.
template <bool kFull, bool kStaged>
__device__ __forceinline__ void decode_segment(uint32_t &x, uint32_t &pos, const uint32_t *slot_s,
                                               uint8_t *ebuf, const uint16_t *wb, uint32_t a0,
                                               const uint16_t *words, uint32_t navail,
                                               uint32_t seg_first, uint32_t nv, uint32_t lane,
                                               uint32_t lt) {
#pragma unroll 16
  for (uint32_t k = 0; k < kSegSteps; ++k) {
    const bool act = kFull || seg_first + 32 * k + lane < nv;
    const uint32_t t = slot_s[x & (kM - 1)];
    const uint32_t q = x >> DF11_RANS_PROB_BITS;
    const uint32_t xn = (t >> 20) * q + q + ((t >> 8) & 0xFFF);  // f * (x / M) + slot - cum
    if (act) x = xn;
    ebuf[32 * k + lane] = (uint8_t)t;
    const bool need = act && x < kL;
    const uint32_t mask = __ballot_sync(~0u, need);
    if (need) {
      const uint32_t idx = pos + __popc(mask & lt);
      uint32_t word;
      if (kStaged)
        word = wb[(idx - a0) & (kWordBuf - 1)];
      else
        word = idx < navail ? __ldg(words + idx) : 0u;
      x = (x << 16) | word;
    }
    pos += __popc(mask);
  }
}

template <bool kFull>
__device__ __forceinline__ void decode_unit(const RansMat &M, uint32_t u, uint32_t lane,
                                            const uint32_t *slot_s, uint16_t *wbuf, uint8_t *ebuf,
                                            uint32_t *status) {
  const uint32_t lt = lanemask_lt();
  const uint32_t o0 = __ldg(M.off16 + u), o1 = __ldg(M.off16 + u + 1);
  const uint32_t oend = __ldg(M.off16 + M.units);
  if (o1 < o0 || o1 > oend || (uint64_t)(o1 - o0) * 16 < kHeader) {
    if (lane == 0) set_status(status, DF11_ERR_CORRUPT);
    return;
  }
  const uint8_t *base = M.stream + (uint64_t)o0 * 16;
  const uint32_t navail = (uint32_t)(((uint64_t)(o1 - o0) * 16 - kHeader) / 2);
  const uint16_t *words = reinterpret_cast<const uint16_t *>(base + kHeader);
  uint32_t x = __ldg(reinterpret_cast<const uint32_t *>(base) + lane);
  // lanes 0..7: first word of each segment; lane 8: the end of the words
  const uint32_t starts =
      lane < DF11_RANS_SEGMENTS ? (uint32_t)__ldg(reinterpret_cast<const uint16_t *>(base + 128) + lane)
                                : navail;
  const uint64_t v0 = (uint64_t)u * kUnit;
  const uint32_t nv = kFull ? kUnit : (uint32_t)(M.n - v0);
  const uint32_t wbuf_addr = (uint32_t)__cvta_generic_to_shared(wbuf);
  uint32_t pos = 0;
  bool bad = false;
  SegRange cur = seg_range(starts, 0, navail);
  stage_words(words, cur, wbuf_addr, lane);
#pragma unroll 1
  for (int g = 0; g < (int)DF11_RANS_SEGMENTS; ++g) {
    SegRange next{0, 0};
    if (g + 1 < (int)DF11_RANS_SEGMENTS) {
      next = seg_range(starts, g + 1, navail);
      stage_words(words, next, wbuf_addr + ((g + 1) & 1) * kWordBuf * 2, lane);
    } else {
      cp_async_commit();  // an empty group keeps the wait below uniform
    }
    const uint32_t seg_first = g * kSegVals;
    uint4 smv[4];
    if (kFull) {
#pragma unroll
      for (int j = 0; j < 4; ++j) smv[j] = ldg_stream(M.sm + v0 + seg_first + 16 * (lane + 32 * j));
    }
    cp_async_wait_all_but_one();
    __syncwarp();
    if (pos != __shfl_sync(~0u, starts, g)) bad = true;
    const uint16_t *wb = wbuf + (g & 1) * kWordBuf;
    if (cur.span <= kWordBuf)
      decode_segment<kFull, true>(x, pos, slot_s, ebuf, wb, cur.a0, words, navail, seg_first, nv,
                                  lane, lt);
    else
      decode_segment<kFull, false>(x, pos, slot_s, ebuf, wb, cur.a0, words, navail, seg_first, nv,
                                   lane, lt);
    __syncwarp();
    uint16_t *out = M.out + v0 + seg_first;
    if (kFull) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint32_t c = lane + 32 * j;  // 16 values
        const uint4 e = *reinterpret_cast<const uint4 *>(ebuf + 16 * c);
        uint4 a, b;
        merge4(e.x, smv[j].x, a.x, a.y);
        merge4(e.y, smv[j].y, a.z, a.w);
        merge4(e.z, smv[j].z, b.x, b.y);
        merge4(e.w, smv[j].w, b.z, b.w);
        stg_stream(out + 16 * c, a);
        stg_stream(out + 16 * c + 8, b);
      }
    } else {
      for (uint32_t i = lane; i < kSegVals; i += 32) {
        if (seg_first + i < nv) {
          const uint32_t e = ebuf[i], s = M.sm[v0 + seg_first + i];
          out[i] = (uint16_t)(((s & 0x80u) << 8) | (e << 7) | (s & 0x7Fu));
        }
      }
    }
    __syncwarp();
    cur = next;
  }
  cp_async_wait_all();
  // every state back at its start, every word read, only zero padding left
  if (!__all_sync(~0u, x == kL)) bad = true;
  if (pos > navail) {
    bad = true;
  } else {
    bool nz = false;
    for (uint32_t j = pos + lane; j < navail; j += 32) nz |= __ldg(words + j) != 0;
    if (__any_sync(~0u, nz)) bad = true;
  }
  if (bad && lane == 0) set_status(status, DF11_ERR_CORRUPT);
}

// Each CTA takes a contiguous share of the batch's units; within the share,
// per matrix: load its slot table, then warps take units round-robin.
__global__ void __launch_bounds__(kDecThreads, 2) rans_decode_kernel(const __grid_constant__ RansDecParams P) {
  extern __shared__ __align__(16) uint8_t smem[];
  uint32_t *slot_s = reinterpret_cast<uint32_t *>(smem);
  const uint32_t warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint8_t *wsm = smem + kM * 4 + warp * kWarpSmem;
  uint16_t *wbuf = reinterpret_cast<uint16_t *>(wsm);
  uint8_t *ebuf = wsm + 2 * kWordBuf * 2;
  const uint32_t g0 = (uint32_t)((uint64_t)blockIdx.x * P.total_units / gridDim.x);
  const uint32_t g1 = (uint32_t)((uint64_t)(blockIdx.x + 1) * P.total_units / gridDim.x);
  uint32_t gu = g0;
  while (gu < g1) {
    uint32_t m = 0;
    while (m + 1 < P.count && gu >= P.m[m + 1].unit0) ++m;
    const RansMat M = P.m[m];
    const uint32_t end = M.unit0 + M.units < g1 ? M.unit0 + M.units : g1;
    __syncthreads();  // the previous matrix's table is no longer read
    for (uint32_t i = threadIdx.x; i < kM / 4; i += kDecThreads)
      reinterpret_cast<uint4 *>(slot_s)[i] = __ldg(reinterpret_cast<const uint4 *>(M.tables) + i);
    __syncthreads();
    for (uint32_t v = gu + warp; v < end; v += kDecWarps) {
      const uint32_t u = v - M.unit0;
      if ((uint64_t)(u + 1) * kUnit <= M.n)
        decode_unit<true>(M, u, lane, slot_s, wbuf, ebuf, P.status);
      else
        decode_unit<false>(M, u, lane, slot_s, wbuf, ebuf, P.status);
    }
    gu = end;
  }
}

// ============================================================ launch helpers

struct DeviceInfo {
  int sms = 0;
  int dec_ctas_per_sm = 0;
  bool configured = false;
};

std::mutex g_mu;
DeviceInfo g_dev[64];

df11_status device_info(int *sms, int *dec_per_sm) {
  int dev;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return DF11_ERR_NO_DEVICE;
  }
  if (dev < 0 || dev >= 64) return DF11_ERR_NO_DEVICE;
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceInfo &d = g_dev[dev];
  if (!d.configured) {
    if (cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return DF11_ERR_CUDA;
    if (cudaFuncSetAttribute(rans_decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kDecSmem) != cudaSuccess)
      return DF11_ERR_CUDA;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&d.dec_ctas_per_sm, rans_decode_kernel,
                                                      kDecThreads, kDecSmem) != cudaSuccess ||
        d.dec_ctas_per_sm < 1)
      return DF11_ERR_CUDA;
    d.configured = true;
  }
  *sms = d.sms;
  *dec_per_sm = d.dec_ctas_per_sm;
  return DF11_OK;
}

inline bool aligned(const void *p, uintptr_t a) { return ((uintptr_t)p & (a - 1)) == 0; }

df11_status launch_status() {
  return cudaGetLastError() == cudaSuccess ? DF11_OK : DF11_ERR_CUDA;
}

df11_status check_encode_args(const uint16_t *d_w, uint64_t n, const void *d_tables) {
  if (n > DF11_MAX_N) return DF11_ERR_TOO_LARGE;
  if (n && (!d_w || !d_tables || !aligned(d_w, 16) || !aligned(d_tables, 16)))
    return DF11_ERR_INVALID_ARG;
  return DF11_OK;
}

uint32_t encode_grid(uint32_t units, int sms) {
  const uint32_t want = (units + kEncWarps - 1) / kEncWarps;
  const uint32_t cap = (uint32_t)sms * 8;
  return want < cap ? want : cap;
}

}  // namespace

// ============================================================ C ABI

extern "C" df11_status df11_rans_encode_sizes(const uint16_t *d_w, uint64_t n, const void *d_tables,
                                              uint32_t *d_unit_words, uint32_t *d_off16,
                                              uint32_t *d_status, df11_stream_t stream) {
  df11_status st = check_encode_args(d_w, n, d_tables);
  if (st != DF11_OK) return st;
  if (!d_off16 || !aligned(d_off16, 4) || (n && (!d_unit_words || !aligned(d_unit_words, 4))))
    return DF11_ERR_INVALID_ARG;
  int sms, per_sm;
  if ((st = device_info(&sms, &per_sm)) != DF11_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const uint32_t units = (uint32_t)df11_rans_units(n);
  if (units == 0) {
    if (cudaMemsetAsync(d_off16, 0, 4, s) != cudaSuccess) return DF11_ERR_CUDA;
    return DF11_OK;
  }
  rans_encode_kernel<false><<<encode_grid(units, sms), kEncThreads, 0, s>>>(
      d_w, n, static_cast<const uint32_t *>(d_tables), units, d_unit_words, nullptr, nullptr,
      nullptr, d_status);
  rans_scan_kernel<<<1, kScanThreads, 0, s>>>(d_unit_words, units, d_off16);
  return launch_status();
}

extern "C" df11_status df11_rans_encode(const uint16_t *d_w, uint64_t n, const void *d_tables,
                                        const uint32_t *d_unit_words, const uint32_t *d_off16,
                                        uint8_t *d_stream, uint8_t *d_sign_mantissa,
                                        uint32_t *d_status, df11_stream_t stream) {
  df11_status st = check_encode_args(d_w, n, d_tables);
  if (st != DF11_OK) return st;
  if (n == 0) return DF11_OK;
  if (!d_unit_words || !d_off16 || !d_stream || !d_sign_mantissa || !aligned(d_off16, 4) ||
      !aligned(d_unit_words, 4) || !aligned(d_stream, 16))
    return DF11_ERR_INVALID_ARG;
  int sms, per_sm;
  if ((st = device_info(&sms, &per_sm)) != DF11_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const uint32_t units = (uint32_t)df11_rans_units(n);
  rans_encode_kernel<true><<<encode_grid(units, sms), kEncThreads, 0, s>>>(
      d_w, n, static_cast<const uint32_t *>(d_tables), units, const_cast<uint32_t *>(d_unit_words),
      d_off16, d_stream, d_sign_mantissa, d_status);
  return launch_status();
}

extern "C" df11_status df11_rans_decode_batch(const df11_rans_matrix *ms, uint32_t count,
                                              uint16_t *const *d_outs, uint32_t *d_status,
                                              df11_stream_t stream) {
  if (count && (!ms || !d_outs)) return DF11_ERR_INVALID_ARG;
  for (uint32_t i = 0; i < count; ++i) {
    const df11_rans_matrix &m = ms[i];
    if (m.n > DF11_MAX_N) return DF11_ERR_TOO_LARGE;
    if (m.n && (!m.stream || !m.off16 || !m.sign_mantissa || !m.tables || !d_outs[i] ||
                !aligned(m.stream, 16) || !aligned(m.off16, 4) || !aligned(m.sign_mantissa, 16) ||
                !aligned(m.tables, 16) || !aligned(d_outs[i], 16)))
      return DF11_ERR_INVALID_ARG;
  }
  int sms, per_sm;
  df11_status st = device_info(&sms, &per_sm);
  if (st != DF11_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  for (uint32_t first = 0; first < count; first += DF11_RANS_MAX_BATCH) {
    RansDecParams P{};
    P.status = d_status;
    uint32_t total = 0;
    for (uint32_t i = first; i < count && P.count < DF11_RANS_MAX_BATCH; ++i) {
      const df11_rans_matrix &m = ms[i];
      const uint32_t units = (uint32_t)df11_rans_units(m.n);
      if (!units) continue;
      RansMat &r = P.m[P.count++];
      r.stream = m.stream;
      r.off16 = m.off16;
      r.sm = m.sign_mantissa;
      r.tables = static_cast<const uint32_t *>(m.tables);
      r.out = d_outs[i];
      r.n = m.n;
      r.units = units;
      r.unit0 = total;
      total += units;
    }
    if (!total) continue;
    P.total_units = total;
    const uint32_t cap = (uint32_t)(sms * per_sm);
    const uint32_t want = (total + kDecWarps - 1) / kDecWarps;
    rans_decode_kernel<<<want < cap ? want : cap, kDecThreads, kDecSmem, s>>>(P);
    if ((st = launch_status()) != DF11_OK) return st;
  }
  return DF11_OK;
}
