// rans_host.cpp -- host side of the rANS exponent-codec variant: frequencies
// from a histogram and the device tables (include/df11_rans.h).
//
// The frequency rule is a largest-remainder apportionment of c*M/n with
// M = 4096: every present exponent first gets floor(c*M/n), at least 1.  If
// that leaves the sum short, the exponents with the largest remainders
// (c*M - f*n) get one more each, ties to the smaller exponent.  If raising
// rare exponents to 1 overshot M, one is taken back at a time from the
// exponent with f > 1 whose current f is most above its share (smallest
// c*M - f*n, ties to the smaller exponent).
#include <stdint.h>
#include <string.h>

#include <algorithm>
#include <vector>

#include "df11_rans.h"

namespace {

constexpr uint32_t kM = 1u << DF11_RANS_PROB_BITS;

}  // namespace

extern "C" df11_status df11_rans_freqs(const uint64_t hist256[256], uint32_t freq[256]) {
  if (!hist256 || !freq) return DF11_ERR_INVALID_ARG;
  uint64_t n = 0;
  std::vector<int> present;
  for (int s = 0; s < 256; s++) {
    freq[s] = 0;
    if (hist256[s]) {
      if (n + hist256[s] < n) return DF11_ERR_TOO_LARGE;
      n += hist256[s];
      present.push_back(s);
    }
  }
  if (present.empty()) return DF11_OK;
  if (n > DF11_MAX_N) return DF11_ERR_TOO_LARGE;
  if (present.size() == 1) {
    freq[present[0]] = kM;
    return DF11_OK;
  }
  // remainder of each exponent's share against its current frequency, in
  // units of 1/n (c*M < 2^44: fits int64 with room)
  auto rem = [&](int s) {
    return (int64_t)(hist256[s] * kM) - (int64_t)freq[s] * (int64_t)n;
  };
  int64_t total = 0;
  for (int s : present) {
    uint64_t share = hist256[s] * kM / n;
    freq[s] = share ? (uint32_t)share : 1u;
    total += freq[s];
  }
  if (total < (int64_t)kM) {
    std::vector<int> order(present);
    std::stable_sort(order.begin(), order.end(),
                     [&](int a, int b) { return rem(a) > rem(b); });  // present is ascending
    const int64_t short_by = (int64_t)kM - total;
    if (short_by > (int64_t)order.size()) return DF11_ERR_INVALID_ARG;  // cannot happen
    for (int64_t i = 0; i < short_by; i++) freq[order[i]]++;
    return DF11_OK;
  }
  while (total > (int64_t)kM) {
    int best = -1;
    for (int s : present)
      if (freq[s] > 1 && (best < 0 || rem(s) < rem(best))) best = s;
    if (best < 0) return DF11_ERR_INVALID_ARG;  // more than 4096 exponents: cannot happen
    freq[best]--;
    total--;
  }
  return DF11_OK;
}

extern "C" df11_status df11_rans_build_tables(const uint32_t freq[256], void *h_tables,
                                              size_t bytes) {
  if (!freq || !h_tables || bytes < DF11_RANS_TABLES_BYTES) return DF11_ERR_INVALID_ARG;
  uint64_t sum = 0;
  for (int s = 0; s < 256; s++) {
    if (freq[s] > kM) return DF11_ERR_INVALID_ARG;
    sum += freq[s];
  }
  if (sum != 0 && sum != kM) return DF11_ERR_INVALID_ARG;
  uint32_t *slot = static_cast<uint32_t *>(h_tables);
  uint32_t *enc = slot + kM;
  memset(h_tables, 0, DF11_RANS_TABLES_BYTES);
  uint32_t cum = 0;
  for (uint32_t s = 0; s < 256; s++) {
    const uint32_t f = freq[s];
    enc[s] = f ? (f | (cum << 16)) : 0u;
    for (uint32_t j = 0; j < f; j++) slot[cum + j] = s | (j << 8) | ((f - 1) << 20);
    cum += f;
  }
  return DF11_OK;
}

extern "C" uint64_t df11_rans_units(uint64_t n) {
  return (n + DF11_RANS_UNIT - 1) / DF11_RANS_UNIT;
}

extern "C" df11_status df11_rans_validate(uint64_t n, const uint8_t *h_stream,
                                          uint64_t stream_bytes, const uint32_t *h_off16,
                                          uint64_t off16_count) {
  if (n > DF11_MAX_N) return DF11_ERR_TOO_LARGE;
  const uint64_t units = df11_rans_units(n);
  if (!h_off16 || off16_count != units + 1 || (stream_bytes && !h_stream))
    return DF11_ERR_INVALID_ARG;
  if (h_off16[0] != 0 || (uint64_t)h_off16[units] * 16 != stream_bytes) return DF11_ERR_CORRUPT;
  // every offset first, so that every unit read below lies inside the stream
  for (uint64_t u = 0; u < units; ++u)
    if (h_off16[u + 1] < h_off16[u]) return DF11_ERR_CORRUPT;
  const uint64_t max_unit = DF11_RANS_HEADER_BYTES + 2ull * DF11_RANS_UNIT + 15;
  for (uint64_t u = 0; u < units; ++u) {
    const uint64_t bytes = (uint64_t)(h_off16[u + 1] - h_off16[u]) * 16;
    if (bytes < DF11_RANS_HEADER_BYTES || bytes > max_unit) return DF11_ERR_CORRUPT;
    const uint8_t *p = h_stream + (uint64_t)h_off16[u] * 16;
    const uint64_t words = (bytes - DF11_RANS_HEADER_BYTES) / 2;
    uint64_t prev = 0;
    for (unsigned g = 0; g < DF11_RANS_SEGMENTS; ++g) {
      const uint64_t st = (uint64_t)p[128 + 2 * g] | (uint64_t)p[129 + 2 * g] << 8;
      if ((g == 0 && st != 0) || st < prev || st > words) return DF11_ERR_CORRUPT;
      prev = st;
    }
    // values of this unit: lane l codes ceil((m - l) / 32) of them
    const uint64_t m = n - u * DF11_RANS_UNIT < DF11_RANS_UNIT ? n - u * DF11_RANS_UNIT
                                                               : DF11_RANS_UNIT;
    for (unsigned l = 0; l < DF11_RANS_LANES; ++l) {
      const uint32_t x = (uint32_t)p[4 * l] | (uint32_t)p[4 * l + 1] << 8 |
                         (uint32_t)p[4 * l + 2] << 16 | (uint32_t)p[4 * l + 3] << 24;
      if (x < (1u << 16)) return DF11_ERR_CORRUPT;
      if (l >= m && x != (1u << 16)) return DF11_ERR_CORRUPT;
    }
  }
  return DF11_OK;
}
