// Host side of the split-KV plan (the device side is plan_block.cuh).  Both follow one rule:
// row (b, j) has len = seq_lens[b] - s_q + j + 1 tokens, cut into ceil(len / chunk) chunks.
#pragma once

#include <stdint.h>

#include <algorithm>

namespace mla {

inline long long plan_count(const int32_t *lens, int batch, int s_q, int chunk);

// Chunk length (a multiple of `granule` tokens) that spreads all rows' tokens over about
// `units` concurrently running workers: the smallest such length whose chunk count fits in
// one wave of `units` when that is possible (more chunks than workers would leave a second,
// mostly idle wave).  Otherwise (more rows than workers) workers take several chunks each, and
// three quarters of the even split of all tokens: the smaller chunks balance the workers'
// totals better (a ragged batch of 128 rows on 74 tcgen05 workers: 275 -> 264 us; half the
// even split paid more in per-chunk overhead than it gained).
inline int plan_chunk(const int32_t *lens, int batch, int s_q, int units, int granule) {
    long long total = 0, longest = 1;
    for (int b = 0; b < batch; ++b)
        for (int j = 0; j < s_q; ++j) {
            const long long len = (long long)lens[b] - s_q + j + 1;
            total += len;
            longest = std::max(longest, len);
        }
    units = std::max(1, units);
    auto round_up = [&](long long c) { return std::max<long long>(granule, (c + granule - 1) / granule * granule); };
    long long lo = round_up((total + units - 1) / units);
    long long hi = round_up(longest);
    if (lo >= hi) return (int)std::min<long long>(lo, 1 << 30);
    if (plan_count(lens, batch, s_q, (int)std::min<long long>(hi, 1 << 30)) > units)
        return (int)std::min<long long>(round_up(lo * 3 / 4), 1 << 30);
    while (lo < hi) {  // smallest multiple of granule in [lo, hi] with count <= units
        const long long mid = round_up((lo + hi) / 2 - granule + 1);
        const long long m = mid < lo ? lo : mid;
        if (plan_count(lens, batch, s_q, (int)m) <= units)
            hi = m;
        else
            lo = m + granule;
    }
    return (int)std::min<long long>(lo, 1 << 30);
}

inline long long plan_count(const int32_t *lens, int batch, int s_q, int chunk) {
    long long n = 0;
    for (int b = 0; b < batch; ++b)
        for (int j = 0; j < s_q; ++j) {
            const long long len = (long long)lens[b] - s_q + j + 1;
            n += (len + chunk - 1) / chunk;
        }
    return n;
}

}  // namespace mla
