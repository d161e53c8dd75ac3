// Host side of the split-KV plan (the device side is plan.cu).  Both follow one rule:
// row (b, j) has len = seq_lens[b] - s_q + j + 1 tokens, cut into ceil(len / chunk) chunks.
#pragma once

#include <stdint.h>

#include <algorithm>

namespace mla {

// Chunk length (a multiple of `granule` tokens) that spreads all rows' tokens over about
// `units` concurrently running workers.
inline int plan_chunk(const int32_t *lens, int batch, int s_q, int units, int granule) {
    long long total = 0;
    for (int b = 0; b < batch; ++b)
        for (int j = 0; j < s_q; ++j) total += (long long)lens[b] - s_q + j + 1;
    long long c = (total + units - 1) / std::max(1, units);
    c = (c + granule - 1) / granule * granule;
    c = std::max<long long>(c, granule);
    return (int)std::min<long long>(c, 1 << 30);
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
