// Tensor-core decode kernels: the tcgen05 absorbed decode (decode_tc.cu) and the grouped
// (GQA-path) decode (decode_grouped.cu).
#pragma once

#include "kernels.h"

namespace mla {

// Absorbed path, bf16, H=128, d_c=512, d_rope=64, page 64.
bool tc_available();
int tc_units(int sms);        // concurrent workers the split plan should cover
int tc_token_granule();       // chunk lengths are multiples of this many tokens
cudaError_t launch_tc_decode(const Dims &d, const void *q_abs, const void *latent, const int *page_table,
                             const Plan &plan, int max_pages, int n_pages, int s_q, float *part_o,
                             float *part_ml, int *err, int sms, cudaStream_t st);

// Test hook of the bounded waits: later tcgen05 decodes on the calling thread skip the completion
// signal of pipeline step `withhold_step` (-1: none) and give up every wait after `wait_ns`
// (0: the default 2 s).
void tc_set_test_fault(int withhold_step, uint64_t wait_ns);

// Grouped path, bf16, d_nope = d_v = 128, d_rope = 64, heads_per_group = 8.
bool grouped_tc_ok(const Dims &d, int s_q);   // s_q <= 4: 16-row tiles of 8 heads x 2 queries
int grouped_units(const Dims &d, int sms);
int grouped_token_granule();
// Head-expanded prefill over the expanded cache (per head with heads_per_group = 1, or per
// group): bf16, d_nope = d_v = 128, d_rope = 64, d_c = 512, page 64.  n_q query tokens per
// request (the last n_q positions), partials [n_work * n_q, H, 128] for the combine.
bool prefill_ok(const Dims &d);
cudaError_t launch_prefill_expanded(const Dims &d, const void *q_rot, const void *expanded, const void *latent,
                                    const int *seq_lens, const int *page_table, const Plan &plan, int max_pages,
                                    int n_pages, int n_q, float *part_o, float *part_ml, int *err, cudaStream_t st);
// tcgen05 head-expanded prefill (prefill_tc.cu), the kernel behind launch_prefill_expanded.
cudaError_t launch_prefill_tc(const Dims &d, const void *q_rot, const void *expanded, const void *latent,
                              const int *seq_lens, const int *page_table, const Plan &plan, int max_pages,
                              int n_pages, int n_q, float *part_o, float *part_ml, int *err, cudaStream_t st);
cudaError_t launch_grouped_decode(const Dims &d, const void *q, const void *expanded, const void *latent,
                                  const int *seq_lens, const int *page_table, const Plan &plan, int max_pages,
                                  int n_pages, int s_q, float *part_o, float *part_ml, int *err, cudaStream_t st);

}  // namespace mla
