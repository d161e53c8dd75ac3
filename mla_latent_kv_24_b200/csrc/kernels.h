// Host-side launchers of the libmla kernels (one per .cu file).  Called only by api.cu.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"

namespace mla {

struct Dims {
    int H, hpw, d_c, d_r, d_n, d_v, page;
    float scale, base;
    int bf16;  // 1 = bf16 storage, 0 = fp32
    int n_groups() const { return H / hpw; }
    int d_row() const { return d_c + d_r; }
};

// Down-projection + RoPE + paged scatter of new tokens (append.cu).
cudaError_t launch_append(const Dims &d, const void *h, int hidden, const void *W_dkv,
                          const void *W_kr, const int *req, const int *pos, int n_tok,
                          const int *page_table, int batch, int max_pages, int n_pages,
                          void *cache, int *err, cudaStream_t st);

// Tensor-core append (bf16, d_c = 512, d_rope = 64, page 64, projected input) (append.cu).
bool append_mma_ok(const Dims &d, int hidden, bool projected);
cudaError_t launch_append_mma(const Dims &d, const void *h, int hidden, const void *W_dkv, const void *W_kr,
                              const int *req, const int *pos, int n_tok, const int *page_table, int batch,
                              int max_pages, int n_pages, void *cache, int *err, cudaStream_t st);

// Split plan from device seq_lens as a kernel of its own (plan.cu).  launch_q_absorb_mma and
// launch_q_rope build the same plan in an extra block instead.
cudaError_t launch_plan(const PlanArgs &a, cudaStream_t st);

// q absorption through W_UK + RoPE of the query's RoPE part (absorb.cu):
//   q_abs [rows, H, d_c + d_r] = [W_UK[w]^T q_nope | RoPE(q_rope, p)], rows = batch * s_q.
cudaError_t launch_q_absorb(const Dims &d, const void *q, const void *W_uk, const int *seq_lens,
                            int batch, int s_q, void *q_abs, cudaStream_t st);

// Tensor-core variant for bf16, d_nope = 128, d_c = 512, d_rope = 64 (absorb.cu).
bool q_absorb_mma_ok(const Dims &d);
// It also builds the split plan `plan` in one extra block.
cudaError_t launch_q_absorb_mma(const Dims &d, const void *q, const void *W_uk, const int *seq_lens, int batch,
                                int s_q, void *q_abs, const PlanArgs &plan, cudaStream_t st);

// RoPE of the query's RoPE part only (absorb.cu): q_rot [rows, H, d_n + d_r]; the split plan
// `plan` is built in one extra block.
cudaError_t launch_q_rope(const Dims &d, const void *q, const int *seq_lens, int batch, int s_q,
                          void *q_rot, const PlanArgs &plan, cudaStream_t st);

// General CUDA-core split flash decode (decode_simt.cu).  mode 0: absorbed (keys and values
// are latent rows); mode 1: grouped (keys = [K_g | k_rope], values = V_g).
struct SimtDecodeArgs {
    const void *q;  // absorbed: q_abs [rows, H, d_c + d_r]; grouped: q_rot [rows, H, d_n + d_r]
    const void *latent;
    const void *expanded;
    const int *page_table;
    Plan plan;
    int max_pages, n_pages, s_q, mode;
    float *part_o;   // [n_work, H, DV]
    float *part_ml;  // [n_work, H, 2]
    int *err;
};
cudaError_t launch_decode_simt(const Dims &d, const SimtDecodeArgs &a, cudaStream_t st);
int simt_heads_per_block(const Dims &d, int mode);

// Split combine (+ W_UV up-projection when W_uv != nullptr) (combine.cu).
//   out [rows, H, d_v].  Output row r = (b, j) merges plan row r / qpi: partial results
//   k * qpi + r % qpi for its work items k (qpi = 1 when every plan row is one query).
cudaError_t launch_combine(const Dims &d, const float *part_o, const float *part_ml,
                           const int *row_first, int rows, int qpi, int DV, const void *W_uv, void *out,
                           cudaStream_t st);

// Tensor-core combine + W_UV for bf16, d_c = 512, d_v = 128 (combine.cu).  oct_layout: the
// partials are in the tcgen05 decode's column-octet layout [n_work, 64, H, 8] instead of
// [n_work, H, 512].
// rows_host: the plan's row starts computed on the host from the host lengths (rows + 1 values),
// or nullptr; batches of at most RowStarts::MAX rows pass them by value, which saves the kernel a
// dependent load (the device plan still validates the lengths and reports a mismatch).
struct RowStarts {
    static constexpr int MAX = 64;
    int n;              // rows covered (0: read row_first from the workspace)
    int v[MAX + 1];
};
bool combine_mma_ok(const Dims &d, int DV, bool project);
cudaError_t launch_combine_mma(const Dims &d, const float *part_o, const float *part_ml, const int *row_first,
                               const int *rows_host, int rows, bool oct_layout, const void *W_uv, void *out,
                               cudaStream_t st);

// Per-group cache expansion (expand.cu).
cudaError_t launch_expand(const Dims &d, const void *W_uk, const void *W_uv, const void *latent,
                          const int *page_ids, int n_ids, int n_pages, void *expanded, int *err,
                          cudaStream_t st);
cudaError_t launch_expand_tokens(const Dims &d, const void *W_uk, const void *W_uv, const void *latent,
                                 const int *req, const int *pos, int n_tok, const int *page_table, int batch,
                                 int max_pages, int n_pages, void *expanded, int *err, cudaStream_t st);

}  // namespace mla
