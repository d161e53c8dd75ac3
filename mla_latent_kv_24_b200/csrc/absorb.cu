// Query preparation.
//
// q absorption ("How to upgrade GQA models to MLA ...", stage "Decompression Multiplex": by
// associativity W_UK folds into the query, which then lives in latent space):
//     q_lat[row, h, :] = W_UK[w(h)]^T q_nope[row, h, :]                (d_c)
// followed by RoPE of the query's RoPE part at its position p = seq_lens[b] - s_q + j.
// Output q_abs[row, h, :] = [q_lat | RoPE(q_rope, p)], in the storage dtype (bf16 rounding
// once, fp32 accumulation).
//
// One CTA handles one head and up to RB query rows, so each W_UK row is read once per RB
// rows; every thread owns two latent columns.
#include "kernels.h"

namespace mla {
namespace {

constexpr int RB = 16;

template <typename T>
__global__ void __launch_bounds__(256) q_absorb_kernel(const T *__restrict__ q, const T *__restrict__ W_uk,
                                                       const int *__restrict__ seq_lens, int rows, int s_q,
                                                       int H, int hpw, int d_c, int d_r, int d_n, float base,
                                                       T *__restrict__ q_abs) {
    __shared__ float qn[RB][128];
    const int h = blockIdx.x, w = h / hpw;
    const int row0 = blockIdx.y * RB;
    const int nr = min(RB, rows - row0);
    const int d_qk = d_n + d_r, d_out = d_c + d_r;
    for (int i = threadIdx.x; i < RB * d_n; i += blockDim.x) {
        int r = i / d_n, k = i % d_n;
        qn[r][k] = r < nr ? to_f32(q[((size_t)(row0 + r) * H + h) * d_qk + k]) : 0.f;
    }
    __syncthreads();
    const T *Wk = W_uk + (size_t)w * d_n * d_c;
    for (int c = threadIdx.x; c < d_c; c += blockDim.x) {
        float acc[RB];
#pragma unroll
        for (int r = 0; r < RB; ++r) acc[r] = 0.f;
        for (int k = 0; k < d_n; ++k) {
            const float wv = to_f32(Wk[(size_t)k * d_c + c]);
#pragma unroll
            for (int r = 0; r < RB; ++r) acc[r] += qn[r][k] * wv;
        }
        for (int r = 0; r < nr; ++r) q_abs[((size_t)(row0 + r) * H + h) * d_out + c] = from_f32<T>(acc[r]);
    }
    // RoPE part: pair i of the query's RoPE vector turns by p * base^(-2i/d_r).
    for (int i = threadIdx.x; i < nr * (d_r / 2); i += blockDim.x) {
        const int r = i / (d_r / 2), pi = i % (d_r / 2);
        const int row = row0 + r, b = row / s_q, j = row % s_q;
        const int p = seq_lens[b] - s_q + j;
        const T *src = q + ((size_t)row * H + h) * d_qk + d_n + 2 * pi;
        float x0 = to_f32(src[0]), x1 = to_f32(src[1]), cs, sn;
        rope_cos_sin(p, pi, d_r, base, &cs, &sn);
        T *dst = q_abs + ((size_t)row * H + h) * d_out + d_c + 2 * pi;
        dst[0] = from_f32<T>(x0 * cs - x1 * sn);
        dst[1] = from_f32<T>(x0 * sn + x1 * cs);
    }
}

// GQA path: the no-position part is used as is; only the RoPE part turns.
template <typename T>
__global__ void q_rope_kernel(const T *__restrict__ q, const int *__restrict__ seq_lens, int rows, int s_q,
                              int H, int d_r, int d_n, float base, T *__restrict__ q_rot) {
    const int d_qk = d_n + d_r;
    const size_t n = (size_t)rows * H * (d_qk / 2);
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
        const int pr = (int)(i % (d_qk / 2));
        const size_t rh = i / (d_qk / 2);
        const int row = (int)(rh / H);
        const T *src = q + rh * d_qk + 2 * pr;
        T *dst = q_rot + rh * d_qk + 2 * pr;
        if (2 * pr < d_n) {
            dst[0] = src[0];
            dst[1] = src[1];
        } else {
            const int b = row / s_q, j = row % s_q, p = seq_lens[b] - s_q + j;
            float x0 = to_f32(src[0]), x1 = to_f32(src[1]), cs, sn;
            rope_cos_sin(p, (2 * pr - d_n) / 2, d_r, base, &cs, &sn);
            dst[0] = from_f32<T>(x0 * cs - x1 * sn);
            dst[1] = from_f32<T>(x0 * sn + x1 * cs);
        }
    }
}

}  // namespace

cudaError_t launch_q_absorb(const Dims &d, const void *q, const void *W_uk, const int *seq_lens, int batch,
                            int s_q, void *q_abs, cudaStream_t st) {
    const int rows = batch * s_q;
    dim3 grid(d.H, ceil_div(rows, RB));
    if (d.bf16)
        q_absorb_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(
            (const __nv_bfloat16 *)q, (const __nv_bfloat16 *)W_uk, seq_lens, rows, s_q, d.H, d.hpw, d.d_c,
            d.d_r, d.d_n, d.base, (__nv_bfloat16 *)q_abs);
    else
        q_absorb_kernel<float><<<grid, 256, 0, st>>>((const float *)q, (const float *)W_uk, seq_lens, rows, s_q,
                                                     d.H, d.hpw, d.d_c, d.d_r, d.d_n, d.base, (float *)q_abs);
    return cudaGetLastError();
}

cudaError_t launch_q_rope(const Dims &d, const void *q, const int *seq_lens, int batch, int s_q, void *q_rot,
                          cudaStream_t st) {
    const int rows = batch * s_q;
    const size_t n = (size_t)rows * d.H * ((d.d_n + d.d_r) / 2);
    const int blocks = (int)std::min<size_t>((n + 255) / 256, 4096);
    if (d.bf16)
        q_rope_kernel<__nv_bfloat16><<<blocks, 256, 0, st>>>((const __nv_bfloat16 *)q, seq_lens, rows, s_q, d.H,
                                                              d.d_r, d.d_n, d.base, (__nv_bfloat16 *)q_rot);
    else
        q_rope_kernel<float><<<blocks, 256, 0, st>>>((const float *)q, seq_lens, rows, s_q, d.H, d.d_r, d.d_n,
                                                     d.base, (float *)q_rot);
    return cudaGetLastError();
}

}  // namespace mla
