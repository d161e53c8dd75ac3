// Cache append: down-projection of the new tokens' hidden states into the latent c^KV and
// the RoPE key k^R, rotation of k^R at the token's position, and scatter into the paged
// latent cache ("MLA and GRPO architecture", "The Mathematics of MLA": c_t^KV = W_DKV h_t;
// "Decoupled RoPE": cached state [c_t^KV, k_t^R]).
//
// One CTA computes a tile of 16 new tokens x 64 output columns of the [n_tok, d_c + d_r]
// projection, streaming the hidden dimension in 32-wide slices through shared memory.  The
// work is bound by reading W_DKV / W_KR once (5.9 MB at DeepSeek-V2 dims); the tile keeps
// every weight element read once per 16 tokens.
#include "kernels.h"

namespace mla {
namespace {

constexpr int TOK = 16, COLS = 64, KT = 32;

template <typename T>
__global__ void __launch_bounds__(256) append_kernel(
    const T *__restrict__ h, int hidden, const T *__restrict__ W_dkv, const T *__restrict__ W_kr,
    const int *__restrict__ req, const int *__restrict__ pos, int n_tok,
    const int *__restrict__ page_table, int batch, int max_pages, int n_pages, int page, int d_c,
    int d_r, float base, T *__restrict__ cache, int *err) {
    const int d_row = d_c + d_r;
    __shared__ float hs[TOK][KT + 1];
    __shared__ float ws[COLS][KT + 1];
    const int tid = threadIdx.x;
    const int n0 = blockIdx.y * TOK, c0 = blockIdx.x * COLS;
    const int tt = tid / 16;          // token inside the tile
    const int cp = tid % 16;          // column pair: columns 2cp, 2cp+1 and 2cp+32, 2cp+33
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    const int n = n0 + tt;

    if (W_dkv != nullptr) {
        for (int k0 = 0; k0 < hidden; k0 += KT) {
            for (int i = tid; i < TOK * KT; i += 256) {
                int r = i / KT, k = i % KT;
                hs[r][k] = (n0 + r < n_tok && k0 + k < hidden) ? to_f32(h[(size_t)(n0 + r) * hidden + k0 + k]) : 0.f;
            }
            for (int i = tid; i < COLS * KT; i += 256) {
                int r = i / KT, k = i % KT, c = c0 + r;
                float v = 0.f;
                if (c < d_row && k0 + k < hidden)
                    v = c < d_c ? to_f32(W_dkv[(size_t)c * hidden + k0 + k])
                                : to_f32(W_kr[(size_t)(c - d_c) * hidden + k0 + k]);
                ws[r][k] = v;
            }
            __syncthreads();
#pragma unroll 8
            for (int k = 0; k < KT; ++k) {
                float x = hs[tt][k];
                acc[0] += x * ws[2 * cp][k];
                acc[1] += x * ws[2 * cp + 1][k];
                acc[2] += x * ws[2 * cp + 32][k];
                acc[3] += x * ws[2 * cp + 33][k];
            }
            __syncthreads();
        }
    } else if (n < n_tok) {
        // Pre-projected input: h already holds [c | k_rope before rotation].
        int cols[4] = {c0 + 2 * cp, c0 + 2 * cp + 1, c0 + 2 * cp + 32, c0 + 2 * cp + 33};
        for (int i = 0; i < 4; ++i)
            acc[i] = cols[i] < d_row ? to_f32(h[(size_t)n * hidden + cols[i]]) : 0.f;
    }
    if (n >= n_tok) return;

    const int b = req[n], p = pos[n];
    if (b < 0 || b >= batch || p < 0 || p >= max_pages * page) {
        report(err, MLA_ERR_DEVICE_BOUNDS);
        return;
    }
    const int pid = page_table[(size_t)b * max_pages + p / page];
    if (pid < 0 || pid >= n_pages) {
        report(err, MLA_ERR_DEVICE_BOUNDS);
        return;
    }
    T *dst = cache + ((size_t)pid * page + p % page) * d_row;
#pragma unroll
    for (int half = 0; half < 2; ++half) {
        const int c = c0 + 2 * cp + 32 * half;
        if (c >= d_row) continue;
        float x0 = acc[2 * half], x1 = acc[2 * half + 1];
        if (c >= d_c) {  // RoPE on the interleaved pair (c - d_c, c - d_c + 1)
            float cs, sn;
            rope_cos_sin(p, (c - d_c) / 2, d_r, base, &cs, &sn);
            float y0 = x0 * cs - x1 * sn, y1 = x0 * sn + x1 * cs;
            x0 = y0;
            x1 = y1;
        }
        dst[c] = from_f32<T>(x0);
        if (c + 1 < d_row) dst[c + 1] = from_f32<T>(x1);
    }
}

}  // namespace

cudaError_t launch_append(const Dims &d, const void *h, int hidden, const void *W_dkv,
                          const void *W_kr, const int *req, const int *pos, int n_tok,
                          const int *page_table, int batch, int max_pages, int n_pages,
                          void *cache, int *err, cudaStream_t st) {
    dim3 grid(ceil_div(d.d_row(), COLS), ceil_div(n_tok, TOK));
    if (d.bf16)
        append_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(
            (const __nv_bfloat16 *)h, hidden, (const __nv_bfloat16 *)W_dkv, (const __nv_bfloat16 *)W_kr,
            req, pos, n_tok, page_table, batch, max_pages, n_pages, d.page, d.d_c, d.d_r, d.base,
            (__nv_bfloat16 *)cache, err);
    else
        append_kernel<float><<<grid, 256, 0, st>>>(
            (const float *)h, hidden, (const float *)W_dkv, (const float *)W_kr, req, pos, n_tok,
            page_table, batch, max_pages, n_pages, d.page, d.d_c, d.d_r, d.base, (float *)cache, err);
    return cudaGetLastError();
}

}  // namespace mla
