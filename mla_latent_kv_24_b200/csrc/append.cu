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
    step_begin();
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
        MLA_STEP_LAUNCH(append_kernel<__nv_bfloat16>, dim3(grid), dim3(256), 0, st, (const __nv_bfloat16 *)h, hidden,
                        (const __nv_bfloat16 *)W_dkv, (const __nv_bfloat16 *)W_kr, req, pos, n_tok, page_table, batch,
                        max_pages, n_pages, d.page, d.d_c, d.d_r, d.base, (__nv_bfloat16 *)cache, err);
    else
        MLA_STEP_LAUNCH(append_kernel<float>, dim3(grid), dim3(256), 0, st, (const float *)h, hidden,
                        (const float *)W_dkv, (const float *)W_kr, req, pos, n_tok, page_table, batch, max_pages,
                        n_pages, d.page, d.d_c, d.d_r, d.base, (float *)cache, err);
    return cudaGetLastError();
}

}  // namespace mla

// ---------------------------------------------------------------------------------------
// Tensor-core append for the DeepSeek-V2 shape (bf16, d_c = 512, d_rope = 64, hidden a multiple
// of 256 up to 10240).  The projection [n_tok, hidden] x [hidden, 576] is weight-bandwidth bound for a
// decode batch (n_tok = batch * s_q), so the weights must stream through many SMs at once: a
// cluster of 8 CTAs splits the hidden dimension, each CTA multiplies its slice of 16 tokens x
// 32 output columns with mma.sync (its two warp quartets taking alternate 32-wide steps of the
// slice), and rank 0 sums the 16 partial tiles in a fixed order through distributed shared
// memory, then applies RoPE and scatters into the paged cache.  Grid: 18 column tiles x 8 hidden
// slices (144 CTAs, one per SM) per 16-token tile.
// ---------------------------------------------------------------------------------------
#include <cooperative_groups.h>

#include "warp_mma.cuh"

namespace mla {
namespace {

constexpr int AP_SPLIT = 8, AP_COLS = 32, AP_TOK = 16, AP_TILES = 576 / AP_COLS;

__global__ void __cluster_dims__(AP_SPLIT, 1, 1) __launch_bounds__(256)
    append_mma_kernel(const __nv_bfloat16 *__restrict__ h, int hidden, const __nv_bfloat16 *__restrict__ W_dkv,
                      const __nv_bfloat16 *__restrict__ W_kr, const int *__restrict__ req,
                      const int *__restrict__ pos, int n_tok, const int *__restrict__ page_table, int batch,
                      int max_pages, int n_pages, float base, __nv_bfloat16 *__restrict__ cache, int *err) {
    step_allow_next();   // loads and products touch inputs only; the cache stores wait (below)
    namespace cg = cooperative_groups;
    cg::cluster_group cluster = cg::this_cluster();
    constexpr int D_C = 512, D_R = 64, D_ROW = 576;
    extern __shared__ __align__(16) uint8_t asm_raw[];
    const int ks = hidden / AP_SPLIT;                  // hidden slice of this CTA
    const int ld = ks + 8;
    __nv_bfloat16 *Ws = reinterpret_cast<__nv_bfloat16 *>(asm_raw);          // [32 cols][ks]
    __nv_bfloat16 *Hs = Ws + AP_COLS * ld;                                    // [16 tok][ks]
    float *part = reinterpret_cast<float *>(Hs + AP_TOK * ld);                // [2 quartets][16][32]
    const int rank = (int)cluster.block_rank();
    const int ct = blockIdx.x / AP_SPLIT, c0 = ct * AP_COLS, k0 = rank * ks;
    const int t0 = blockIdx.y * AP_TOK;
    const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
    for (int c = tid; c < AP_COLS * ks / 8; c += 256) {
        const int r = c / (ks / 8), k = (c % (ks / 8)) * 8, col = c0 + r;
        const __nv_bfloat16 *src = col < D_C ? W_dkv + (size_t)col * hidden : W_kr + (size_t)(col - D_C) * hidden;
        cp_async16(Ws + r * ld + k, src + k0 + k, true);
    }
    for (int c = tid; c < AP_TOK * ks / 8; c += 256) {
        const int r = c / (ks / 8), k = (c % (ks / 8)) * 8, tok = t0 + r;
        cp_async16(Hs + r * ld + k, h + (size_t)(tok < n_tok ? tok : 0) * hidden + k0 + k, tok < n_tok);
    }
    cp_async_commit();
    cp_async_wait<0>();
    __syncthreads();
    // warp w: tokens 0..15 x columns [8 (w % 4), 8 (w % 4) + 8), 32-wide steps w / 4, w / 4 + 2, ...
    const int wc = warp % 4, wq = warp / 4;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    for (int kk = 32 * wq; kk < ks; kk += 64) {
        uint32_t a0[4], a1[4], b[4];
        ldmatrix_x4(a0[0], a0[1], a0[2], a0[3], Hs + ((lane % 8) + 8 * ((lane / 8) % 2)) * ld + kk + 8 * (lane / 16));
        ldmatrix_x4(a1[0], a1[1], a1[2], a1[3],
                    Hs + ((lane % 8) + 8 * ((lane / 8) % 2)) * ld + kk + 16 + 8 * (lane / 16));
        ldmatrix_x4(b[0], b[1], b[2], b[3], Ws + (8 * wc + (lane % 8)) * ld + kk + 8 * (lane / 8));
        mma_bf16(acc, a0, b[0], b[1]);
        mma_bf16(acc, a1, b[2], b[3]);
    }
    const int gid = lane / 4, t4 = lane % 4;
    float *pq = part + wq * AP_TOK * AP_COLS;
    pq[gid * AP_COLS + 8 * wc + 2 * t4] = acc[0];
    pq[gid * AP_COLS + 8 * wc + 2 * t4 + 1] = acc[1];
    pq[(gid + 8) * AP_COLS + 8 * wc + 2 * t4] = acc[2];
    pq[(gid + 8) * AP_COLS + 8 * wc + 2 * t4 + 1] = acc[3];
    cluster.sync();
    if (rank == 0) {
        step_wait_prev();
        for (int pi = tid; pi < AP_TOK * AP_COLS / 2; pi += 256) {
            const int r = pi / (AP_COLS / 2), cp = pi % (AP_COLS / 2);
            const int n = t0 + r, col = c0 + 2 * cp;
            if (n >= n_tok) continue;
            float x0 = 0.f, x1 = 0.f;
#pragma unroll
            for (int q = 0; q < AP_SPLIT; ++q) {
                const float *rp = cluster.map_shared_rank(part, q);
#pragma unroll
                for (int hq = 0; hq < 2; ++hq) {
                    const float2 x = *reinterpret_cast<const float2 *>(rp + (hq * AP_TOK + r) * AP_COLS + 2 * cp);
                    x0 += x.x;
                    x1 += x.y;
                }
            }
            const int b = req[n], p = pos[n];
            if (b < 0 || b >= batch || p < 0 || p >= max_pages * 64) {
                report(err, MLA_ERR_DEVICE_BOUNDS);
                continue;
            }
            const int pid = page_table[(size_t)b * max_pages + p / 64];
            if (pid < 0 || pid >= n_pages) {
                report(err, MLA_ERR_DEVICE_BOUNDS);
                continue;
            }
            if (col >= D_C) {
                float cs, sn;
                rope_cos_sin(p, (col - D_C) / 2, D_R, base, &cs, &sn);
                const float y0 = x0 * cs - x1 * sn, y1 = x0 * sn + x1 * cs;
                x0 = y0;
                x1 = y1;
            }
            __nv_bfloat16 *dst = cache + ((size_t)pid * 64 + p % 64) * D_ROW + col;
            *reinterpret_cast<uint32_t *>(dst) = pack_bf16(x0, x1);
        }
    }
    cluster.sync();   // partner tiles stay alive until rank 0 has read them
}

}  // namespace

bool append_mma_ok(const Dims &d, int hidden, bool projected) {
    // hidden slices must be whole 32-column MMA steps, and the slice tiles must fit shared memory
    return projected && d.bf16 && d.d_c == 512 && d.d_r == 64 && d.page == 64 && hidden % (32 * AP_SPLIT) == 0 &&
           hidden >= 32 * AP_SPLIT && hidden <= 10240;
}

cudaError_t launch_append_mma(const Dims &d, const void *h, int hidden, const void *W_dkv, const void *W_kr,
                              const int *req, const int *pos, int n_tok, const int *page_table, int batch,
                              int max_pages, int n_pages, void *cache, int *err, cudaStream_t st) {
    const int ks = hidden / AP_SPLIT, ld = ks + 8;
    const size_t smem = sizeof(__nv_bfloat16) * (size_t)(AP_COLS + AP_TOK) * ld + sizeof(float) * 2 * AP_TOK * AP_COLS;
    cudaError_t e = raise_smem_limit((const void *)append_mma_kernel, smem);
    if (e != cudaSuccess) return e;
    dim3 grid(AP_TILES * AP_SPLIT, ceil_div(n_tok, AP_TOK));
    MLA_STEP_LAUNCH(append_mma_kernel, dim3(grid), dim3(256), smem, st, (const __nv_bfloat16 *)h, hidden,
                    (const __nv_bfloat16 *)W_dkv, (const __nv_bfloat16 *)W_kr, req, pos, n_tok, page_table, batch,
                    max_pages, n_pages, d.base, (__nv_bfloat16 *)cache, err);
    return cudaGetLastError();
}

}  // namespace mla
