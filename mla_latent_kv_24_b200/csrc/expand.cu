// GQA-path cache expansion ("GQLA: Group-Query Latent Attention ..." abstract: a GQA path
// with a per-group expanded cache; AI Radio episode: per-group K and V plus the shared RoPE
// key, which stays in the latent cache):
//     K_g,t = W_UK[g] c_t   (d_nope),    V_g,t = W_UV[g] c_t   (d_v)
// written as expanded[page][g][row] = [K_g | V_g].
//
// Tensor-core kernel (bf16, d_nope = d_v = 128, d_c a multiple of 64): one CTA computes a
// 128-token x 128-output tile (the K or the V half of one group) over d_c, streaming 64-wide
// slices of the latent rows and of the weight rows through a 3-stage cp.async ring into
// padded shared memory, with mma.sync m16n8k16 and fp32 accumulators.  A CUDA-core kernel
// covers every other shape.
//
// The rows to expand are either every row of a list of pages (a prefill, or a rebuild) or the
// rows of single tokens given as (request, position) through the page table, which is how a
// decode step expands exactly what the cache append wrote.
#include "kernels.h"
#include "warp_mma.cuh"

namespace mla {
namespace {

constexpr int BM = 128, BN = 128, BK = 64, LDS = BK + 8, STAGES = 3;

// Row slot i -> (page id, row in page) of the latent / expanded caches.
struct RowMap {
    const int *page_ids;          // page mode: [n] page ids, or null for pages 0..n-1
    const int *req, *pos;         // token mode (req != null): [n] request and position
    const int *page_table;        // token mode: [batch, max_pages]
    int n, batch, max_pages;
    __host__ __device__ long long slots(int page) const { return req ? (long long)n : (long long)n * page; }
};

// False when slot i is past the end or names a row outside the caches (reported as a bounds error).
__device__ __forceinline__ bool map_row(const RowMap &m, long long i, int page, int n_pages, int *pid, int *r,
                                        int *err) {
    if (i >= m.slots(page)) return false;
    int p;
    if (m.req) {
        const int b = m.req[i], t = m.pos[i];
        if (b < 0 || b >= m.batch || t < 0 || t >= m.max_pages * page) {
            report(err, MLA_ERR_DEVICE_BOUNDS);
            return false;
        }
        p = m.page_table[(size_t)b * m.max_pages + t / page];
        *r = t % page;
    } else {
        const long long e = i / page;
        p = m.page_ids ? m.page_ids[e] : (int)e;
        *r = (int)(i % page);
    }
    if (p < 0 || p >= n_pages) {
        report(err, MLA_ERR_DEVICE_BOUNDS);
        return false;
    }
    *pid = p;
    return true;
}

__global__ void __launch_bounds__(256) expand_mma_kernel(const __nv_bfloat16 *__restrict__ W_uk,
                                                         const __nv_bfloat16 *__restrict__ W_uv,
                                                         const __nv_bfloat16 *__restrict__ latent, RowMap map,
                                                         int n_pages, int page, int d_c, int d_r, int G,
                                                         __nv_bfloat16 *__restrict__ out, int *err) {
    step_begin();
    extern __shared__ __align__(16) __nv_bfloat16 sm[];
    __nv_bfloat16 *As = sm;                          // [STAGES][BM][LDS]
    __nv_bfloat16 *Bs = sm + STAGES * BM * LDS;      // [STAGES][BN][LDS]
    __shared__ long long row_off[BM];                // latent row offset (elements), -1 = skip
    __shared__ long long out_off[BM];

    const int g = blockIdx.y, half = blockIdx.z;
    const int d_row = d_c + d_r;
    const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
    const __nv_bfloat16 *W = (half == 0 ? W_uk : W_uv) + (size_t)g * 128 * d_c;

    if (tid < BM) {
        int pid, r;
        long long ro = -1, oo = -1;
        if (map_row(map, (long long)blockIdx.x * BM + tid, page, n_pages, &pid, &r, err)) {
            ro = ((long long)pid * page + r) * d_row;
            oo = (((long long)pid * G + g) * page + r) * 256 + half * 128;
        }
        row_off[tid] = ro;
        out_off[tid] = oo;
    }
    __syncthreads();

    auto load_stage = [&](int s, int k0) {
        // 128 rows x 64 cols = 1024 16-byte chunks per operand, 4 per thread each.
        for (int c = tid; c < BM * BK / 8; c += 256) {
            const int r = c / (BK / 8), kc = (c % (BK / 8)) * 8;
            const long long ro = row_off[r];
            cp_async16(As + (s * BM + r) * LDS + kc, latent + (ro < 0 ? 0 : ro) + k0 + kc, ro >= 0);
            cp_async16(Bs + (s * BN + r) * LDS + kc, W + (size_t)r * d_c + k0 + kc, true);
        }
    };

    const int wm = warp / 4, wn = warp % 4;  // warp tile: 64 rows x 32 cols
    float acc[4][4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int k = 0; k < 4; ++k) acc[i][j][k] = 0.f;

    const int KT = d_c / BK;
#pragma unroll
    for (int s = 0; s < STAGES - 1; ++s) {
        if (s < KT) load_stage(s, s * BK);
        cp_async_commit();
    }
    for (int kt = 0; kt < KT; ++kt) {
        cp_async_wait<STAGES - 2>();
        __syncthreads();
        const int nk = kt + STAGES - 1;
        if (nk < KT) load_stage(nk % STAGES, nk * BK);
        cp_async_commit();
        const __nv_bfloat16 *A = As + (kt % STAGES) * BM * LDS;
        const __nv_bfloat16 *Bt = Bs + (kt % STAGES) * BN * LDS;
#pragma unroll
        for (int kk = 0; kk < BK; kk += 16) {
            uint32_t a[4][4], b[4][2];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int r = wm * 64 + i * 16 + (lane % 8) + 8 * ((lane / 8) % 2);
                const int c = kk + 8 * (lane / 16);
                ldmatrix_x4(a[i][0], a[i][1], a[i][2], a[i][3], A + r * LDS + c);
            }
#pragma unroll
            for (int j = 0; j < 4; j += 2) {
                const int r = wn * 32 + j * 8 + (lane % 8) + 8 * (lane / 16);
                const int c = kk + 8 * ((lane / 8) % 2);
                ldmatrix_x4(b[j][0], b[j][1], b[j + 1][0], b[j + 1][1], Bt + r * LDS + c);
            }
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) mma_bf16(acc[i][j], a[i], b[j][0], b[j][1]);
        }
    }
    cp_async_wait<0>();

    const int gid = lane / 4, t4 = lane % 4;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
#pragma unroll
        for (int hr = 0; hr < 2; ++hr) {
            const int r = wm * 64 + i * 16 + gid + 8 * hr;
            const long long oo = out_off[r];
            if (oo < 0) continue;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int c = wn * 32 + j * 8 + 2 * t4;
                *reinterpret_cast<uint32_t *>(out + oo + c) = pack_bf16(acc[i][j][2 * hr], acc[i][j][2 * hr + 1]);
            }
        }
    }
}

// CUDA-core expansion for other shapes / fp32: one thread per output element.
template <typename T>
__global__ void expand_simt_kernel(const T *__restrict__ W_uk, const T *__restrict__ W_uv,
                                   const T *__restrict__ latent, RowMap map, int n_pages, int page, int d_c,
                                   int d_r, int d_n, int d_v, int G, T *__restrict__ out, int *err) {
    step_begin();
    const int w_out = d_n + d_v;
    const long long n = map.slots(page) * G * w_out;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n;
         i += (long long)gridDim.x * blockDim.x) {
        const int o = (int)(i % w_out);
        const long long rest = i / w_out;
        const int g = (int)(rest % G);
        int pid, r;
        if (!map_row(map, rest / G, page, n_pages, &pid, &r, err)) continue;
        const T *c = latent + ((size_t)pid * page + r) * (d_c + d_r);
        const T *w = o < d_n ? W_uk + ((size_t)g * d_n + o) * d_c : W_uv + ((size_t)g * d_v + (o - d_n)) * d_c;
        float acc = 0.f;
        for (int k = 0; k < d_c; ++k) acc += to_f32(w[k]) * to_f32(c[k]);
        out[(((size_t)pid * G + g) * page + r) * w_out + o] = from_f32<T>(acc);
    }
}

}  // namespace

static cudaError_t launch_expand_rows(const Dims &d, const void *W_uk, const void *W_uv, const void *latent,
                                      const RowMap &map, int n_pages, void *expanded, int *err, cudaStream_t st) {
    const int G = d.n_groups();
    const long long slots = map.slots(d.page);
    if (slots == 0) return cudaSuccess;
    if (d.bf16 && d.d_n == 128 && d.d_v == 128 && d.d_c % BK == 0) {
        const size_t smem = sizeof(__nv_bfloat16) * STAGES * (BM + BN) * LDS;
        cudaError_t e = raise_smem_limit((const void *)expand_mma_kernel, smem);
        if (e != cudaSuccess) return e;
        dim3 grid((unsigned)((slots + BM - 1) / BM), G, 2);
        MLA_STEP_LAUNCH(expand_mma_kernel, dim3(grid), dim3(256), smem, st, (const __nv_bfloat16 *)W_uk,
                        (const __nv_bfloat16 *)W_uv, (const __nv_bfloat16 *)latent, map, n_pages, d.page, d.d_c,
                        d.d_r, G, (__nv_bfloat16 *)expanded, err);
        return cudaGetLastError();
    }
    const long long n = slots * G * (d.d_n + d.d_v);
    const int blocks = (int)std::min<long long>((n + 255) / 256, 65535);
    if (d.bf16)
        MLA_STEP_LAUNCH(expand_simt_kernel<__nv_bfloat16>, dim3(blocks), dim3(256), 0, st,
                        (const __nv_bfloat16 *)W_uk, (const __nv_bfloat16 *)W_uv, (const __nv_bfloat16 *)latent, map,
                        n_pages, d.page, d.d_c, d.d_r, d.d_n, d.d_v, G, (__nv_bfloat16 *)expanded, err);
    else
        MLA_STEP_LAUNCH(expand_simt_kernel<float>, dim3(blocks), dim3(256), 0, st, (const float *)W_uk,
                        (const float *)W_uv, (const float *)latent, map, n_pages, d.page, d.d_c, d.d_r, d.d_n, d.d_v,
                        G, (float *)expanded, err);
    return cudaGetLastError();
}

cudaError_t launch_expand(const Dims &d, const void *W_uk, const void *W_uv, const void *latent,
                          const int *page_ids, int n_ids, int n_pages, void *expanded, int *err,
                          cudaStream_t st) {
    const RowMap map{page_ids, nullptr, nullptr, nullptr, n_ids, 0, 0};
    return launch_expand_rows(d, W_uk, W_uv, latent, map, n_pages, expanded, err, st);
}

cudaError_t launch_expand_tokens(const Dims &d, const void *W_uk, const void *W_uv, const void *latent,
                                 const int *req, const int *pos, int n_tok, const int *page_table, int batch,
                                 int max_pages, int n_pages, void *expanded, int *err, cudaStream_t st) {
    const RowMap map{nullptr, req, pos, page_table, n_tok, batch, max_pages};
    return launch_expand_rows(d, W_uk, W_uv, latent, map, n_pages, expanded, err, st);
}

}  // namespace mla
