// General CUDA-core split flash decode, for dims/dtypes the tensor-core kernels are not built
// for (the fp32 workload, small test shapes).
//
// Absorbed mode (MQA-absorb path: the latent row is the key shared by all heads, its first
// d_c columns the shared value):   s_t = scale * q_abs[h] . [c_t | k^R_t],   V_t = c_t.
// Grouped mode (GQA path over the per-group expanded cache): s_t = scale * [q_nope | q_rope'] .
// [K_g,t | k^R_t],  V_t = V_g,t.
// Each CTA takes one work item (row, token range) and HB heads (of one group in grouped mode);
// tiles of 32 tokens (one per lane) are staged in shared memory as fp32, every warp runs an
// online softmax for its heads with warp-shuffle max/sum, and writes the unnormalised partial
// output with its running max m and sum l for the combine kernel.
#include <math.h>

#include "kernels.h"

namespace mla {
namespace {

constexpr int TT = 32;        // tokens per tile (one per lane)
constexpr int WARPS = 8;
constexpr int MAX_HB = 16;    // heads per CTA
constexpr int HPW = MAX_HB / WARPS;
constexpr int MAX_VL = 16;    // value columns per lane (DV <= 512)

struct P {
    const void *q, *latent, *expanded;
    const int *page_table;
    Plan plan;
    float *part_o, *part_ml;
    int *err;
    int H, hpw, HB, DK, DV, d_c, d_r, d_n, d_v, page, G, max_pages, n_pages, s_q;
    float scale;
};

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

template <typename T, int MODE>
__global__ void __launch_bounds__(WARPS * 32) decode_simt_kernel(P p) {
    step_begin();
    extern __shared__ float smem[];
    const int KS = p.DK + 1, VS = p.DV + 1;
    float *qs = smem;                         // [HB][DK]
    float *ks = qs + MAX_HB * p.DK;           // [TT][DK + 1]
    float *vs = ks + TT * KS;                 // [TT][DV + 1] (grouped mode)
    __shared__ int tok_ok[TT];

    const WorkItem it = p.plan.items[blockIdx.x];
    const int h0 = blockIdx.y * p.HB;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int d_row = p.d_c + p.d_r;
    const int b = it.row / p.s_q;
    const int g = MODE == 1 ? h0 / p.hpw : 0;
    const T *q = (const T *)p.q;
    const T *lat = (const T *)p.latent;
    const T *exq = (const T *)p.expanded;

    const int nh = min(p.HB, p.H - h0);  // heads of this CTA
    for (int i = threadIdx.x; i < nh * p.DK; i += blockDim.x) {
        const int hh = i / p.DK, k = i % p.DK;
        qs[i] = to_f32(q[((size_t)it.row * p.H + h0 + hh) * p.DK + k]);
    }

    float m[HPW], l[HPW], acc[HPW][MAX_VL];
#pragma unroll
    for (int i = 0; i < HPW; ++i) {
        m[i] = -INFINITY;
        l[i] = 0.f;
#pragma unroll
        for (int v = 0; v < MAX_VL; ++v) acc[i][v] = 0.f;
    }
    const int nvl = (p.DV + 31) / 32;

    for (int tb = it.t0; tb < it.t1; tb += TT) {
        __syncthreads();
        if (threadIdx.x < TT) {
            const int tok = tb + threadIdx.x;
            int ok = tok < it.t1;
            if (ok) {
                const int pid = p.page_table[(size_t)b * p.max_pages + tok / p.page];
                if (pid < 0 || pid >= p.n_pages) {
                    report(p.err, MLA_ERR_DEVICE_BOUNDS);
                    ok = 0;
                } else {
                    ok = pid + 1;  // page id + 1
                }
            }
            tok_ok[threadIdx.x] = ok;
        }
        __syncthreads();
        for (int i = threadIdx.x; i < TT * p.DK; i += blockDim.x) {
            const int t = i / p.DK, k = i % p.DK;
            const int okp = tok_ok[t];
            float v = 0.f;
            if (okp) {
                const size_t pid = (size_t)(okp - 1), r = (size_t)((tb + t) % p.page);
                if (MODE == 0) {
                    v = to_f32(lat[(pid * p.page + r) * d_row + k]);
                } else {
                    v = k < p.d_n ? to_f32(exq[((pid * p.G + g) * p.page + r) * (p.d_n + p.d_v) + k])
                                  : to_f32(lat[(pid * p.page + r) * d_row + p.d_c + (k - p.d_n)]);
                }
            }
            ks[t * KS + k] = v;
        }
        if (MODE == 1) {
            for (int i = threadIdx.x; i < TT * p.DV; i += blockDim.x) {
                const int t = i / p.DV, c = i % p.DV;
                const int okp = tok_ok[t];
                float v = 0.f;
                if (okp) {
                    const size_t pid = (size_t)(okp - 1), r = (size_t)((tb + t) % p.page);
                    v = to_f32(exq[((pid * p.G + g) * p.page + r) * (p.d_n + p.d_v) + p.d_n + c]);
                }
                vs[t * VS + c] = v;
            }
        }
        __syncthreads();
        const float *V = MODE == 0 ? ks : vs;
        const int VST = MODE == 0 ? KS : VS;
        const bool valid = tok_ok[lane] != 0;
#pragma unroll
        for (int i = 0; i < HPW; ++i) {
            const int hh = warp + WARPS * i;
            if (hh >= nh) break;
            const float *qh = qs + hh * p.DK;
            const float *kt = ks + lane * KS;
            float s = 0.f;
            for (int k = 0; k < p.DK; ++k) s += qh[k] * kt[k];
            s = valid ? s * p.scale : -INFINITY;
            const float mnew = fmaxf(m[i], warp_max(s));
            float alpha = 1.f, e = 0.f;
            if (mnew != -INFINITY) {
                alpha = expf(m[i] - mnew);
                e = valid ? expf(s - mnew) : 0.f;
            }
            l[i] = l[i] * alpha + warp_sum(e);
            m[i] = mnew;
#pragma unroll
            for (int v = 0; v < MAX_VL; ++v) acc[i][v] *= alpha;
            for (int t = 0; t < TT; ++t) {
                const float pt = __shfl_sync(0xffffffffu, e, t);
                const float *vr = V + t * VST;
#pragma unroll
                for (int v = 0; v < MAX_VL; ++v)
                    if (v < nvl && lane + 32 * v < p.DV) acc[i][v] += pt * vr[lane + 32 * v];
            }
        }
    }
#pragma unroll
    for (int i = 0; i < HPW; ++i) {
        const int hh = warp + WARPS * i;
        if (hh >= nh) break;
        const size_t base = (size_t)blockIdx.x * p.H + h0 + hh;
#pragma unroll
        for (int v = 0; v < MAX_VL; ++v)
            if (v < nvl && lane + 32 * v < p.DV) p.part_o[base * p.DV + lane + 32 * v] = acc[i][v];
        if (lane == 0) {
            p.part_ml[base * 2] = m[i];
            p.part_ml[base * 2 + 1] = l[i];
        }
    }
}

template <typename T, int MODE>
cudaError_t launch_t(const P &p, dim3 grid, size_t smem, cudaStream_t st) {
    auto k = decode_simt_kernel<T, MODE>;
    cudaError_t e = raise_smem_limit((const void *)k, smem);
    if (e != cudaSuccess) return e;
    MLA_STEP_LAUNCH(k, dim3(grid), dim3(WARPS * 32), smem, st, p);
    return cudaGetLastError();
}

}  // namespace

int simt_heads_per_block(const Dims &d, int mode) {
    if (mode == 0) return d.H < MAX_HB ? d.H : MAX_HB;
    return d.hpw < MAX_HB ? d.hpw : MAX_HB;
}

cudaError_t launch_decode_simt(const Dims &d, const SimtDecodeArgs &a, cudaStream_t st) {
    P p;
    p.q = a.q;
    p.latent = a.latent;
    p.expanded = a.expanded;
    p.page_table = a.page_table;
    p.plan = a.plan;
    p.part_o = a.part_o;
    p.part_ml = a.part_ml;
    p.err = a.err;
    p.H = d.H;
    p.hpw = d.hpw;
    p.HB = simt_heads_per_block(d, a.mode);
    p.DK = a.mode == 0 ? d.d_c + d.d_r : d.d_n + d.d_r;
    p.DV = a.mode == 0 ? d.d_c : d.d_v;
    p.d_c = d.d_c;
    p.d_r = d.d_r;
    p.d_n = d.d_n;
    p.d_v = d.d_v;
    p.page = d.page;
    p.G = d.n_groups();
    p.max_pages = a.max_pages;
    p.n_pages = a.n_pages;
    p.s_q = a.s_q;
    p.scale = d.scale;
    if (a.plan.n_work == 0) return cudaSuccess;
    dim3 grid(a.plan.n_work, ceil_div(d.H, p.HB));
    size_t smem = sizeof(float) * ((size_t)MAX_HB * p.DK + (size_t)TT * (p.DK + 1) +
                                   (a.mode == 1 ? (size_t)TT * (p.DV + 1) : 0));
    if (d.bf16)
        return a.mode == 0 ? launch_t<__nv_bfloat16, 0>(p, grid, smem, st) : launch_t<__nv_bfloat16, 1>(p, grid, smem, st);
    return a.mode == 0 ? launch_t<float, 0>(p, grid, smem, st) : launch_t<float, 1>(p, grid, smem, st);
}

}  // namespace mla
