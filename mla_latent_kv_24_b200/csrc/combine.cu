// Split combine and output up-projection.
//
// Partial results of the chunks of one row (b, j) merge exactly:
//     M = max_i m_i,   O = sum_i e^{m_i - M} O_i / sum_i e^{m_i - M} l_i
// then, on the absorbed path, the head's output leaves latent space through W_UV
// ("MLA and GRPO architecture", "The Mathematics of MLA": v^C = W_UV c; by associativity
// W_UV applies once to the probability-weighted latent):  out = W_UV[w(h)] O.
// On the grouped path O already is the head's d_v-wide output.
//
// One CTA per (head, block of RB rows): the merged rows sit in shared memory and each W_UV
// row is read once per RB rows.
#include <math.h>

#include "kernels.h"

namespace mla {
namespace {

constexpr int RB = 8;

template <typename T>
__global__ void __launch_bounds__(256) combine_kernel(const float *__restrict__ part_o,
                                                      const float *__restrict__ part_ml,
                                                      const int *__restrict__ row_first, int rows, int qpi,
                                                      int H, int DV, const T *__restrict__ W_uv, int hpw,
                                                      int d_v, T *__restrict__ out) {
    extern __shared__ float O[];  // [RB][DV]
    const int h = blockIdx.x;
    const int row0 = blockIdx.y * RB;
    const int nr = min(RB, rows - row0);
    for (int r = 0; r < nr; ++r) {
        const int pr = (row0 + r) / qpi, j = (row0 + r) % qpi;
        const int k0 = row_first[pr], k1 = row_first[pr + 1];
        auto ml = [&](int k, int e) { return part_ml[(((size_t)k * qpi + j) * H + h) * 2 + e]; };
        float M = -INFINITY;
        for (int k = k0; k < k1; ++k) M = fmaxf(M, ml(k, 0));
        float den = 0.f;
        for (int k = k0; k < k1; ++k) {
            const float mk = ml(k, 0);
            if (mk != -INFINITY) den += expf(mk - M) * ml(k, 1);
        }
        const float inv = den > 0.f ? 1.f / den : 0.f;
        for (int c = threadIdx.x; c < DV; c += blockDim.x) {
            float num = 0.f;
            for (int k = k0; k < k1; ++k) {
                const float mk = ml(k, 0);
                if (mk != -INFINITY) num += expf(mk - M) * part_o[(((size_t)k * qpi + j) * H + h) * DV + c];
            }
            O[r * DV + c] = num * inv;
        }
    }
    __syncthreads();
    if (W_uv == nullptr) {
        for (int i = threadIdx.x; i < nr * DV; i += blockDim.x) {
            const int r = i / DV, c = i % DV;
            out[((size_t)(row0 + r) * H + h) * DV + c] = from_f32<T>(O[r * DV + c]);
        }
        return;
    }
    const T *W = W_uv + (size_t)(h / hpw) * d_v * DV;
    for (int v = threadIdx.x; v < d_v; v += blockDim.x) {
        float acc[RB];
#pragma unroll
        for (int r = 0; r < RB; ++r) acc[r] = 0.f;
        const T *wr = W + (size_t)v * DV;
        for (int k = 0; k < DV; ++k) {
            const float wv = to_f32(wr[k]);
#pragma unroll
            for (int r = 0; r < RB; ++r) acc[r] += wv * O[r * DV + k];
        }
        for (int r = 0; r < nr; ++r) out[((size_t)(row0 + r) * H + h) * d_v + v] = from_f32<T>(acc[r]);
    }
}

}  // namespace

cudaError_t launch_combine(const Dims &d, const float *part_o, const float *part_ml, const int *row_first,
                           int rows, int qpi, int DV, const void *W_uv, void *out, cudaStream_t st) {
    dim3 grid(d.H, ceil_div(rows, RB));
    const size_t smem = sizeof(float) * RB * DV;
    if (d.bf16) {
        auto k = combine_kernel<__nv_bfloat16>;
        cudaError_t e = raise_smem_limit((const void *)k, smem);
        if (e != cudaSuccess) return e;
        k<<<grid, 256, smem, st>>>(part_o, part_ml, row_first, rows, qpi, d.H, DV, (const __nv_bfloat16 *)W_uv,
                                   d.hpw, d.d_v, (__nv_bfloat16 *)out);
    } else {
        auto k = combine_kernel<float>;
        cudaError_t e = raise_smem_limit((const void *)k, smem);
        if (e != cudaSuccess) return e;
        k<<<grid, 256, smem, st>>>(part_o, part_ml, row_first, rows, qpi, d.H, DV, (const float *)W_uv, d.hpw, d.d_v,
                                   (float *)out);
    }
    return cudaGetLastError();
}

}  // namespace mla

// ---------------------------------------------------------------------------------------
// Tensor-core combine + W_UV for the DeepSeek-V2 shape (bf16, d_c = 512, d_v = 128).  One CTA
// takes one head and 32 query rows: it merges each row's chunk partials into bf16 latent rows
// in shared memory (the same exact merge as above), then computes out[rows, 128] =
// O[rows, 512] W_UV[w]^T with mma.sync m16n8k16, streaming W_UV[w] in four 128-column slices
// through a double-buffered cp.async ring.  W_UV is read once per head (16.8 MB for H = 128)
// and the fp32 partials once.
// ---------------------------------------------------------------------------------------
#include "warp_mma.cuh"

namespace mla {
namespace {

constexpr int CM = 32, CN = 128, CK = 512, CKC = 128, O_LD = CK + 8, W_LD = CKC + 8;

// OCT: partials in the column-octet layout [k][64][H][8] of the tcgen05 decode (else [k][H][512]).
template <bool OCT>
__global__ void __launch_bounds__(256) combine_mma_kernel(const float *__restrict__ part_o,
                                                          const float *__restrict__ part_ml,
                                                          const int *__restrict__ row_first, int rows, int H,
                                                          const __nv_bfloat16 *__restrict__ W_uv, int hpw,
                                                          __nv_bfloat16 *__restrict__ out) {
    extern __shared__ __align__(16) __nv_bfloat16 csm[];
    __nv_bfloat16 *Os = csm;                       // [64][512 + 8]
    __nv_bfloat16 *Ws = csm + CM * O_LD;           // [2][128 v][128 + 8]
    const int h = blockIdx.x, row0 = blockIdx.y * CM;
    const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
    const __nv_bfloat16 *W = W_uv + (size_t)(h / hpw) * CN * CK;
    auto load_w = [&](int s, int c0) {
        for (int c = tid; c < CN * CKC / 8; c += 256) {   // 2048 chunks of 16 B
            const int v = c / (CKC / 8), k = (c % (CKC / 8)) * 8;
            cp_async16(Ws + (s * CN + v) * W_LD + k, W + (size_t)v * CK + c0 + k, true);
        }
        cp_async_commit();
    };
    load_w(0, 0);
    // Merge the chunk partials of every row of this tile: warp w takes rows w, w + 8, ...; lane
    // l owns latent columns [16 l, 16 l + 16).
    for (int r = warp; r < CM; r += 8) {
        const int row = row0 + r;
        float4 acc4[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) acc4[q] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (row < rows) {
            const int k0 = row_first[row], k1 = row_first[row + 1];
            float M = -INFINITY;
            for (int k = k0 + lane; k < k1; k += 32) M = fmaxf(M, part_ml[((size_t)k * H + h) * 2]);
#pragma unroll
            for (int o = 16; o; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
            float den = 0.f;
            // Partials are merged in batches of KB whose loads are all issued before any is used,
            // so a row with many chunks pays the memory latency once per batch, not per chunk.
            constexpr int KB = 8;
            for (int kb = k0; kb < k1; kb += KB) {
                float4 v[KB][4];
                float wk[KB];
#pragma unroll
                for (int u = 0; u < KB; ++u) {
                    const int k = kb + u;
                    wk[u] = 0.f;
#pragma unroll
                    for (int q = 0; q < 4; ++q) v[u][q] = make_float4(0.f, 0.f, 0.f, 0.f);
                    if (k < k1) {
                        const float2 ml = *reinterpret_cast<const float2 *>(part_ml + ((size_t)k * H + h) * 2);
                        wk[u] = ml.x == -INFINITY ? 0.f : expf(ml.x - M);
                        den += wk[u] * ml.y;
                        if (OCT) {
                            const float4 *po0 = reinterpret_cast<const float4 *>(part_o + (((size_t)k * 64 + 2 * lane) * H + h) * 8);
                            const float4 *po1 = reinterpret_cast<const float4 *>(part_o + (((size_t)k * 64 + 2 * lane + 1) * H + h) * 8);
                            v[u][0] = po0[0];
                            v[u][1] = po0[1];
                            v[u][2] = po1[0];
                            v[u][3] = po1[1];
                        } else {
                            const float4 *po = reinterpret_cast<const float4 *>(part_o + ((size_t)k * H + h) * CK + 16 * lane);
#pragma unroll
                            for (int q = 0; q < 4; ++q) v[u][q] = po[q];
                        }
                    }
                }
#pragma unroll
                for (int u = 0; u < KB; ++u)
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        acc4[q].x += wk[u] * v[u][q].x;
                        acc4[q].y += wk[u] * v[u][q].y;
                        acc4[q].z += wk[u] * v[u][q].z;
                        acc4[q].w += wk[u] * v[u][q].w;
                    }
            }
            const float inv = den > 0.f ? 1.f / den : 0.f;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                acc4[q].x *= inv;
                acc4[q].y *= inv;
                acc4[q].z *= inv;
                acc4[q].w *= inv;
            }
        }
        uint4 pk0 = make_uint4(pack_bf16(acc4[0].x, acc4[0].y), pack_bf16(acc4[0].z, acc4[0].w),
                               pack_bf16(acc4[1].x, acc4[1].y), pack_bf16(acc4[1].z, acc4[1].w));
        uint4 pk1 = make_uint4(pack_bf16(acc4[2].x, acc4[2].y), pack_bf16(acc4[2].z, acc4[2].w),
                               pack_bf16(acc4[3].x, acc4[3].y), pack_bf16(acc4[3].z, acc4[3].w));
        *reinterpret_cast<uint4 *>(Os + r * O_LD + 16 * lane) = pk0;
        *reinterpret_cast<uint4 *>(Os + r * O_LD + 16 * lane + 8) = pk1;
    }
    const int wm = warp % 2, wn = warp / 2;   // warp tile 16 rows x 32 columns
    float acc[4][4];
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[j][e] = 0.f;
    for (int kc = 0; kc < CK / CKC; ++kc) {
        if (kc + 1 < CK / CKC) {
            load_w((kc + 1) & 1, (kc + 1) * CKC);
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();
        const __nv_bfloat16 *Wt = Ws + (kc & 1) * CN * W_LD;
#pragma unroll
        for (int kk = 0; kk < CKC; kk += 16) {
            uint32_t a[4];
            ldmatrix_x4(a[0], a[1], a[2], a[3],
                        Os + (wm * 16 + (lane % 8) + 8 * ((lane / 8) % 2)) * O_LD + kc * CKC + kk + 8 * (lane / 16));
#pragma unroll
            for (int j = 0; j < 4; j += 2) {
                uint32_t b0, b1, b2, b3;
                ldmatrix_x4(b0, b1, b2, b3,
                            Wt + (wn * 32 + j * 8 + (lane % 8) + 8 * (lane / 16)) * W_LD + kk + 8 * ((lane / 8) % 2));
                mma_bf16(acc[j], a, b0, b1);
                mma_bf16(acc[j + 1], a, b2, b3);
            }
        }
        __syncthreads();   // the next load overwrites this slice's buffer
    }
    const int gid = lane / 4, t4 = lane % 4;
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {
        const int row = row0 + wm * 16 + gid + 8 * hr;
        if (row >= rows) continue;
        __nv_bfloat16 *dst = out + ((size_t)row * H + h) * CN + wn * 32;
#pragma unroll
        for (int j = 0; j < 4; ++j)
            *reinterpret_cast<uint32_t *>(dst + j * 8 + 2 * t4) = pack_bf16(acc[j][2 * hr], acc[j][2 * hr + 1]);
    }
}

}  // namespace

bool combine_mma_ok(const Dims &d, int DV, bool project) {
    return project && d.bf16 && DV == CK && d.d_v == CN;
}

cudaError_t launch_combine_mma(const Dims &d, const float *part_o, const float *part_ml, const int *row_first,
                               int rows, bool oct_layout, const void *W_uv, void *out, cudaStream_t st) {
    const size_t smem = sizeof(__nv_bfloat16) * ((size_t)CM * O_LD + 2 * (size_t)CN * W_LD);
    dim3 grid(d.H, ceil_div(rows, CM));
    auto k = oct_layout ? combine_mma_kernel<true> : combine_mma_kernel<false>;
    cudaError_t e = raise_smem_limit((const void *)k, smem);
    if (e != cudaSuccess) return e;
    k<<<grid, 256, smem, st>>>(part_o, part_ml, row_first, rows, d.H, (const __nv_bfloat16 *)W_uv, d.hpw,
                               (__nv_bfloat16 *)out);
    return cudaGetLastError();
}

}  // namespace mla
