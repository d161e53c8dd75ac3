// Split combine and output up-projection.
//
// Partial results of the chunks of one row (b, j) merge exactly:
//     M = max_i m_i,   O = sum_i e^{m_i - M} O_i / sum_i e^{m_i - M} l_i
// then, on the absorbed path, the head's output leaves latent space through W_UV
// ("MLA and GRPO architecture", "The Mathematics of MLA": v^C = W_UV c; by associativity
// W_UV applies once to the probability-weighted latent):  out = W_UV[w(h)] O.
// On the grouped path O already is the head's d_v-wide output.
//
// Without projection, one warp merges one (row, head); with it, one CTA takes a head and a
// block of RB rows, the merged rows sit in shared memory and each W_UV row is read once per RB
// rows.  The bf16 DeepSeek-V2 shape takes the tensor-core kernel at the end of this file.
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
    step_begin();
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

// Merge without projection (grouped path, prefill): one warp per (row, head), consecutive warps
// taking consecutive heads so a CTA reads contiguous partials; each lane owns 4 columns per
// 128-column pass.  The chunk weights e^{m_i - M} are formed lane-parallel, the denominator
// is summed by a fixed shuffle tree, and the partial loads are issued KB at a time.
template <typename T>
__global__ void __launch_bounds__(256) combine_rows_kernel(const float *__restrict__ part_o,
                                                           const float *__restrict__ part_ml,
                                                           const int *__restrict__ row_first, int rows, int qpi,
                                                           int H, int DV, T *__restrict__ out) {
    step_begin();
    const int lane = threadIdx.x % 32;
    const long long wid = (long long)blockIdx.x * 8 + threadIdx.x / 32;
    if (wid >= (long long)rows * H) return;
    const int row = (int)(wid / H), h = (int)(wid % H);
    const int pr = row / qpi, j = row % qpi;
    const int k0 = row_first[pr], k1 = row_first[pr + 1];
    auto idx = [&](int k) { return ((size_t)k * qpi + j) * H + h; };
    float M = -INFINITY;
    for (int k = k0 + lane; k < k1; k += 32) M = fmaxf(M, part_ml[idx(k) * 2]);
#pragma unroll
    for (int o = 16; o; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    float den = 0.f;
    for (int k = k0 + lane; k < k1; k += 32) {
        const float mk = part_ml[idx(k) * 2];
        if (mk != -INFINITY) den += expf(mk - M) * part_ml[idx(k) * 2 + 1];
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
    const float inv = den > 0.f ? 1.f / den : 0.f;
    for (int c = 4 * lane; c < DV; c += 128) {
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        constexpr int KB = 8;
        for (int kb = k0; kb < k1; kb += KB) {
            float4 v[KB];
            float mk[KB];
#pragma unroll
            for (int u = 0; u < KB; ++u) {
                v[u] = make_float4(0.f, 0.f, 0.f, 0.f);
                mk[u] = -INFINITY;
                if (kb + u < k1) {
                    mk[u] = part_ml[idx(kb + u) * 2];
                    v[u] = *reinterpret_cast<const float4 *>(part_o + idx(kb + u) * DV + c);
                }
            }
#pragma unroll
            for (int u = 0; u < KB; ++u) {
                const float wk = mk[u] == -INFINITY ? 0.f : expf(mk[u] - M);
                acc.x += wk * v[u].x;
                acc.y += wk * v[u].y;
                acc.z += wk * v[u].z;
                acc.w += wk * v[u].w;
            }
        }
        T *dst = out + ((size_t)row * H + h) * DV + c;
        dst[0] = from_f32<T>(acc.x * inv);
        dst[1] = from_f32<T>(acc.y * inv);
        dst[2] = from_f32<T>(acc.z * inv);
        dst[3] = from_f32<T>(acc.w * inv);
    }
}

}  // namespace

cudaError_t launch_combine(const Dims &d, const float *part_o, const float *part_ml, const int *row_first,
                           int rows, int qpi, int DV, const void *W_uv, void *out, cudaStream_t st) {
    if (W_uv == nullptr && DV % 4 == 0) {
        const long long warps = (long long)rows * d.H;
        if (warps == 0) return cudaSuccess;
        const unsigned blocks = (unsigned)((warps + 7) / 8);
        if (d.bf16)
            MLA_STEP_LAUNCH(combine_rows_kernel<__nv_bfloat16>, dim3(blocks), dim3(256), 0, st, part_o, part_ml,
                            row_first, rows, qpi, d.H, DV, (__nv_bfloat16 *)out);
        else
            MLA_STEP_LAUNCH(combine_rows_kernel<float>, dim3(blocks), dim3(256), 0, st, part_o, part_ml, row_first,
                            rows, qpi, d.H, DV, (float *)out);
        return cudaGetLastError();
    }
    dim3 grid(d.H, ceil_div(rows, RB));
    const size_t smem = sizeof(float) * RB * DV;
    if (d.bf16) {
        auto k = combine_kernel<__nv_bfloat16>;
        cudaError_t e = raise_smem_limit((const void *)k, smem);
        if (e != cudaSuccess) return e;
        MLA_STEP_LAUNCH(k, dim3(grid), dim3(256), smem, st, part_o, part_ml, row_first, rows, qpi, d.H, DV,
                        (const __nv_bfloat16 *)W_uv, d.hpw, d.d_v, (__nv_bfloat16 *)out);
    } else {
        auto k = combine_kernel<float>;
        cudaError_t e = raise_smem_limit((const void *)k, smem);
        if (e != cudaSuccess) return e;
        MLA_STEP_LAUNCH(k, dim3(grid), dim3(256), smem, st, part_o, part_ml, row_first, rows, qpi, d.H, DV,
                        (const float *)W_uv, d.hpw, d.d_v, (float *)out);
    }
    return cudaGetLastError();
}

}  // namespace mla

// ---------------------------------------------------------------------------------------
// Tensor-core combine + W_UV for the DeepSeek-V2 shape (bf16, d_c = 512, d_v = 128).
//
// A decode batch has few rows (batch x s_q) and many chunks per row, so the work of one head is
// spread over a cluster of four CTAs, one per 128-column slice of the latent: CTA s merges the
// chunk partials of its columns into bf16 latent rows in shared memory (the same exact merge as
// above), multiplies them by its slice of W_UV[w] (out_s[rows, 128] = O[:, slice] W_UV[w][:, slice]^T
// with mma.sync m16n8k16), and the four fp32 products are summed in a fixed order through
// distributed shared memory, each CTA adding and storing 32 of the 128 output columns.  All of a
// CTA's loads (its 32 KB of W_UV and its partials) are issued up front, and four times as many
// SMs pull them as with one CTA per head.  W_UV is read once per head, the partials once.
// ---------------------------------------------------------------------------------------
#include <cooperative_groups.h>

#include "warp_mma.cuh"

namespace mla {
namespace {

constexpr int CM = 32, CN = 128, CK = 512;                // rows per tile, d_v, d_c
constexpr int XS = 4, XC = CK / XS, X_LD = XC + 8;        // cluster size, columns per CTA, smem row

// OCT: partials in the column-octet layout [k][64][H][8] of the tcgen05 decode (else [k][H][512]).
template <bool OCT>
__global__ void __cluster_dims__(XS, 1, 1) __launch_bounds__(256, 4)
    combine_split_kernel(const float *__restrict__ part_o, const float *__restrict__ part_ml,
                         const int *__restrict__ row_first, const RowStarts rs, int rows, int H,
                         const __nv_bfloat16 *__restrict__ W_uv, int hpw, __nv_bfloat16 *__restrict__ out) {
    step_allow_next();   // the W_UV slice (an input) streams in while the decode finishes
    namespace cg = cooperative_groups;
    cg::cluster_group cluster = cg::this_cluster();
    extern __shared__ __align__(16) uint8_t xsm[];
    __nv_bfloat16 *Ws = reinterpret_cast<__nv_bfloat16 *>(xsm);   // [128 v][128 c + 8]
    __nv_bfloat16 *Os = Ws + CN * X_LD;                               // [32 rows][128 c + 8]
    float *Red = reinterpret_cast<float *>(xsm);                     // [32][128], over Ws after the MMA
    const int s = (int)cluster.block_rank(), c0 = s * XC;
    const int h = blockIdx.y, row0 = blockIdx.z * CM, nr = min(CM, rows - row0);
    const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
    const __nv_bfloat16 *W = W_uv + (size_t)(h / hpw) * CN * CK;
    for (int c = tid; c < CN * XC / 8; c += 256) {   // 2048 chunks of 16 B
        const int v = c / (XC / 8), k = (c % (XC / 8)) * 8;
        cp_async16(Ws + v * X_LD + k, W + (size_t)v * CK + c0 + k, true);
    }
    cp_async_commit();
    step_wait_prev();   // partials and row starts come from the decode
    // Merge: four rows per pass, two warps per row, each lane two adjacent columns of the slice.
    for (int r = warp / 2; r < CM; r += 4) {
        const int col = 64 * (warp % 2) + 2 * lane;              // column inside the slice
        float2 acc = make_float2(0.f, 0.f);
        if (r < nr) {
            const int row = row0 + r;
            const int k0 = rs.n ? rs.v[row] : row_first[row], k1 = rs.n ? rs.v[row + 1] : row_first[row + 1];
            // One batch of up to KB chunks per memory round trip: lane u fetches chunk kb + u's
            // (m, l), every lane its two columns of each chunk, all before any is used; the
            // running max, sum and accumulator are rescaled between batches (exact).
            constexpr int KB = 12;   // the largest batch that fits 64 registers (4 CTAs per SM)
            float M = -INFINITY, den = 0.f;
            for (int kb = k0; kb < k1; kb += KB) {
                const int n = min(KB, k1 - kb);
                float2 ml = make_float2(-INFINITY, 0.f);
                if (lane < n) ml = *reinterpret_cast<const float2 *>(part_ml + ((size_t)(kb + lane) * H + h) * 2);
                float2 v[KB];
#pragma unroll
                for (int u = 0; u < KB; ++u) {
                    v[u] = make_float2(0.f, 0.f);
                    if (u < n) {
                        const int k = kb + u, c = c0 + col;
                        const size_t off = OCT ? (((size_t)k * 64 + c / 8) * H + h) * 8 + c % 8
                                               : ((size_t)k * H + h) * CK + c;
                        v[u] = *reinterpret_cast<const float2 *>(part_o + off);
                    }
                }
                float mb = ml.x;
#pragma unroll
                for (int o = 16; o; o >>= 1) mb = fmaxf(mb, __shfl_xor_sync(0xffffffffu, mb, o));
                const float Mn = fmaxf(M, mb);
                if (Mn == -INFINITY) continue;   // every chunk so far is empty
                const float keep = M == -INFINITY ? 0.f : expf(M - Mn);
                acc.x *= keep;
                acc.y *= keep;
                den *= keep;
                const float wl = ml.x == -INFINITY ? 0.f : expf(ml.x - Mn);   // weight of chunk kb + lane
                float dl = wl * ml.y;
#pragma unroll
                for (int o = 16; o; o >>= 1) dl += __shfl_xor_sync(0xffffffffu, dl, o);
                den += dl;
#pragma unroll
                for (int u = 0; u < KB; ++u) {
                    const float wk = __shfl_sync(0xffffffffu, wl, u);
                    acc.x += wk * v[u].x;
                    acc.y += wk * v[u].y;
                }
                M = Mn;
            }
            const float inv = den > 0.f ? 1.f / den : 0.f;
            acc.x *= inv;
            acc.y *= inv;
        }
        *reinterpret_cast<uint32_t *>(Os + r * X_LD + col) = pack_bf16(acc.x, acc.y);   // rows >= nr: zero
    }
    cp_async_wait<0>();
    __syncthreads();
    const int wm = warp % 2, wn = warp / 2;   // warp tile 16 rows x 32 columns
    float acc[4][4];
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[j][e] = 0.f;
#pragma unroll
    for (int kk = 0; kk < XC; kk += 16) {
        uint32_t a[4];
        ldmatrix_x4(a[0], a[1], a[2], a[3], Os + (wm * 16 + (lane % 8) + 8 * ((lane / 8) % 2)) * X_LD + kk + 8 * (lane / 16));
#pragma unroll
        for (int j = 0; j < 4; j += 2) {
            uint32_t b0, b1, b2, b3;
            ldmatrix_x4(b0, b1, b2, b3, Ws + (wn * 32 + j * 8 + (lane % 8) + 8 * (lane / 16)) * X_LD + kk + 8 * ((lane / 8) % 2));
            mma_bf16(acc[j], a, b0, b1);
            mma_bf16(acc[j + 1], a, b2, b3);
        }
    }
    __syncthreads();   // Red overwrites Ws
    const int gid = lane / 4, t4 = lane % 4;
#pragma unroll
    for (int hr = 0; hr < 2; ++hr)
#pragma unroll
        for (int j = 0; j < 4; ++j)
            *reinterpret_cast<float2 *>(Red + (wm * 16 + gid + 8 * hr) * CN + wn * 32 + j * 8 + 2 * t4) =
                make_float2(acc[j][2 * hr], acc[j][2 * hr + 1]);
    cluster.sync();
    // CTA s sums output columns [32 s, 32 s + 32) over the four slices, in slice order.
    for (int i = tid; i < nr * 16; i += 256) {
        const int r = i / 16, v = 32 * s + 2 * (i % 16);
        float2 sum = make_float2(0.f, 0.f);
#pragma unroll
        for (int q = 0; q < XS; ++q) {
            const float2 x = *reinterpret_cast<const float2 *>(cluster.map_shared_rank(Red, q) + r * CN + v);
            sum.x += x.x;
            sum.y += x.y;
        }
        *reinterpret_cast<uint32_t *>(out + ((size_t)(row0 + r) * H + h) * CN + v) = pack_bf16(sum.x, sum.y);
    }
    cluster.sync();   // the other CTAs' products stay alive until every CTA has read them
}

}  // namespace

bool combine_mma_ok(const Dims &d, int DV, bool project) {
    return project && d.bf16 && DV == CK && d.d_v == CN;
}

cudaError_t launch_combine_mma(const Dims &d, const float *part_o, const float *part_ml, const int *row_first,
                               const int *rows_host, int rows, bool oct_layout, const void *W_uv, void *out,
                               cudaStream_t st) {
    RowStarts rs;
    rs.n = 0;
    if (rows_host != nullptr && rows <= RowStarts::MAX) {
        rs.n = rows;
        for (int r = 0; r <= rows; ++r) rs.v[r] = rows_host[r];
    }
    const size_t smem = sizeof(__nv_bfloat16) * (size_t)(CN + CM) * X_LD;
    static_assert(sizeof(float) * CM * CN <= sizeof(__nv_bfloat16) * CN * X_LD, "Red fits over Ws");
    if (rows <= 0) return cudaSuccess;
    if (ceil_div(rows, CM) > 65535 || d.H > 65535) return cudaErrorInvalidValue;
    dim3 grid(XS, d.H, ceil_div(rows, CM));
    auto k = oct_layout ? combine_split_kernel<true> : combine_split_kernel<false>;
    cudaError_t e = raise_smem_limit((const void *)k, smem);
    if (e != cudaSuccess) return e;
    MLA_STEP_LAUNCH(k, dim3(grid), dim3(256), smem, st, part_o, part_ml, row_first, rs, rows, d.H,
                    (const __nv_bfloat16 *)W_uv, d.hpw, (__nv_bfloat16 *)out);
    return cudaGetLastError();
}

}  // namespace mla
