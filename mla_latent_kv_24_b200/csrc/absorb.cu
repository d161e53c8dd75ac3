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
#include "plan_block.cuh"

namespace mla {
namespace {

constexpr int RB = 16;

template <typename T>
__global__ void __launch_bounds__(256) q_absorb_kernel(const T *__restrict__ q, const T *__restrict__ W_uk,
                                                       const int *__restrict__ seq_lens, int rows, int s_q,
                                                       int H, int hpw, int d_c, int d_r, int d_n, float base,
                                                       T *__restrict__ q_abs) {
    step_begin();
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
// The last block builds the split plan instead.
template <typename T>
__global__ void __launch_bounds__(256) q_rope_kernel(const T *__restrict__ q, const int *__restrict__ seq_lens,
                                                     int rows, int s_q, int H, int d_r, int d_n, float base,
                                                     T *__restrict__ q_rot, PlanArgs plan) {
    step_begin();
    if (blockIdx.x == gridDim.x - 1) {
        __shared__ int scratch[2 * 512 + 1];
        plan_block<256>(plan, scratch, 512);
        return;
    }
    const int d_qk = d_n + d_r;
    const size_t n = (size_t)rows * H * (d_qk / 2);
    const size_t stride = (size_t)(gridDim.x - 1) * blockDim.x;
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += stride) {
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
        MLA_STEP_LAUNCH(q_absorb_kernel<__nv_bfloat16>, dim3(grid), dim3(256), 0, st, (const __nv_bfloat16 *)q,
                        (const __nv_bfloat16 *)W_uk, seq_lens, rows, s_q, d.H, d.hpw, d.d_c, d.d_r, d.d_n, d.base,
                        (__nv_bfloat16 *)q_abs);
    else
        MLA_STEP_LAUNCH(q_absorb_kernel<float>, dim3(grid), dim3(256), 0, st, (const float *)q, (const float *)W_uk,
                        seq_lens, rows, s_q, d.H, d.hpw, d.d_c, d.d_r, d.d_n, d.base, (float *)q_abs);
    return cudaGetLastError();
}

cudaError_t launch_q_rope(const Dims &d, const void *q, const int *seq_lens, int batch, int s_q, void *q_rot,
                          const PlanArgs &plan, cudaStream_t st) {
    const int rows = batch * s_q;
    const size_t n = (size_t)rows * d.H * ((d.d_n + d.d_r) / 2);
    const int blocks = (int)std::min<size_t>((n + 255) / 256, 4096) + 1;   // + the plan block
    if (d.bf16)
        MLA_STEP_LAUNCH(q_rope_kernel<__nv_bfloat16>, dim3(blocks), dim3(256), 0, st, (const __nv_bfloat16 *)q,
                        seq_lens, rows, s_q, d.H, d.d_r, d.d_n, d.base, (__nv_bfloat16 *)q_rot, plan);
    else
        MLA_STEP_LAUNCH(q_rope_kernel<float>, dim3(blocks), dim3(256), 0, st, (const float *)q, seq_lens, rows, s_q,
                        d.H, d.d_r, d.d_n, d.base, (float *)q_rot, plan);
    return cudaGetLastError();
}

}  // namespace mla

// ---------------------------------------------------------------------------------------
// Tensor-core q absorption for the DeepSeek-V2 shape (bf16, d_nope = 128, d_c = 512,
// d_rope = 64).  Per head it is the GEMM q_lat[rows, 512] = q_nope[rows, 128] W_UK[w]
// ([128, 512], row k = nope dim).  One CTA computes 64 query rows x 128 latent columns of one
// head with mma.sync m16n8k16: the W_UK tile [128 k][64 n] and the q tile [64][128] are staged
// in padded shared memory by cp.async, B fragments come through ldmatrix.trans.  Every W_UK
// element is read once per head (16.8 MB in total for H = 128), the bound of this step.
// CTAs of the first column tile also rotate the query's RoPE part.
// ---------------------------------------------------------------------------------------
#include "warp_mma.cuh"

namespace mla {
namespace {

constexpr int AB_K = 128, AB_LD = AB_K + 8;

// TM query rows x TN latent columns of one head per CTA; eight warps as (TM / 16) row tiles x
// (8 / (TM / 16)) column groups.  Small batches take 16 x 128 tiles, so that a decode step's
// whole grid (4 column tiles per head) is one wave of CTAs: a CTA stores only after the previous
// kernel has completed, and a second wave would start its loads only then.
template <int TM, int TN>
__global__ void __launch_bounds__(256) q_absorb_mma_kernel(const __nv_bfloat16 *__restrict__ q,
                                                           const __nv_bfloat16 *__restrict__ W_uk,
                                                           const int *__restrict__ seq_lens, int rows, int s_q,
                                                           int H, int hpw, float base,
                                                           __nv_bfloat16 *__restrict__ q_abs, PlanArgs plan) {
    constexpr int LDB = TN + 8, WM = TM / 16, WN = 8 / WM, CW = TN / WN, NT = CW / 8;
    static_assert(TM % 16 == 0 && 8 % WM == 0 && NT % 2 == 0, "warp tiling");
    step_allow_next();   // loads and products touch inputs only; every store waits (below)
    __shared__ __align__(16) __nv_bfloat16 As[TM * AB_LD];     // [rows][128 k]
    __shared__ __align__(16) __nv_bfloat16 Bs[AB_K * LDB];     // [128 k][TN n]
    if (blockIdx.x == H) {   // the extra column of blocks: its first block builds the split plan
        constexpr int CAP = ((int)sizeof(Bs) / 4 - 1) / 2;      // row starts and lengths in Bs
        if (blockIdx.y == 0 && blockIdx.z == 0) plan_block<256>(plan, reinterpret_cast<int *>(Bs), CAP);
        return;
    }
    const int h = blockIdx.x, n0 = blockIdx.y * TN, row0 = blockIdx.z * TM;
    const int w = h / hpw, tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
    constexpr int D_C = 512, D_N = 128, D_R = 64, D_QK = 192, D_OUT = 576;
    const __nv_bfloat16 *Wk = W_uk + (size_t)w * D_N * D_C;
    for (int c = tid; c < AB_K * TN / 8; c += 256) {            // 16-byte chunks of the W_UK tile
        const int k = c / (TN / 8), n = (c % (TN / 8)) * 8;
        cp_async16(Bs + k * LDB + n, Wk + (size_t)k * D_C + n0 + n, true);
    }
    for (int c = tid; c < TM * AB_K / 8; c += 256) {
        const int r = c / (AB_K / 8), k = (c % (AB_K / 8)) * 8;
        const int row = row0 + r;
        cp_async16(As + r * AB_LD + k, q + ((size_t)(row < rows ? row : 0) * H + h) * D_QK + k, row < rows);
    }
    cp_async_commit();
    cp_async_wait<0>();
    __syncthreads();
    // warp tile: 16 rows x CW columns (NT n8 tiles)
    const int wm = warp % WM, wn = warp / WM;
    float acc[NT][4];
#pragma unroll
    for (int j = 0; j < NT; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[j][e] = 0.f;
#pragma unroll
    for (int kk = 0; kk < AB_K; kk += 16) {
        uint32_t a[4];
        ldmatrix_x4(a[0], a[1], a[2], a[3],
                    As + (wm * 16 + (lane % 8) + 8 * ((lane / 8) % 2)) * AB_LD + kk + 8 * (lane / 16));
#pragma unroll
        for (int j = 0; j < NT; j += 2) {
            // B stored [k][n]: .trans gives the k-major fragments of two n8 tiles
            uint32_t b0, b1, b2, b3;
            const int kr = kk + (lane % 8) + 8 * ((lane / 8) % 2);
            const int nc = wn * CW + j * 8 + 8 * (lane / 16);
            ldmatrix_x4_trans(b0, b1, b2, b3, Bs + kr * LDB + nc);
            mma_bf16(acc[j], a, b0, b1);
            mma_bf16(acc[j + 1], a, b2, b3);
        }
    }
    const int gid = lane / 4, t4 = lane % 4;
    step_wait_prev();   // q_abs is workspace the previous call's kernels may still read
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {
        const int row = row0 + wm * 16 + gid + 8 * hr;
        if (row >= rows) continue;
        __nv_bfloat16 *dst = q_abs + ((size_t)row * H + h) * D_OUT + n0 + wn * CW;
#pragma unroll
        for (int j = 0; j < NT; ++j)
            *reinterpret_cast<uint32_t *>(dst + j * 8 + 2 * t4) = pack_bf16(acc[j][2 * hr], acc[j][2 * hr + 1]);
    }
    if (blockIdx.y == 0) {   // RoPE part of the query, rows of this tile
        for (int i = tid; i < TM * (D_R / 2); i += 256) {
            const int r = i / (D_R / 2), pi = i % (D_R / 2), row = row0 + r;
            if (row >= rows) continue;
            const int b = row / s_q, j = row % s_q, pos = seq_lens[b] - s_q + j;
            const __nv_bfloat16 *src = q + ((size_t)row * H + h) * D_QK + D_N + 2 * pi;
            float x0 = __bfloat162float(src[0]), x1 = __bfloat162float(src[1]), cs, sn;
            rope_cos_sin(pos, pi, D_R, base, &cs, &sn);
            __nv_bfloat16 *o = q_abs + ((size_t)row * H + h) * D_OUT + D_C + 2 * pi;
            o[0] = __float2bfloat16_rn(x0 * cs - x1 * sn);
            o[1] = __float2bfloat16_rn(x0 * sn + x1 * cs);
        }
    }
}

}  // namespace

bool q_absorb_mma_ok(const Dims &d) { return d.bf16 && d.d_n == 128 && d.d_c == 512 && d.d_r == 64; }

cudaError_t launch_q_absorb_mma(const Dims &d, const void *q, const void *W_uk, const int *seq_lens, int batch,
                                int s_q, void *q_abs, const PlanArgs &plan, cudaStream_t st) {
    const int rows = batch * s_q;
    if (rows <= 16) {
        dim3 grid(d.H + 1, 512 / 128, 1);   // + one column for the plan block
        MLA_STEP_LAUNCH(q_absorb_mma_kernel<16, 128>, dim3(grid), dim3(256), 0, st, (const __nv_bfloat16 *)q,
                        (const __nv_bfloat16 *)W_uk, seq_lens, rows, s_q, d.H, d.hpw, d.base, (__nv_bfloat16 *)q_abs,
                        plan);
    } else {
        dim3 grid(d.H + 1, 512 / 64, ceil_div(rows, 64));
        MLA_STEP_LAUNCH(q_absorb_mma_kernel<64, 64>, dim3(grid), dim3(256), 0, st, (const __nv_bfloat16 *)q,
                        (const __nv_bfloat16 *)W_uk, seq_lens, rows, s_q, d.H, d.hpw, d.base, (__nv_bfloat16 *)q_abs,
                        plan);
    }
    return cudaGetLastError();
}

}  // namespace mla
