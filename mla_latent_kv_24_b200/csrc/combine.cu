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
                                                      const int *__restrict__ row_first, int rows, int H,
                                                      int DV, const T *__restrict__ W_uv, int hpw, int d_v,
                                                      T *__restrict__ out) {
    extern __shared__ float O[];  // [RB][DV]
    const int h = blockIdx.x;
    const int row0 = blockIdx.y * RB;
    const int nr = min(RB, rows - row0);
    for (int r = 0; r < nr; ++r) {
        const int k0 = row_first[row0 + r], k1 = row_first[row0 + r + 1];
        float M = -INFINITY;
        for (int k = k0; k < k1; ++k) M = fmaxf(M, part_ml[((size_t)k * H + h) * 2]);
        float den = 0.f;
        for (int k = k0; k < k1; ++k) {
            const float mk = part_ml[((size_t)k * H + h) * 2];
            if (mk != -INFINITY) den += expf(mk - M) * part_ml[((size_t)k * H + h) * 2 + 1];
        }
        const float inv = den > 0.f ? 1.f / den : 0.f;
        for (int c = threadIdx.x; c < DV; c += blockDim.x) {
            float num = 0.f;
            for (int k = k0; k < k1; ++k) {
                const float mk = part_ml[((size_t)k * H + h) * 2];
                if (mk != -INFINITY) num += expf(mk - M) * part_o[((size_t)k * H + h) * DV + c];
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
                           int rows, int DV, const void *W_uv, void *out, cudaStream_t st) {
    dim3 grid(d.H, ceil_div(rows, RB));
    const size_t smem = sizeof(float) * RB * DV;
    if (d.bf16) {
        auto k = combine_kernel<__nv_bfloat16>;
        cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        k<<<grid, 256, smem, st>>>(part_o, part_ml, row_first, rows, d.H, DV, (const __nv_bfloat16 *)W_uv,
                                   d.hpw, d.d_v, (__nv_bfloat16 *)out);
    } else {
        auto k = combine_kernel<float>;
        cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        k<<<grid, 256, smem, st>>>(part_o, part_ml, row_first, rows, d.H, DV, (const float *)W_uv, d.hpw, d.d_v,
                                   (float *)out);
    }
    return cudaGetLastError();
}

}  // namespace mla
