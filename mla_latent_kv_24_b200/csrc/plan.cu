// Split-KV plan built on the device from the device copy of seq_lens, so that no host-to-
// device copy is needed per call.  Row r = (b, j) has len = seq_lens[b] - s_q + j + 1
// visible tokens, cut into ceil(len / chunk) chunks.  The host computes the same count from
// its copy of seq_lens to size the grid and workspace; a disagreement (or a length outside
// [s_q, max_pages * page]) sets MLA_ERR_INVALID_ARG and leaves an all-empty plan, so no
// kernel reads or writes out of range.
#include "kernels.h"

namespace mla {
namespace {

constexpr int PT = 1024;   // threads; PT / 32 == 32 warps, so one warp scans the warp totals

__global__ void __launch_bounds__(PT) plan_kernel(const int *__restrict__ seq_lens, int batch, int s_q,
                                                  int max_pages, int page, int chunk, int n_expected,
                                                  WorkItem *__restrict__ items, int *__restrict__ row_first,
                                                  int *err) {
    step_begin();
    __shared__ int warp_sum[PT / 32];
    __shared__ int bad;
    const int rows = batch * s_q;
    const int per = ceil_div(rows, PT);
    const int r0 = min(rows, threadIdx.x * per), r1 = min(rows, r0 + per);
    const int lane = threadIdx.x % 32, warp = threadIdx.x / 32;
    if (threadIdx.x == 0) bad = 0;
    __syncthreads();
    int local = 0;
    for (int r = r0; r < r1; ++r) {
        const int b = r / s_q, j = r % s_q;
        const int L = seq_lens[b];
        if (L < s_q || L > max_pages * page) atomicOr(&bad, 1);
        const int len = L - s_q + j + 1;
        local += len > 0 ? ceil_div(len, chunk) : 0;
    }
    // Exclusive prefix of the per-thread counts: warp scans, then a scan of the warp totals.
    int incl = local;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += v;
    }
    if (lane == 31) warp_sum[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int w = warp_sum[lane];
        int wi = w;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, wi, off);
            if (lane >= off) wi += v;
        }
        warp_sum[lane] = wi - w;   // exclusive
        if (lane == 31 && wi != n_expected) bad = 1;
    }
    __syncthreads();
    const int first = warp_sum[warp] + incl - local;
    if (bad) {
        if (threadIdx.x == 0) report(err, MLA_ERR_INVALID_ARG);
        for (int i = threadIdx.x; i < n_expected; i += PT) items[i] = WorkItem{0, 0, 0, 0};
        for (int i = threadIdx.x; i <= rows; i += PT) row_first[i] = 0;
        return;
    }
    int k = first;
    for (int r = r0; r < r1; ++r) {
        const int b = r / s_q, j = r % s_q;
        row_first[r] = k;
        k += ceil_div(seq_lens[b] - s_q + j + 1, chunk);
    }
    if (threadIdx.x == PT - 1) row_first[rows] = n_expected;
    __syncthreads();   // row_first (global) is visible to the whole block after this barrier
    // Items in parallel: item i belongs to the last row r with row_first[r] <= i.
    for (int i = threadIdx.x; i < n_expected; i += PT) {
        int lo = 0, hi = rows - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) / 2;
            if (row_first[mid] <= i) lo = mid;
            else hi = mid - 1;
        }
        const int b = lo / s_q, j = lo % s_q;
        const int len = seq_lens[b] - s_q + j + 1;
        const int c = i - row_first[lo];
        items[i] = WorkItem{lo, c * chunk, min(len, (c + 1) * chunk), c};
    }
}

}  // namespace

cudaError_t launch_plan(const int *seq_lens, int batch, int s_q, int max_pages, int page, int chunk,
                        int n_work_expected, WorkItem *items, int *row_first, int *err, cudaStream_t st) {
    MLA_STEP_LAUNCH(plan_kernel, dim3(1), dim3(PT), 0, st, seq_lens, batch, s_q, max_pages, page, chunk,
                    n_work_expected, items, row_first, err);
    return cudaGetLastError();
}

}  // namespace mla
