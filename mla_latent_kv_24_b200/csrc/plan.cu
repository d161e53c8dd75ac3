// Split-KV plan built on the device from the device copy of seq_lens, so that no host-to-
// device copy is needed per call.  Row r = (b, j) has len = seq_lens[b] - s_q + j + 1
// visible tokens, cut into ceil(len / chunk) chunks.  The host computes the same count from
// its copy of seq_lens to size the grid and workspace; a disagreement (or a length outside
// [s_q, max_pages * page]) sets MLA_ERR_INVALID_ARG and leaves an all-empty plan, so no
// kernel reads or writes out of range.
#include "kernels.h"

namespace mla {
namespace {

constexpr int PT = 1024;

__global__ void __launch_bounds__(PT) plan_kernel(const int *__restrict__ seq_lens, int batch, int s_q,
                                                  int max_pages, int page, int chunk, int n_expected,
                                                  WorkItem *__restrict__ items, int *__restrict__ row_first,
                                                  int *err) {
    __shared__ int part[PT];
    __shared__ int bad;
    const int rows = batch * s_q;
    const int per = ceil_div(rows, PT);
    const int r0 = min(rows, threadIdx.x * per), r1 = min(rows, r0 + per);
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
    part[threadIdx.x] = local;
    __syncthreads();
    if (threadIdx.x == 0) {
        int s = 0;
        for (int i = 0; i < PT; ++i) {
            int v = part[i];
            part[i] = s;
            s += v;
        }
        if (s != n_expected) bad = 1;
    }
    __syncthreads();
    if (bad) {
        if (threadIdx.x == 0) report(err, MLA_ERR_INVALID_ARG);
        for (int i = threadIdx.x; i < n_expected; i += PT) items[i] = WorkItem{0, 0, 0, 0};
        for (int i = threadIdx.x; i <= rows; i += PT) row_first[i] = 0;
        return;
    }
    int k = part[threadIdx.x];
    for (int r = r0; r < r1; ++r) {
        const int b = r / s_q, j = r % s_q;
        const int len = seq_lens[b] - s_q + j + 1;
        row_first[r] = k;
        const int n = ceil_div(len, chunk);
        for (int i = 0; i < n; ++i) items[k + i] = WorkItem{r, i * chunk, min(len, (i + 1) * chunk), i};
        k += n;
    }
    if (threadIdx.x == PT - 1) row_first[rows] = n_expected;
}

}  // namespace

cudaError_t launch_plan(const int *seq_lens, int batch, int s_q, int max_pages, int page, int chunk,
                        int n_work_expected, WorkItem *items, int *row_first, int *err, cudaStream_t st) {
    plan_kernel<<<1, PT, 0, st>>>(seq_lens, batch, s_q, max_pages, page, chunk, n_work_expected, items,
                                  row_first, err);
    return cudaGetLastError();
}

}  // namespace mla
