// Split-KV plan built on the device by one thread block, from the device copy of seq_lens, so
// that no host-to-device copy is needed per call.  Row r = (b, j) has len = seq_lens[b] - s_q +
// j + 1 visible tokens, cut into ceil(len / chunk) chunks.  The host computes the same count
// from its copy of seq_lens to size the grid and workspace; a disagreement (or a length outside
// [s_q, max_pages * page]) sets MLA_ERR_INVALID_ARG and leaves an all-empty plan, so no kernel
// reads or writes out of range.
//
// The block is either a kernel of its own (plan.cu) or one extra block of the query-preparation
// kernel that runs before the decode, which saves a launch per call.
#pragma once

#include "common.cuh"

namespace mla {

// `scratch` is shared memory of the calling block (2 * cap_rows + 1 ints, the block's own
// buffers, which the plan block does not otherwise use): batches of at most cap_rows rows keep
// the row starts and lengths there, so the block's dependent reads (the binary searches of the
// items) never wait on global memory.  Larger batches read them back from global memory.
// Run by all PT threads of one block (PT a multiple of 32, at most 1024).
template <int PT>
__device__ __forceinline__ void plan_block(const PlanArgs &a, int *scratch, int cap_rows) {
    static_assert(PT % 32 == 0 && PT <= 1024, "one warp scans the warp totals");
    __shared__ int warp_sum[PT / 32];
    __shared__ int bad;
    const int rows = a.batch * a.s_q;
    const bool in_smem = rows <= cap_rows;
    int *s_first = scratch, *s_len = scratch + cap_rows + 1;
    const int per = ceil_div(rows, PT);
    const int r0 = min(rows, (int)threadIdx.x * per), r1 = min(rows, r0 + per);
    const int lane = threadIdx.x % 32, warp = threadIdx.x / 32;
    if (threadIdx.x == 0) bad = 0;
    __syncthreads();
    int local = 0;
    for (int r = r0; r < r1; ++r) {
        const int b = r / a.s_q, j = r % a.s_q;
        const int L = a.seq_lens[b];
        if (L < a.s_q || L > a.max_pages * a.page) atomicOr(&bad, 1);
        const int len = L - a.s_q + j + 1;
        if (in_smem) s_len[r] = len;
        local += len > 0 ? ceil_div(len, a.chunk) : 0;
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
        const int w = lane < PT / 32 ? warp_sum[lane] : 0;
        int wi = w;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, wi, off);
            if (lane >= off) wi += v;
        }
        if (lane < PT / 32) warp_sum[lane] = wi - w;   // exclusive
        if (lane == 31 && wi != a.n_expected) bad = 1;
    }
    __syncthreads();
    const int first = warp_sum[warp] + incl - local;
    step_wait_prev();   // a no-op once the kernel waited; else the plan is workspace the previous call may still read
    if (bad) {
        if (threadIdx.x == 0) report(a.err, MLA_ERR_INVALID_ARG);
        for (int i = threadIdx.x; i < a.n_expected; i += PT) a.items[i] = WorkItem{0, 0, 0, 0};
        for (int i = threadIdx.x; i <= rows; i += PT) a.row_first[i] = 0;
        if (a.order)
            for (int i = threadIdx.x; i < a.n_expected; i += PT) a.order[i] = i;
        return;
    }
    int k = first;
    for (int r = r0; r < r1; ++r) {
        const int b = r / a.s_q, j = r % a.s_q;
        a.row_first[r] = k;
        if (in_smem) s_first[r] = k;
        k += ceil_div(in_smem ? s_len[r] : a.seq_lens[b] - a.s_q + j + 1, a.chunk);
    }
    if (threadIdx.x == PT - 1) {
        a.row_first[rows] = a.n_expected;
        if (in_smem) s_first[rows] = a.n_expected;
    }
    // Take order (optional).  A row's chunks all have `chunk` tokens except, usually, its last one;
    // the order lists the full chunks first, in index order, then the rows' shorter last chunks,
    // longest first (OB length buckets; inside a bucket in the order the atomics give, which only
    // decides which worker runs an item, never its result).  A full chunk's position is its index
    // minus the number of shorter last chunks before it, i.e. of the rows before its own that end
    // in one (an exclusive prefix P over rows, kept after the order).  A persistent decode that
    // deals these positions to its workers in snake order (0..U-1, U-1..0, ...) gives every worker
    // a similar number of tokens even when the rows' lengths differ widely.
    constexpr int OB = 64;
    __shared__ int o_hist[OB], o_start[OB], o_fill[OB], o_full;
    int *P = a.order ? a.order + a.n_expected : nullptr;
    if (a.order) {
        for (int i = threadIdx.x; i < OB; i += PT) o_hist[i] = 0, o_fill[i] = 0;
        __syncthreads();
        int lp = 0;   // rows of this thread that end in a shorter chunk
        for (int r = r0; r < r1; ++r) {
            const int b = r / a.s_q, j = r % a.s_q;
            const int len = in_smem ? s_len[r] : a.seq_lens[b] - a.s_q + j + 1;
            const int last = len - (ceil_div(len, a.chunk) - 1) * a.chunk;
            if (last < a.chunk) {
                ++lp;
                atomicAdd(&o_hist[min(OB - 1, (int)((long long)last * OB / a.chunk))], 1);
            }
        }
        int inc = lp;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, inc, off);
            if (lane >= off) inc += v;
        }
        __syncthreads();   // warp_sum is reused
        if (lane == 31) warp_sum[warp] = inc;
        __syncthreads();
        if (warp == 0) {
            const int w = lane < PT / 32 ? warp_sum[lane] : 0;
            int wi = w;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int v = __shfl_up_sync(0xffffffffu, wi, off);
                if (lane >= off) wi += v;
            }
            if (lane < PT / 32) warp_sum[lane] = wi - w;   // exclusive
            if (lane == 31) o_full = a.n_expected - wi;
        }
        __syncthreads();
        int pr = warp_sum[warp] + inc - lp;
        for (int r = r0; r < r1; ++r) {
            P[r] = pr;
            const int b = r / a.s_q, j = r % a.s_q;
            const int len = in_smem ? s_len[r] : a.seq_lens[b] - a.s_q + j + 1;
            if (len - (ceil_div(len, a.chunk) - 1) * a.chunk < a.chunk) ++pr;
        }
        if (threadIdx.x == 0) {
            int acc = 0;
            for (int bk = OB - 1; bk >= 0; --bk) {   // longest bucket first
                o_start[bk] = acc;
                acc += o_hist[bk];
            }
        }
    }
    __syncthreads();   // row_first, P and the buckets are visible to the whole block after this barrier
    const int *rf = in_smem ? s_first : a.row_first;
    // Items in parallel: item i belongs to the last row r with row_first[r] <= i.
    for (int i = threadIdx.x; i < a.n_expected; i += PT) {
        int lo = 0, hi = rows - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) / 2;
            if (rf[mid] <= i) lo = mid;
            else hi = mid - 1;
        }
        const int b = lo / a.s_q, j = lo % a.s_q;
        const int len = in_smem ? s_len[lo] : a.seq_lens[b] - a.s_q + j + 1;
        const int c = i - rf[lo];
        a.items[i] = WorkItem{lo, c * a.chunk, min(len, (c + 1) * a.chunk), c};
        if (a.order) {
            const int n_c = ceil_div(len, a.chunk), last = len - (n_c - 1) * a.chunk;
            int pos;
            if (c == n_c - 1 && last < a.chunk) {
                const int bk = min(OB - 1, (int)((long long)last * OB / a.chunk));
                pos = o_full + o_start[bk] + atomicAdd(&o_fill[bk], 1);
            } else {
                pos = i - P[lo];
            }
            a.order[pos] = i;
        }
    }
}

}  // namespace mla
