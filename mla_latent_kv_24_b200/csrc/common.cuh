// Shared device helpers for libmla kernels (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include <mutex>
#include <utility>

#include "mla.h"

namespace mla {

// ---------------------------------------------------------------------------------------
// Device error word: kernels never trap; they record the first error code and skip the
// offending access.  The host reads and clears it in mla_get_device_status().
// ---------------------------------------------------------------------------------------
__device__ __forceinline__ void report(int *err, int code) {
    if (err) atomicCAS(err, 0, code);
}

// ---------------------------------------------------------------------------------------
// Storage types.
// ---------------------------------------------------------------------------------------
__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

// RoPE angle for pair i of a d-wide vector at position pos: pos * base^(-2i/d), with the
// product and the trigonometry in double precision so that large positions (2^17) keep
// full single-precision accuracy after rounding.
__device__ __forceinline__ void rope_cos_sin(int pos, int i, int d, float base, float *c, float *s) {
    double theta = pow((double)base, -2.0 * (double)i / (double)d);
    double ang = (double)pos * theta;
    double sd, cd;
    sincos(ang, &sd, &cd);
    *c = (float)cd;
    *s = (float)sd;
}

__host__ __device__ __forceinline__ int ceil_div(int a, int b) { return (a + b - 1) / b; }

// ---------------------------------------------------------------------------------------
// Programmatic dependent launch.  The kernels of a call are launched with programmatic stream
// serialisation, so a kernel's CTAs may be launched while the previous kernel of the stream is
// still running.  Every such kernel calls step_begin() before anything else: it waits until the
// previous kernel has completed and its writes are visible (griddepcontrol.wait), then allows
// the next kernel to start launching (griddepcontrol.launch_dependents).  Execution order and
// memory order therefore stay those of a plain stream, and only the launch latency of the next
// kernel overlaps this one.  Both instructions do nothing in a kernel launched without the
// attribute.
// ---------------------------------------------------------------------------------------
__device__ __forceinline__ void step_begin() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
// The split form, for kernels whose loads touch only the caller's inputs (weights, queries, hidden
// states, lengths, page tables), which no kernel of this library writes: they let the next kernel
// launch at once, load and compute while the previous kernel finishes, and call step_wait_prev()
// before their first store.  Every thread that stores calls it, so the kernel completes only after
// its predecessor has, and ordering down the stream stays that of a plain stream.
__device__ __forceinline__ void step_allow_next() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void step_wait_prev() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// ---------------------------------------------------------------------------------------
// Split-KV plan.  Row r = (b, j) has len_r = seq_lens[b] - s_q + j + 1 visible tokens and
// is cut into ceil(len_r / chunk) chunks of `chunk` tokens (the last one ragged).  Work item
// k covers tokens [t0, t1) of one row; partial results are stored at index k.
// ---------------------------------------------------------------------------------------
struct WorkItem {
    int row;     // b * s_q + j
    int t0, t1;  // token range
    int split;   // chunk index inside the row
};

// Inputs and outputs of the device-side plan builder (plan_block.cuh).
struct PlanArgs {
    const int *seq_lens;
    int batch, s_q, max_pages, page, chunk, n_expected;
    WorkItem *items;     // [n_expected]
    int *row_first;      // [batch * s_q + 1]
    int *err;
    int *order;          // optional: [n_expected] take order of the items (see plan_block), then
                         // [batch * s_q + 1] scratch
};

struct Plan {
    const WorkItem *items;  // [n_work]
    const int *row_first;   // [rows + 1] first work item of each row (prefix sums)
    int n_work;
    int rows;
    int chunk;
    const int *order;       // nullptr, or the order in which a persistent decode takes the items
};

}  // namespace mla

namespace mla {
// Launches `kernel` on `st` with programmatic stream serialisation (the kernel must call
// step_begin() first).  Host only.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_step(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                               Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// One statement: launch with launch_step() and return its error, if any, from the caller.
#define MLA_STEP_LAUNCH(kernel, grid, block, smem, st, ...)                                       \
    do {                                                                                          \
        const cudaError_t e_launch_ = ::mla::launch_step(kernel, grid, block, smem, st, __VA_ARGS__); \
        if (e_launch_ != cudaSuccess) return e_launch_;                                           \
    } while (0)

// Raises a kernel's dynamic shared-memory limit on the current device once, to the largest size
// asked so far; later launches that need no more skip the driver call (it costs microseconds of
// host time per launch).  Host only; thread-safe.
inline cudaError_t raise_smem_limit(const void *kernel, size_t bytes) {
    struct Entry {
        const void *kernel;
        int device;
        size_t bytes;
    };
    static std::mutex mu;
    static Entry table[256];
    static int n = 0;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lock(mu);
    Entry *hit = nullptr;
    for (int i = 0; i < n; ++i)
        if (table[i].kernel == kernel && table[i].device == dev) hit = &table[i];
    if (hit && hit->bytes >= bytes) return cudaSuccess;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e != cudaSuccess) return e;
    if (hit)
        hit->bytes = bytes;
    else if (n < 256)
        table[n++] = Entry{kernel, dev, bytes};
    return cudaSuccess;
}
}  // namespace mla
