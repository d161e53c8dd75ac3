// The split-KV plan as a kernel of its own, for the query-preparation kernels that do not carry
// the plan block (plan_block.cuh has the plan itself).
#include "kernels.h"
#include "plan_block.cuh"

namespace mla {
namespace {

constexpr int PT = 1024;

constexpr int CAP = 2048;

__global__ void __launch_bounds__(PT) plan_kernel(PlanArgs a) {
    step_begin();
    __shared__ int scratch[2 * CAP + 1];
    plan_block<PT>(a, scratch, CAP);
}

}  // namespace

cudaError_t launch_plan(const PlanArgs &a, cudaStream_t st) {
    MLA_STEP_LAUNCH(plan_kernel, dim3(1), dim3(PT), 0, st, a);
    return cudaGetLastError();
}

}  // namespace mla
