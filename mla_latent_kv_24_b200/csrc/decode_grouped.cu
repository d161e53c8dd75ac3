// Grouped (GQA-path) tensor-core decode (not built yet: the CUDA-core kernel runs meanwhile).
#include "tc_decode.h"

namespace mla {

bool grouped_tc_ok(const Dims &) { return false; }
int grouped_units(const Dims &, int sms) { return sms; }
int grouped_token_granule() { return 64; }
cudaError_t launch_grouped_decode(const Dims &, const void *, const void *, const void *, const int *, const int *,
                                  const Plan &, int, int, int, float *, float *, int *, cudaStream_t) {
    return cudaErrorNotSupported;
}

}  // namespace mla
