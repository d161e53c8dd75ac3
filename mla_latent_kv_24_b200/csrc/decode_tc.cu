// tcgen05 absorbed decode (not built yet: the CUDA-core kernel runs meanwhile).
#include "tc_decode.h"

namespace mla {

bool tc_available() { return false; }
int tc_units(int sms) { return sms / 2; }
int tc_token_granule() { return 128; }
cudaError_t launch_tc_decode(const Dims &, const void *, const void *, const int *, const Plan &, int, int, int,
                             float *, float *, int *, int, cudaStream_t) {
    return cudaErrorNotSupported;
}

}  // namespace mla
