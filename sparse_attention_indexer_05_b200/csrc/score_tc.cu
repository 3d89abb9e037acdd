// score_tc.cu -- tcgen05 / TMEM / TMA score kernels (bf16, H = 64, d = 128).
#include "common.cuh"
#include "internal.h"

namespace idx {

bool tc_supported(int H, int d, int dtype) {
    (void)H; (void)d; (void)dtype;
    return false;
}

cudaError_t launch_score_tc(const ScoreArgs &, cudaStream_t) { return cudaErrorNotSupported; }
cudaError_t launch_decode_tc(const DecodeArgs &, cudaStream_t) { return cudaErrorNotSupported; }
cudaError_t launch_gather_tc(const GatherArgs &, cudaStream_t) { return cudaErrorNotSupported; }

}  // namespace idx
