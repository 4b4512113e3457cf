// Gated DeltaNet kernels (not built yet in this revision).
#include "rssm_device.cuh"

namespace rssm {

bool gdn_supported(int, int) { return false; }

cudaError_t gdn_step(const StepArgs &, int, int, cudaStream_t) { return cudaErrorNotSupported; }

cudaError_t gdn_conventional(const ConvArgs &, int, cudaStream_t) { return cudaErrorNotSupported; }

}  // namespace rssm
