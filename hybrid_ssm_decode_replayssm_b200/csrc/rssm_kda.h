// Launchers of the KDA kernels (kda.cu) for the C-ABI host code.
#pragma once

#include "rssm_internal.h"

namespace rssm {

bool kda_supported(int R, int C);
// decode (m = 1) and flush (m = 0); verify is not built for KDA
cudaError_t kda_step(const StepArgs &a, int in_dtype, cudaStream_t s);
// fp32 state only
cudaError_t kda_conventional(const ConvArgs &a, int in_dtype, cudaStream_t s);

}  // namespace rssm
