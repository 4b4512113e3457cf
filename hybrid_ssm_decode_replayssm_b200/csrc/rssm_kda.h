// Launchers of the KDA kernels (kda.cu, kda_decode.cu) for the C-ABI host code.
#pragma once

#include "rssm_internal.h"

namespace rssm {

bool kda_supported(int R, int C);
// decode (m = 1), verify (m = k drafts) and flush (m = 0); read_fmt: the
// layer's read copy (RSSM_READ_FP32: none)
cudaError_t kda_step(const StepArgs &a, int in_dtype, int read_fmt, cudaStream_t s);
// The decode serving path (one token, bf16 inputs): its own persistent kernel
// with prologue warps and tensor-core folds (kda_decode.cu).
bool kda_decode_fast_path(const StepArgs &a, int in_dtype);
// Bytes of that kernel's per-CTA fold-operand scratch in the ring buffer (0 if
// the kernel does not serve the descriptor).
size_t kda_fold_scratch_bytes(const rssm_layer_desc &d);
cudaError_t kda_decode_step(const StepArgs &a, cudaStream_t s);
// fp32 state only
cudaError_t kda_conventional(const ConvArgs &a, int in_dtype, cudaStream_t s);

}  // namespace rssm
