// Read-copy quantiser and integer bookkeeping kernels.
#include "rssm_device.cuh"

namespace rssm {
namespace {

// Whole read copy from the fp32 checkpoint: a warp walks rows of C elements,
// each lane owning 4 consecutive columns (C = 64: two rows per warp step).
template <int C, int RF>
__global__ void __launch_bounds__(256) quantize_kernel(const QuantArgs a) {
  constexpr int LPR = C / 4, RPI = 32 / LPR;
  constexpr int RB = RF == RSSM_READ_NVFP4 ? C / 2 : C;
  const int lane = threadIdx.x & 31;
  const size_t warp = ((size_t)blockIdx.x * blockDim.x + threadIdx.x) / 32;
  const size_t nwarps = (size_t)gridDim.x * blockDim.x / 32;
  const int c0 = (lane % LPR) * 4;
  for (size_t r0 = warp * RPI; r0 < a.rows; r0 += nwarps * RPI) {
    const size_t row = r0 + lane / LPR;
    const float4 v = ld_stream(a.hc + row * C + c0);
    quantize4<RF, LPR>(v, a.codes + row * RB, a.scales, row, C, c0, lane);
  }
}

__global__ void rollback_kernel(int B, const int32_t *n_reject, int32_t *len, int32_t *pending,
                                uint32_t *status) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= B) return;
  const int n = n_reject[b], p = pending[b];
  if (n < 0 || n > p) {
    atomicOr(status, (unsigned)RSSM_STATUS_STATE);
    return;
  }
  len[b] += p - n;
  pending[b] = 0;
}

__global__ void gather_kernel(int B, const int32_t *start, const int32_t *len,
                              const int32_t *pending, const int32_t *flushes, int32_t *out) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= B) return;
  out[b] = start[b];
  out[B + b] = len[b];
  out[2 * B + b] = pending[b];
  out[3 * B + b] = flushes[b];
}

template <int C, int RF>
cudaError_t launch_quant(const QuantArgs &a, cudaStream_t s) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const size_t warps_needed = (a.rows * (C / 4) + 31) / 32;
  size_t blocks = (warps_needed + 7) / 8;
  blocks = blocks < (size_t)sms * 8 ? blocks : (size_t)sms * 8;
  if (blocks == 0) return cudaSuccess;
  quantize_kernel<C, RF><<<dim3((unsigned)blocks), dim3(256), 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t quantize_read_copy(const QuantArgs &a, int read_fmt, cudaStream_t s) {
  if (a.C == 64)
    return read_fmt == RSSM_READ_NVFP4 ? launch_quant<64, RSSM_READ_NVFP4>(a, s)
                                       : launch_quant<64, RSSM_READ_FP8_E4M3_ROW>(a, s);
  return read_fmt == RSSM_READ_NVFP4 ? launch_quant<128, RSSM_READ_NVFP4>(a, s)
                                     : launch_quant<128, RSSM_READ_FP8_E4M3_ROW>(a, s);
}

cudaError_t rollback(int B, const int32_t *n_reject, int32_t *len, int32_t *pending,
                     uint32_t *status, cudaStream_t s) {
  rollback_kernel<<<dim3((unsigned)((B + 255) / 256)), dim3(256), 0, s>>>(B, n_reject, len, pending, status);
  return cudaGetLastError();
}

cudaError_t gather_bookkeeping(int B, const int32_t *start, const int32_t *len,
                               const int32_t *pending, const int32_t *flushes, int32_t *out,
                               cudaStream_t s) {
  gather_kernel<<<dim3((unsigned)((B + 255) / 256)), dim3(256), 0, s>>>(B, start, len, pending, flushes, out);
  return cudaGetLastError();
}

}  // namespace rssm
