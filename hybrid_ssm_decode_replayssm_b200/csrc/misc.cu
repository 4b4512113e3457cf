// Read-copy quantiser, integer bookkeeping and branching kernels.
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

// ------------------------------------------------------------ branching
// Exclusive prefix sum of one int per thread over the block (blockDim.x a
// multiple of 32, at most 1024); `total` is the block's sum.
__device__ __forceinline__ void block_scan(int v, int &excl, int &total) {
  __shared__ int warp_tot[32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  int inc = v;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const int t = __shfl_up_sync(kFull, inc, d);
    if (lane >= d) inc += t;
  }
  if (lane == 31) warp_tot[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    int w = lane < nw ? warp_tot[lane] : 0;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int t = __shfl_up_sync(kFull, w, d);
      if (lane >= d) w += t;
    }
    if (lane < nw) warp_tot[lane] = w;   // inclusive over warps
  }
  __syncthreads();
  excl = inc - v + (warp > 0 ? warp_tot[warp - 1] : 0);
  total = warp_tot[nw - 1];
  __syncthreads();   // warp_tot is reused by the next call
}

// A fold of the previous launch wrote row b's new checkpoint to dst[b] and
// counted itself in flushes[b]: make that slot the row's own.
__device__ __forceinline__ void adopt_folds(int B, int32_t *slot, const int32_t *dst, int32_t *seen,
                                            const int32_t *flushes) {
  for (int b = threadIdx.x; b < B; b += blockDim.x) {
    const int f = flushes[b];
    if (f != seen[b]) {
      slot[b] = dst[b];
      seen[b] = f;
    }
  }
}

// One CTA.  Slots are 0 .. 2B-1; rows reference at most B of them, so at
// least B are free and every row that folds in the coming launch gets a
// distinct free slot: a fold never writes a slot that any row reads.
__global__ void __launch_bounds__(1024) plan_slots_kernel(const StepArgs a, int32_t *slot, int32_t *dst,
                                                          int32_t *seen, int32_t *freelist) {
  const int B = a.B, S = 2 * B, nt = blockDim.x;
  adopt_folds(B, slot, dst, seen, a.flushes);
  __syncthreads();
  for (int s = threadIdx.x; s < S; s += nt) freelist[s] = 1;
  __syncthreads();
  for (int b = threadIdx.x; b < B; b += nt) {
    const int sl = slot[b];
    if (sl >= 0 && sl < S) freelist[sl] = 0;
  }
  __syncthreads();
  // compact the free slot ids to the front, tile by tile (a tile's flags are
  // read before any id is written, and ids land at or before their slot)
  int nfree = 0;
  for (int s0 = 0; s0 < S; s0 += nt) {
    const int s = s0 + threadIdx.x;
    const int flag = s < S ? freelist[s] : 0;
    __syncthreads();
    int excl, tot;
    block_scan(flag, excl, tot);
    if (flag) freelist[nfree + excl] = s;
    nfree += tot;
    __syncthreads();
  }
  int rank = 0;
  for (int b0 = 0; b0 < B; b0 += nt) {
    const int b = b0 + threadIdx.x;
    int fold = 0;
    if (b < B) {
      const RowPlan r = plan_row(a, b);
      fold = !r.refuse && (r.pre || r.post);
    }
    int excl, tot;
    block_scan(fold, excl, tot);
    if (fold) dst[b] = rank + excl < nfree ? freelist[rank + excl] : slot[b];   // nfree >= B always
    rank += tot;
  }
}

// rssm_branch, step 1 (one CTA): adopt pending folds; decide each row's
// effective parent (eff = parent, or -1 when refused); gather the parents'
// slot and pointers (all read before any is written).
__global__ void __launch_bounds__(1024) branch_book_kernel(const BranchArgs a, const int32_t *parent,
                                                           int32_t *tmp) {
  const int B = a.B, nt = blockDim.x;
  adopt_folds(B, a.slot, a.dst, a.seen, a.flushes);
  __syncthreads();
  for (int b = threadIdx.x; b < B; b += nt) {
    const int p = parent[b];
    const bool ok = p >= 0 && p < B && a.pending[p] == 0;
    a.eff[b] = ok ? p : -1;
    if (!ok) atomicOr(a.status, (unsigned)RSSM_STATUS_STATE);
    if (ok && p != b) {
      tmp[b] = a.slot[p];
      tmp[B + b] = a.start[p];
      tmp[2 * B + b] = a.len[p];
      tmp[3 * B + b] = a.flushes[p];
    }
  }
  __syncthreads();
  for (int b = threadIdx.x; b < B; b += nt) {
    const int p = a.eff[b];
    if (p >= 0 && p != b) {
      a.slot[b] = tmp[b];
      a.start[b] = tmp[B + b];
      a.len[b] = tmp[2 * B + b];
      a.flushes[b] = tmp[3 * B + b];
      a.seen[b] = tmp[3 * B + b];
      a.pending[b] = 0;
    }
  }
}

// rssm_branch, steps 2 and 3: the live window entries of every row with a
// new parent go ring -> scratch (from the parent's rings) and then scratch ->
// ring (into the row's), so a row that is both a parent and a child is read
// before it is overwritten.  After step 1 the child's start and len are the
// parent's, so both passes copy entries (start + e) % cap, e < len, of each of
// the row's rings.  One warp per (row, ring); 16-byte words where the entry
// size allows, else 4-byte words.
template <bool kToScratch>
__global__ void __launch_bounds__(256) branch_copy_kernel(const BranchArgs a) {
  const int lane = threadIdx.x & 31;
  const long long warp = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const long long nwarps = ((long long)gridDim.x * blockDim.x) >> 5;
  int per_row = 0;
  for (int r = 0; r < a.nreg; ++r) per_row += a.outer[r];
  const long long total = (long long)a.B * per_row;
  for (long long it = warp; it < total; it += nwarps) {
    const int b = (int)(it / per_row);
    int k = (int)(it - (long long)b * per_row);
    const int p = a.eff[b];
    const int n = a.len[b];
    if (p < 0 || p == b || n == 0) continue;
    int r = 0;
    while (k >= a.outer[r]) k -= a.outer[r++];
    const size_t eb = (size_t)a.entry_bytes[r];
    const size_t rb = (size_t)a.outer[r] * a.cap * eb;   // bytes of one row in region r
    const uint8_t *src = kToScratch ? a.ring[r] + (size_t)p * rb : a.scratch[r] + (size_t)b * rb;
    uint8_t *dst = kToScratch ? a.scratch[r] + (size_t)b * rb : a.ring[r] + (size_t)b * rb;
    const size_t ring0 = (size_t)k * a.cap * eb;          // this ring inside the row
    const int st = a.start[b];
    const int n1 = n < a.cap - st ? n : a.cap - st;       // entries before the wrap
    for (int seg = 0; seg < 2; ++seg) {
      const int e0 = seg ? 0 : st, cnt = seg ? n - n1 : n1;
      if (cnt <= 0) continue;
      const size_t off = ring0 + (size_t)e0 * eb, bytes = (size_t)cnt * eb;
      if (eb % 16 == 0) {
        const uint4 *s4 = reinterpret_cast<const uint4 *>(src + off);
        uint4 *d4 = reinterpret_cast<uint4 *>(dst + off);
        for (size_t w = lane; w < bytes / 16; w += 32) d4[w] = s4[w];
      } else {
        const uint32_t *s1 = reinterpret_cast<const uint32_t *>(src + off);
        uint32_t *d1 = reinterpret_cast<uint32_t *>(dst + off);
        for (size_t w = lane; w < bytes / 4; w += 32) d1[w] = s1[w];
      }
    }
  }
}

__global__ void restore_kernel(int B, const int32_t *keep, int32_t *len, const int32_t *pending,
                               uint32_t *status) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= B) return;
  const int k = keep[b];
  if (pending[b] != 0 || k < 0 || k > len[b]) {
    atomicOr(status, (unsigned)RSSM_STATUS_STATE);
    return;
  }
  len[b] = k;
}

__global__ void init_slots_kernel(int B, int32_t *slot, int32_t *dst) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= B) return;
  slot[b] = b;
  dst[b] = b;
}

__global__ void effective_slots_kernel(int B, const int32_t *slot, const int32_t *dst, const int32_t *seen,
                                       const int32_t *flushes, int32_t *out) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= B) return;
  out[b] = flushes[b] != seen[b] ? dst[b] : slot[b];
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

cudaError_t plan_slots(const StepArgs &a, int32_t *slot, int32_t *dst, int32_t *seen, int32_t *freelist,
                       cudaStream_t s) {
  plan_slots_kernel<<<1, 1024, 0, s>>>(a, slot, dst, seen, freelist);
  return cudaGetLastError();
}

cudaError_t branch_rows(const BranchArgs &b, const int32_t *parent, int32_t *tmp, cudaStream_t s) {
  branch_book_kernel<<<1, 1024, 0, s>>>(b, parent, tmp);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  branch_copy_kernel<true><<<dim3((unsigned)sms * 8), dim3(256), 0, s>>>(b);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  branch_copy_kernel<false><<<dim3((unsigned)sms * 8), dim3(256), 0, s>>>(b);
  return cudaGetLastError();
}

cudaError_t restore_rows(int B, const int32_t *keep, int32_t *len, const int32_t *pending,
                         uint32_t *status, cudaStream_t s) {
  restore_kernel<<<dim3((unsigned)((B + 255) / 256)), dim3(256), 0, s>>>(B, keep, len, pending, status);
  return cudaGetLastError();
}

cudaError_t init_slots(int B, int32_t *slot, int32_t *dst, cudaStream_t s) {
  init_slots_kernel<<<dim3((unsigned)((B + 255) / 256)), dim3(256), 0, s>>>(B, slot, dst);
  return cudaGetLastError();
}

cudaError_t effective_slots(int B, const int32_t *slot, const int32_t *dst, const int32_t *seen,
                            const int32_t *flushes, int32_t *out, cudaStream_t s) {
  effective_slots_kernel<<<dim3((unsigned)((B + 255) / 256)), dim3(256), 0, s>>>(B, slot, dst, seen, flushes,
                                                                                 out);
  return cudaGetLastError();
}

}  // namespace rssm
