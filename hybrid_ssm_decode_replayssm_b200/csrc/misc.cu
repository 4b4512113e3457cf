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

// rssm_branch, two launches of one 1024-thread block per sequence.
//
// Pass 1 (gather): block b decides its sequence's effective parent (eff =
// parent, or -1 when refused), gathers the parent's checkpoint slot (taking a
// fold of the previous launch into account) and pointers into tmp [4][B], and
// copies the live window entries of the parent's rings into b's scratch rows.
// Nothing that pass reads is written in it.
// Pass 2 (scatter): block b writes the gathered pointers (or, for a sequence
// that keeps its own state, adopts its last fold's slot) and copies its
// scratch rows into its rings.  A sequence that is both parent and child is
// read in pass 1 before pass 2 overwrites it.
//
// A ring region is [B][outer][cap][entry]; the live entries of each ring are
// (start + e) % cap, e < len.  A block walks all live words of its sequence
// (16-byte words where the entry size allows, else 4-byte words) with flat
// indices, four independent loads in flight per thread before their stores.
template <typename W>
__device__ __forceinline__ void copy_live_words(const uint8_t *__restrict__ src, uint8_t *__restrict__ dst,
                                                int outer, int cap, int ew, int n, int st) {
  const W *s = reinterpret_cast<const W *>(src);
  W *d = reinterpret_cast<W *>(dst);
  const int per_ring = n * ew;
  const int total = outer * per_ring;
  auto word = [&](int w) -> size_t {   // flat live-word index -> word offset in the row
    const int o = w / per_ring, rem = w - o * per_ring;
    const int e = rem / ew, c = rem - e * ew;
    int idx = st + e;
    if (idx >= cap) idx -= cap;
    return ((size_t)o * cap + idx) * ew + c;
  };
  const int bd = blockDim.x;
  for (int w0 = threadIdx.x; w0 < total; w0 += 4 * bd) {
    size_t off[4];
    W v[4];
#pragma unroll
    for (int q = 0; q < 4; ++q)
      if (w0 + q * bd < total) {
        off[q] = word(w0 + q * bd);
        v[q] = s[off[q]];
      }
#pragma unroll
    for (int q = 0; q < 4; ++q)
      if (w0 + q * bd < total) d[off[q]] = v[q];
  }
}

__device__ __forceinline__ void copy_row(const BranchArgs &a, const uint8_t *const *src_base, size_t src_row,
                                         uint8_t *const *dst_base, size_t dst_row, int n, int st) {
  for (int r = 0; r < a.nreg; ++r) {
    const int eb = a.entry_bytes[r];
    const size_t rb = (size_t)a.outer[r] * a.cap * eb;   // one sequence's row in region r
    const uint8_t *src = src_base[r] + src_row * rb;
    uint8_t *dst = dst_base[r] + dst_row * rb;
    if (eb % 16 == 0) copy_live_words<uint4>(src, dst, a.outer[r], a.cap, eb / 16, n, st);
    else copy_live_words<uint32_t>(src, dst, a.outer[r], a.cap, eb / 4, n, st);
  }
}

__global__ void __launch_bounds__(1024) branch_gather_kernel(const BranchArgs a, const int32_t *parent,
                                                             int32_t *tmp) {
  const int B = a.B, b = blockIdx.x;
  const int p = parent[b];
  const bool ok = p >= 0 && p < B && a.pending[p] == 0;
  if (threadIdx.x == 0) {
    a.eff[b] = ok ? p : -1;
    if (!ok) atomicOr(a.status, (unsigned)RSSM_STATUS_STATE);
    if (ok && p != b) {
      const int f = a.flushes[p];
      tmp[b] = f != a.seen[p] ? a.dst[p] : a.slot[p];
      tmp[B + b] = a.start[p];
      tmp[2 * B + b] = a.len[p];
      tmp[3 * B + b] = f;
    }
  }
  if (!ok || p == b) return;
  const int n = a.len[p];
  if (n > 0) copy_row(a, a.ring, (size_t)p, a.scratch, (size_t)b, n, a.start[p]);
}

__global__ void __launch_bounds__(1024) branch_scatter_kernel(const BranchArgs a, const int32_t *tmp) {
  const int B = a.B, b = blockIdx.x;
  const int p = a.eff[b];
  const bool moved = p >= 0 && p != b;
  if (threadIdx.x == 0) {
    if (moved) {
      a.slot[b] = tmp[b];
      a.start[b] = tmp[B + b];
      a.len[b] = tmp[2 * B + b];
      a.flushes[b] = tmp[3 * B + b];
      a.seen[b] = tmp[3 * B + b];
      a.pending[b] = 0;
    } else {
      const int f = a.flushes[b];
      if (f != a.seen[b]) {   // this sequence's own fold of the previous launch
        a.slot[b] = a.dst[b];
        a.seen[b] = f;
      }
    }
  }
  if (!moved) return;
  const int n = tmp[2 * B + b];
  if (n > 0) copy_row(a, a.scratch, (size_t)b, a.ring, (size_t)b, n, tmp[B + b]);
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
  branch_gather_kernel<<<dim3((unsigned)b.B), dim3(1024), 0, s>>>(b, parent, tmp);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  branch_scatter_kernel<<<dim3((unsigned)b.B), dim3(1024), 0, s>>>(b, tmp);
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
