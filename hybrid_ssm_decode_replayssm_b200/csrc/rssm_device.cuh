// Device helpers shared by the librssm kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp4.h>
#include <cuda_fp8.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "rssm_internal.h"

namespace rssm {

constexpr unsigned kFull = 0xffffffffu;

// ------------------------------------------------------------ row plan
// What one call does to sequence b, decided from its pointers alone (the
// window rules of rssm.h): refuse the row (with a status bit), fold the
// committed window before appending (pre), fold the full window after the
// decode (post).  src / dst: the checkpoint slot the row reads, and the one a
// fold of this call writes (both b unless the layer branches).
struct RowPlan {
  int st, n, src, dst;
  bool refuse, pre, post;
  unsigned bit;
};
// The pointers a plan is made from, loaded apart from their use so that a
// warp can request the next item's while it works on the current one (they
// cannot move before this CTA's own part of that sequence is done).
struct RowRaw {
  int st, n, src, dst, pend, mask;
};
__device__ __forceinline__ RowRaw load_row(const StepArgs &a, int b) {
  RowRaw w;
  w.st = a.start[b];
  w.n = a.len[b];
  w.src = a.slot ? a.slot[b] : b;
  w.dst = a.dst ? a.dst[b] : b;
  w.pend = a.pending[b];
  w.mask = a.mask ? a.mask[b] : 1;
  return w;
}
__device__ __forceinline__ RowPlan plan_from(const StepArgs &a, const RowRaw &w) {
  RowPlan r;
  r.st = w.st;
  r.n = w.n;
  r.src = w.src;
  r.dst = w.dst;
  const int pend = w.pend;
  r.refuse = r.pre = r.post = false;
  r.bit = 0;
  if (a.mode == kFlush) {
    if (w.mask == 0) r.refuse = true;
    else if (pend != 0) { r.refuse = true; r.bit = RSSM_STATUS_STATE; }
    else if (r.n == 0) r.refuse = true;
    else r.pre = true;
  } else if (pend != 0) {
    r.refuse = true;
    r.bit = RSSM_STATUS_STATE;
  } else {
    r.pre = r.n + a.m > a.L;
    if (r.pre && !a.auto_flush) {
      r.refuse = true;
      r.bit = RSSM_STATUS_CAPACITY;
    }
    r.post = !r.refuse && a.mode == kDecode && a.auto_flush && ((r.pre ? 0 : r.n) + 1 == a.L);
  }
  return r;
}
__device__ __forceinline__ RowPlan plan_row(const StepArgs &a, int b) { return plan_from(a, load_row(a, b)); }

// ---------------------------------------------------------------- loads
// The checkpoint is streamed once per call: keep it out of L1 and mark it
// evict-first in L2 so the window buffers (re-read every step) stay cached.
__device__ __forceinline__ float4 ld_stream(const float *p) {
  return __ldcs(reinterpret_cast<const float4 *>(p));
}
__device__ __forceinline__ void st_stream(float *p, float4 v) {
  __stcs(reinterpret_cast<float4 *>(p), v);
}

template <typename T> __device__ __forceinline__ float to_f32(T v);
template <> __device__ __forceinline__ float to_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 v) {
  return __bfloat162float(v);
}

// Copy `n` elements (n % 8 == 0, 16-byte aligned source) of type T from global
// memory into fp32 shared memory, using the threads [t0, t0 + nt).
template <typename T>
__device__ __forceinline__ void stage_row(float *dst, const T *src, int n, int t, int nt) {
  constexpr int kPer = 16 / sizeof(T);
  for (int i = t; i < n / kPer; i += nt) {
    uint4 raw = __ldg(reinterpret_cast<const uint4 *>(src) + i);
    const T *e = reinterpret_cast<const T *>(&raw);
#pragma unroll
    for (int c = 0; c < kPer; ++c) dst[i * kPer + c] = to_f32<T>(e[c]);
  }
}

// Copy n elements of T (n % 8 == 0) global -> global (ring-buffer append).
template <typename T>
__device__ __forceinline__ void copy_row(T *dst, const T *src, int n, int t, int nt) {
  constexpr int kPer = 16 / sizeof(T);
  for (int i = t; i < n / kPer; i += nt)
    reinterpret_cast<uint4 *>(dst)[i] = __ldg(reinterpret_cast<const uint4 *>(src) + i);
}

// ------------------------------------------------------ warp reductions
// Transposed reduction.  Each lane holds NV partial sums v[0..NV); lanes are
// grouped in aligned groups of W consecutive lanes that must be summed.  At
// every level the pair of lanes (lane, lane ^ O) trades half of its values so
// the number of live values halves; once one value is left the remaining
// levels are plain butterflies.  On return the lane's live values v[0..R),
// R = max(1, NV / W), are complete sums of the original indices
// tr_base<NV, W/2>(lane) + i.  NV and W are powers of two.
template <int NV, int O>
__device__ __forceinline__ void tr_sum(float *v, int lane) {
  if constexpr (O >= 1) {
    if constexpr (NV > 1) {
      constexpr int H = NV / 2;
      const bool up = (lane & O) != 0;
#pragma unroll
      for (int i = 0; i < H; ++i) {
        const float keep = up ? v[i + H] : v[i];
        const float send = up ? v[i] : v[i + H];
        v[i] = keep + __shfl_xor_sync(kFull, send, O);
      }
      tr_sum<H, O / 2>(v, lane);
    } else {
      v[0] += __shfl_xor_sync(kFull, v[0], O);
      tr_sum<1, O / 2>(v, lane);
    }
  }
}

template <int NV, int O>
__device__ __forceinline__ int tr_base(int lane) {
  if constexpr (O >= 1 && NV > 1) {
    return ((lane & O) ? NV / 2 : 0) + tr_base<NV / 2, O / 2>(lane);
  } else {
    return 0;
  }
}

// Suffix sums over a warp: lanes l < len hold v (the others 0).  Returns in
// `after` the sum of v over lanes l' > l (direct sums of the terms, no
// differences of prefix sums) and in `total` the sum over all lanes.
__device__ __forceinline__ void suffix_scan(float v, int lane, float &after, float &total) {
  float incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const float t = __shfl_down_sync(kFull, incl, o);
    if (lane + o < 32) incl += t;
  }
  after = __shfl_down_sync(kFull, incl, 1);
  if (lane == 31) after = 0.0f;
  total = __shfl_sync(kFull, incl, 0);
}

// Max over aligned groups of W lanes (all lanes get the result).
template <int W>
__device__ __forceinline__ float group_max(float v) {
#pragma unroll
  for (int o = W / 2; o >= 1; o >>= 1) v = fmaxf(v, __shfl_xor_sync(kFull, v, o));
  return v;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
  return v;
}

// ---------------------------------------------------------- read-copy codecs
// OCP E4M3 (satfinite, round to nearest even) and FP4 E2M1 via CUDA's
// conversion functions; the divisions that feed them are IEEE fp32 divisions.
__device__ __forceinline__ uint32_t enc_e4m3(float x) {
  return (uint32_t)__nv_cvt_float_to_fp8(x, __NV_SATFINITE, __NV_E4M3);
}
__device__ __forceinline__ float dec_e4m3(uint32_t c) {
  __half_raw r = __nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)c, __NV_E4M3);
  return __half2float(__half(r));
}
__device__ __forceinline__ uint32_t enc_e2m1(float x) {
  return (uint32_t)__nv_cvt_float_to_fp4(x, __NV_E2M1, cudaRoundNearest) & 0xFu;
}
__device__ __forceinline__ float dec_e2m1(uint32_t c) {
  __half_raw r = __nv_cvt_fp4_to_halfraw((__nv_fp4_storage_t)c, __NV_E2M1);
  return __half2float(__half(r));
}
// Four E4M3 codes packed little-endian in w -> fp32.
__device__ __forceinline__ void dec_e4m3x4(uint32_t w, float s, float4 &o) {
  __half2_raw lo = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(w & 0xFFFFu), __NV_E4M3);
  __half2_raw hi = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(w >> 16), __NV_E4M3);
  float2 a = __half22float2(__half2(lo)), b = __half22float2(__half2(hi));
  o = make_float4(a.x * s, a.y * s, b.x * s, b.y * s);
}
// Four E2M1 codes packed in 16 bits (element 0 in the lowest nibble) -> fp32.
__device__ __forceinline__ void dec_e2m1x4(uint32_t w, float s, float4 &o) {
  __half2_raw lo = __nv_cvt_fp4x2_to_halfraw2((__nv_fp4x2_storage_t)(w & 0xFFu), __NV_E2M1);
  __half2_raw hi = __nv_cvt_fp4x2_to_halfraw2((__nv_fp4x2_storage_t)((w >> 8) & 0xFFu), __NV_E2M1);
  float2 a = __half22float2(__half2(lo)), b = __half22float2(__half2(hi));
  o = make_float4(a.x * s, a.y * s, b.x * s, b.y * s);
}

__device__ __forceinline__ float f4get(const float4 &v, int c) {
  return c == 0 ? v.x : c == 1 ? v.y : c == 2 ? v.z : v.w;
}

// Quantise the 4 elements a lane holds of one state row (columns c0..c0+3) into
// the read copy, and return the dequantised values the reads will see.
//   FP8 row:  lanes of the row (a group of LPR lanes) share one fp32 scale.
//   NVFP4:    groups of 4 lanes (16 elements) share one E4M3 scale.
template <int RF, int LPR>
__device__ __forceinline__ float4 quantize4(const float4 v, uint8_t *codes_row, void *scales,
                                            size_t row, int ncols, int c0, int lane) {
  float4 out;
  if constexpr (RF == RSSM_READ_FP8_E4M3_ROW) {
    float am = fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w)));
    am = group_max<LPR>(am);
    const float s = am / 448.0f;
    uint32_t w = 0;
    if (s != 0.0f) {
      w = enc_e4m3(v.x / s) | (enc_e4m3(v.y / s) << 8) | (enc_e4m3(v.z / s) << 16) |
          (enc_e4m3(v.w / s) << 24);
    }
    *reinterpret_cast<uint32_t *>(codes_row + c0) = w;
    if ((lane % LPR) == 0) reinterpret_cast<float *>(scales)[row] = s;
    dec_e4m3x4(w, s, out);
  } else {
    float am = fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w)));
    am = group_max<4>(am);
    const uint32_t sc = enc_e4m3(am / 6.0f);
    const float sv = dec_e4m3(sc);
    uint32_t w = 0;
    if (sv != 0.0f) {
      w = enc_e2m1(v.x / sv) | (enc_e2m1(v.y / sv) << 4) | (enc_e2m1(v.z / sv) << 8) |
          (enc_e2m1(v.w / sv) << 12);
    }
    *reinterpret_cast<uint16_t *>(codes_row + c0 / 2) = (uint16_t)w;
    if ((c0 % 16) == 0)
      reinterpret_cast<uint8_t *>(scales)[row * (ncols / 16) + c0 / 16] = (uint8_t)sc;
    dec_e2m1x4(w, sv, out);
  }
  return out;
}

// Load the 4 read-copy elements of (row, c0..c0+3) and dequantise them.
template <int RF>
__device__ __forceinline__ float4 load_read_copy4(const uint8_t *codes_row, const void *scales,
                                                  size_t row, int ncols, int c0) {
  float4 out;
  if constexpr (RF == RSSM_READ_FP8_E4M3_ROW) {
    const uint32_t w = __ldcs(reinterpret_cast<const unsigned int *>(codes_row + c0));
    const float s = __ldg(reinterpret_cast<const float *>(scales) + row);
    dec_e4m3x4(w, s, out);
  } else {
    const uint32_t w = __ldcs(reinterpret_cast<const unsigned short *>(codes_row + c0 / 2));
    const uint32_t sc = __ldg(reinterpret_cast<const uint8_t *>(scales) + row * (ncols / 16) + c0 / 16);
    dec_e2m1x4(w, dec_e4m3(sc), out);
  }
  return out;
}

// ------------------------------------------------- TMA bulk copies + mbarrier
// 1-D bulk copies (cp.async.bulk, no tensor map, no multicast) from global to
// this CTA's shared memory, completing on an mbarrier with a transaction count.
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_fence_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
// Add `bytes` to the current phase's expected transaction count (no arrival).
__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.expect_tx.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}
// Add `bytes` to the expected transaction count, then arrive (count 1).
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.b32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Non-blocking test of a phase (mbarrier.try_wait may suspend the thread for
// a while; a thread that polls several barriers must not be held on one).
__device__ __forceinline__ bool mbar_test_wait(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.b32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
// Wait for the phase with the given parity; give up after ~`limit` clock cycles
// (about a second) or as soon as *abort is set, returning false, so that a copy
// that never lands cannot hang the GPU.  A timeout sets *abort.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, uint32_t parity,
                                                  volatile int *abort = nullptr,
                                                  long long limit = 2000000000LL) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (abort && *abort) return false;
    if (clock64() - t0 > limit) {
      if (abort) *abort = 1;
      return false;
    }
  }
  return true;
}
// Combine a per-lane wait result across the warp: every lane of the warp waits
// on its own, and the warp goes on only if all of them succeeded, so a wait
// that gives up in some lanes (an abort seen at slightly different times)
// cannot split the warp before its collective operations (shuffles, named
// barriers, tcgen05 loads).  Call with all 32 lanes.
__device__ __forceinline__ bool warp_all(bool v) { return __all_sync(0xffffffffu, v); }

// Spin (bounded, abort-aware) until the shared int *flag reaches `value`.
__device__ __forceinline__ bool wait_flag_at_least(const int *flag, int value, volatile int *abort,
                                                   long long limit = 2000000000LL) {
  const volatile int *f = flag;
  if (*f >= value) return true;
  const long long t0 = clock64();
  while (*f < value) {
    if (*abort) return false;
    if (clock64() - t0 > limit) {
      *abort = 1;
      return false;
    }
    __nanosleep(64);
  }
  return true;
}

// The timeout self-test: wait (bounded) for a shared flag that nothing sets.
// Sets *abort and returns once the limit runs out, like any other wait.
__device__ __forceinline__ void stall_on_unset_flag(const int *never_set, volatile int *abort, long long limit) {
  wait_flag_at_least(never_set, 1, abort, limit);
}

// Asynchronous 16-byte global -> shared copies (cp.async, L1 bypassed): issued
// without holding registers; a thread's copies are complete after
// cp_async_wait_all(), and visible to the other threads after a barrier.
__device__ __forceinline__ void cp_async16(void *dst_smem, const void *src_gmem) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst_smem)), "l"(src_gmem) : "memory");
}
__device__ __forceinline__ void cp_async4(void *dst_smem, const void *src_gmem) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(dst_smem)), "l"(src_gmem) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}

// Named barrier `id` (1..15) over `n` threads (a group of consumer warps of a
// warp-specialised CTA), optionally OR-reducing a predicate.
__device__ __forceinline__ void named_sync(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}
__device__ __forceinline__ bool named_sync_or(int id, int n, bool p) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred pi, po;\n\t"
      "setp.ne.u32 pi, %1, 0;\n\t"
      "bar.red.or.pred po, %2, %3, pi;\n\t"
      "selp.u32 %0, 1, 0, po;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)p), "r"(id), "r"(n)
      : "memory");
  return r != 0;
}
__device__ __forceinline__ void bulk_g2s(void *dst_smem, const void *src_gmem, uint32_t bytes,
                                         uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
      ::"r"(smem_u32(dst_smem)), "l"(src_gmem), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}
// The same copy with an L2 eviction-priority hint (a createpolicy value): the
// checkpoint is streamed once per call, so its lines are marked evict-first and
// the small window rows re-read every step stay in L2.
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ void bulk_g2s_hint(void *dst_smem, const void *src_gmem, uint32_t bytes, uint64_t *bar,
                                              uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;"
      ::"r"(smem_u32(dst_smem)), "l"(src_gmem), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}
__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Arrival counter: returns true in exactly one thread (thread 0 of the last of
// `expected` CTAs to arrive for this counter).  Call after __syncthreads().
__device__ __forceinline__ bool last_arrival(int32_t *counter, int expected) {
  bool last = false;
  if (threadIdx.x == 0) {
    __threadfence();
    last = atomicAdd(counter, 1) == expected - 1;
    if (last) *counter = 0;
  }
  return last;
}

}  // namespace rssm
