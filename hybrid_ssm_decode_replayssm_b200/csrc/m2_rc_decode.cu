// Mamba-2 decode of layers whose reads come from a quantised copy of the
// checkpoint (FP8 row / NVFP4), one token, bf16 inputs, headdim 64, dstate 128.
//
// "ReplaySSM: Rethinking State Storage for Faster Hybrid-Model Decoding"
// (deskofai.com summary, paragraph 4): the recurrence stays in high precision
// while the reads between folds come from a low-precision copy, so a decode
// moves a quarter (FP8) or about a seventh (NVFP4 with its scales) of the
// fp32 checkpoint's bytes.  The replay form is that of mamba2.cu:
//   y_t = e^{G_t} h_c C_t + sum_{s<=t} e^{seg(s,t)} dt_s (B_s . C_t) x_s + D x_t
//   fold: h_c <- e^{G_l} h_c + sum_{s<=l} e^{seg(s,l)} dt_s x_s B_s^T,
// with h_c C_t read from the copy, and folds reading and writing the fp32
// checkpoint and quantising the new copy.
//
// A head's copy is only 4.5 KiB (NVFP4) or 8.25 KiB (FP8), too small a unit
// for a stage pipeline fed by one producer thread.  So this kernel has no
// producer and no waits: one CTA of 8 warps per (sequence, group, chunk of
// heads), several CTAs resident per SM, and each warp loads its own head's
// codes and scales straight into registers (requested before the CTA's
// shared prologue so that their latency hides behind it) and multiplies them
// with C on the tensor cores (mma.sync m16n8k16, f16 in, fp32 out).  The
// products are exact: a dequantised code is exact in f16 (an E2M1 value times
// an E4M3 block scale has at most 6 significant bits and lies in [2^-10, 2688];
// an E4M3 code is exact, its fp32 row scale is applied to the sum), and C is
// scaled by a power of two into [2^14, 2^15) before rounding to f16.  The CTA's prologue stages the window: B rows (fp32), C,
// the dt windows, B.C, the window scalars and every head's x rows, with the
// ring appends.  A row that folds this call does so on the CUDA cores, 4 state
// rows at a time (fp32 read, rank-l update, fp32 store, new copy); its outputs
// come from the copy as well: the old one when the window fills with this
// token, the new one when the token did not fit and the window was folded
// first.  At 64 registers a thread, four CTAs (32 warps) share an SM.
#include "m2_common.cuh"
#include "rssm_device.cuh"

namespace rssm {
namespace {

constexpr int RP = 64, RN = 128;          // headdim P, dstate N
constexpr int kRcWarps = 8;
constexpr int kRcThreads = kRcWarps * 32;
constexpr int kHS = 32 + 1 + 64 + 2;      // per head: output coefficients, decay, two fold weight rows, two fold decays
constexpr int kXRow = RP * 2;             // bytes of one bf16 x row

// Shared memory of one CTA, in floats (host and device agree): B rows [L+1][N],
// C [N], C as f16 [N/2] and 1/its scale [4], dt windows [hc][L+1], B.C [L+1],
// head scalars [hc][kHS] (folds), A [hc], then the x rows [hc][L+1][P] bf16 (16-byte aligned;
// entry i < n at row i, the new token at row L, as a stage of mamba2.cu).
struct RcSmem {
  int L, hc;
  __host__ __device__ int c_off() const { return (L + 1) * RN; }
  __host__ __device__ int ch_off() const { return c_off() + RN; }
  __host__ __device__ int dt_off() const { return ch_off() + RN / 2 + 4; }
  __host__ __device__ int bc_off() const { return dt_off() + hc * (L + 1); }
  __host__ __device__ int sc_off() const { return bc_off() + L + 1; }
  __host__ __device__ int a_off() const { return sc_off() + hc * kHS; }
  __host__ __device__ int x_off() const { return (a_off() + hc + 3) & ~3; }
  __host__ __device__ size_t bytes() const { return (size_t)x_off() * 4 + (size_t)hc * (L + 1) * kXRow; }
};

// The codes and scales a lane needs for one batch of m-tiles (16 rows each) of
// a head: NVFP4 two m-tiles, FP8 one (16 registers of codes either way, so that
// four CTAs fit on an SM).
template <int RF>
struct RcCodes {
  static constexpr int kTiles = RF == RSSM_READ_NVFP4 ? 2 : 1;
  static constexpr int kBatches = 4 / kTiles;
  uint4 q[8];
  uint32_t s[8];
};

// Lane (g8, t4) of the m16n8k16 layout takes rows ra = 16 mt + g8 and ra + 8:
// NVFP4 bytes [16 t4, 16 t4 + 16) of each row and the two E4M3 scales of those
// 32 elements; FP8 bytes [32 t4, 32 t4 + 32) and the fp32 row scales.
template <int RF>
__device__ __forceinline__ void load_batch(RcCodes<RF> &c, const uint8_t *codes, const void *scales, size_t row_base,
                                           int bi, int lane) {
  const int g8 = lane >> 2, t4 = lane & 3;
#pragma unroll
  for (int k = 0; k < RcCodes<RF>::kTiles; ++k) {
    const int ra = (bi * RcCodes<RF>::kTiles + k) * 16 + g8, rb = ra + 8;
    if constexpr (RF == RSSM_READ_NVFP4) {
      constexpr int RB = RN / 2;
      c.q[2 * k] = __ldcs(reinterpret_cast<const uint4 *>(codes + (size_t)ra * RB + 16 * t4));
      c.q[2 * k + 1] = __ldcs(reinterpret_cast<const uint4 *>(codes + (size_t)rb * RB + 16 * t4));
      const uint8_t *sc = reinterpret_cast<const uint8_t *>(scales);
      c.s[2 * k] = __ldcs(reinterpret_cast<const unsigned short *>(sc + (row_base + ra) * (RN / 16) + 2 * t4));
      c.s[2 * k + 1] = __ldcs(reinterpret_cast<const unsigned short *>(sc + (row_base + rb) * (RN / 16) + 2 * t4));
    } else {
      constexpr int RB = RN;
      c.q[4 * k] = __ldcs(reinterpret_cast<const uint4 *>(codes + (size_t)ra * RB + 32 * t4));
      c.q[4 * k + 1] = __ldcs(reinterpret_cast<const uint4 *>(codes + (size_t)ra * RB + 32 * t4 + 16));
      c.q[4 * k + 2] = __ldcs(reinterpret_cast<const uint4 *>(codes + (size_t)rb * RB + 32 * t4));
      c.q[4 * k + 3] = __ldcs(reinterpret_cast<const uint4 *>(codes + (size_t)rb * RB + 32 * t4 + 16));
      const float *sc = reinterpret_cast<const float *>(scales);
      c.s[2 * k] = __float_as_uint(__ldcs(sc + row_base + ra));
      c.s[2 * k + 1] = __float_as_uint(__ldcs(sc + row_base + rb));
    }
  }
}

// (copy . C) of row 16 mt + (lane & 15) for m-tile k of the batch (the scale of
// C not yet removed), from eight m16n8k16 steps; C sits in column 0 of B.
template <int RF>
__device__ __forceinline__ float tile_hc(const RcCodes<RF> &c, int k, const uint2 *cfrag, int lane) {
  float d[4] = {0.0f, 0.0f, 0.0f, 0.0f};
  uint32_t af[4];
  const bool holder = (lane >> 2) == 0;   // column 0 of B: lanes 0..3
  if constexpr (RF == RSSM_READ_NVFP4) {
    const uint32_t wa[4] = {c.q[2 * k].x, c.q[2 * k].y, c.q[2 * k].z, c.q[2 * k].w};
    const uint32_t wb[4] = {c.q[2 * k + 1].x, c.q[2 * k + 1].y, c.q[2 * k + 1].z, c.q[2 * k + 1].w};
    const __half2 sa = __half2(__nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(c.s[2 * k] & 0xFFFFu), __NV_E4M3));
    const __half2 sb = __half2(__nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(c.s[2 * k + 1] & 0xFFFFu), __NV_E4M3));
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {   // bytes 2 ks, 2 ks + 1 of the lane's 16; scale block 2 t4 + ks / 4
      const __half2 sca = ks < 4 ? __low2half2(sa) : __high2half2(sa);
      const __half2 scb = ks < 4 ? __low2half2(sb) : __high2half2(sb);
      const int sh = (ks & 1) * 16;
      af[0] = e2m1x2_scaled(wa[ks >> 1] >> sh, sca);
      af[1] = e2m1x2_scaled(wb[ks >> 1] >> sh, scb);
      af[2] = e2m1x2_scaled(wa[ks >> 1] >> (sh + 8), sca);
      af[3] = e2m1x2_scaled(wb[ks >> 1] >> (sh + 8), scb);
      const uint2 bv = holder ? cfrag[8 * (lane & 3) + ks] : make_uint2(0u, 0u);
      mma_16816(d, af, bv.x, bv.y);
    }
  } else {
    const uint32_t wa[8] = {c.q[4 * k].x, c.q[4 * k].y, c.q[4 * k].z, c.q[4 * k].w,
                            c.q[4 * k + 1].x, c.q[4 * k + 1].y, c.q[4 * k + 1].z, c.q[4 * k + 1].w};
    const uint32_t wb[8] = {c.q[4 * k + 2].x, c.q[4 * k + 2].y, c.q[4 * k + 2].z, c.q[4 * k + 2].w,
                            c.q[4 * k + 3].x, c.q[4 * k + 3].y, c.q[4 * k + 3].z, c.q[4 * k + 3].w};
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {   // bytes 4 ks .. 4 ks + 3 of the lane's 32
      af[0] = e4m3x2_h2(wa[ks]);
      af[1] = e4m3x2_h2(wb[ks]);
      af[2] = e4m3x2_h2(wa[ks] >> 16);
      af[3] = e4m3x2_h2(wb[ks] >> 16);
      const uint2 bv = holder ? cfrag[8 * (lane & 3) + ks] : make_uint2(0u, 0u);
      mma_16816(d, af, bv.x, bv.y);
    }
    d[0] *= __uint_as_float(c.s[2 * k]);
    d[2] *= __uint_as_float(c.s[2 * k + 1]);
  }
  // column 0 of row g (d[0]) and of row g + 8 (d[2]) sit in lane 4 g
  const int r16 = lane & 15;
  const float va = __shfl_sync(kFull, d[0], 4 * (r16 & 7));
  const float vb = __shfl_sync(kFull, d[2], 4 * (r16 & 7));
  return r16 < 8 ? va : vb;
}

template <int RF>
__global__ void __launch_bounds__(kRcThreads, 4) m2_rc_decode_kernel(const StepArgs a, const int hc) {
  using Tin = __nv_bfloat16;
  using T = Tile<RP, RN, 16>;   // the folds' 4-row groups: a lane holds 4 columns of 4 rows
  using Codes = RcCodes<RF>;
  constexpr int TB = tile_bytes<RF, RP, RN>();
  constexpr int RB = rc_row_bytes<RF, RN>();
  constexpr int kChunks = RN / 8;   // 16-byte chunks of a B row
  extern __shared__ __align__(16) float sm[];
  const RcSmem Y{a.L, hc};
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int L = a.L, cap = a.cap, WM = L + 1;
  const int nchunk = a.hpg / hc;
  const int item = (int)blockIdx.x;
  const int b = item / (a.G * nchunk), rem = item - b * (a.G * nchunk);
  const int g = rem / nchunk, chunk = rem - g * nchunk;
  const int h0 = g * a.hpg + chunk * hc;
  const size_t bh0 = (size_t)b * a.H + h0;

  // This warp's first head's codes are requested before anything waits: with
  // no slot indirection the copy's address needs only b (a row that folds this
  // call does not use them; they are 1/7 to 1/4 of its fp32 traffic).
  Codes cq;
  const bool early = a.slot == nullptr && warp < hc;
  if (early) load_batch<RF>(cq, a.rc_codes + (bh0 + warp) * TB, a.rc_scales, (bh0 + warp) * RP, 0, lane);
  const RowPlan rp = plan_row(a, b);
  if (rp.refuse) {
    if (rp.bit && g == 0 && chunk == 0 && tid == 0) atomicOr(a.status, rp.bit);
    return;
  }
  const int st = rp.st, n = rp.n;
  const bool pre = rp.pre, post = rp.post, fold = pre || post;
  const int w0 = pre ? n : 0;
  if (!early && !pre && warp < hc)
    load_batch<RF>(cq, a.rc_codes + ((size_t)rp.src * a.H + h0 + warp) * TB, a.rc_scales,
                   ((size_t)rp.src * a.H + h0 + warp) * RP, 0, lane);

  float *sB = sm, *sC = sm + Y.c_off(), *sdt = sm + Y.dt_off(), *sBC = sm + Y.bc_off(), *ssc = sm + Y.sc_off();
  __half *sCh = reinterpret_cast<__half *>(sm + Y.ch_off());
  float *sCinv = sm + Y.ch_off() + RN / 2;
  float *sA = sm + Y.a_off();
  uint8_t *sX = reinterpret_cast<uint8_t *>(sm + Y.x_off());
  const Tin *xin = reinterpret_cast<const Tin *>(a.in[0]);
  const Tin *Bin = reinterpret_cast<const Tin *>(a.in[1]);
  const Tin *Cin = reinterpret_cast<const Tin *>(a.in[2]);
  const Tin *dtin = reinterpret_cast<const Tin *>(a.in[3]);
  Tin *xring = reinterpret_cast<Tin *>(a.buf0);
  Tin *Bring = reinterpret_cast<Tin *>(a.buf1) + ((size_t)b * a.G + g) * cap * RN;
  const int slot_new = (st + n) % cap;

  // ---- staging, all loads issued before any store: committed x rows (async
  //      copies), the new x rows, B rows with their dot products with C, C
  //      itself (fp32, and f16 scaled for the tensor-core reads), dt windows, A
  for (int idx = tid; idx < hc * n * (RP / 8); idx += kRcThreads) {
    const int jh = idx / (n * (RP / 8)), r = idx - jh * (n * (RP / 8));
    const int i = r / (RP / 8), c = (r - i * (RP / 8)) * 8;
    cp_async16(sX + ((size_t)jh * WM + i) * kXRow + c * 2, xring + ((bh0 + jh) * cap + (st + i) % cap) * RP + c);
  }
  const int nxc = hc * (RP / 8);   // new x chunks (<= 128)
  uint4 xnew = make_uint4(0u, 0u, 0u, 0u);
  if (tid < nxc) xnew = __ldg(reinterpret_cast<const uint4 *>(xin + ((size_t)b * a.H + h0 + tid / 8) * RP + (tid % 8) * 8));
  const int cch = tid % kChunks;   // this thread's 8 columns of every B row it stages
  const uint4 craw = __ldg(reinterpret_cast<const uint4 *>(Cin + ((size_t)b * a.G + g) * RN + cch * 8));
  constexpr int kMaxB = (33 * kChunks + kRcThreads - 1) / kRcThreads;   // window <= 32
  const int nbc = (n + 1) * kChunks, bpass = (nbc + kRcThreads - 1) / kRcThreads;
  uint4 braw[kMaxB];
#pragma unroll
  for (int k = 0; k < kMaxB; ++k) {
    const int idx = tid + k * kRcThreads, i = idx / kChunks;
    braw[k] = make_uint4(0u, 0u, 0u, 0u);
    if (k < bpass && idx < nbc) {
      const Tin *src = i < n ? Bring + (size_t)((st + i) % cap) * RN + cch * 8 : Bin + ((size_t)b * a.G + g) * RN + cch * 8;
      braw[k] = __ldg(reinterpret_cast<const uint4 *>(src));
    }
  }
  const int ndt = hc * (n + 1), dpass = (ndt + kRcThreads - 1) / kRcThreads;
  float dtv[kMaxB + 1];
#pragma unroll
  for (int k = 0; k < kMaxB + 1; ++k) {
    const int idx = tid + k * kRcThreads;
    dtv[k] = 0.0f;
    if (k < dpass && idx < ndt) {
      const int jh = idx / (n + 1), i = idx - jh * (n + 1);
      dtv[k] = i < n ? a.buf2[(bh0 + jh) * cap + (st + i) % cap] : to_f32<Tin>(dtin[(size_t)b * a.H + h0 + jh]);
    }
  }
  if (tid < hc) sA[tid] = __ldg(a.A + h0 + tid);
  // -- stores
  if (tid < nxc) {
    const int jh = tid / 8, c = (tid % 8) * 8;
    *reinterpret_cast<uint4 *>(sX + ((size_t)jh * WM + L) * kXRow + c * 2) = xnew;
    *reinterpret_cast<uint4 *>(xring + ((bh0 + jh) * cap + slot_new) * RP + c) = xnew;
  }
  float cf[8];
  {
    const Tin *e = reinterpret_cast<const Tin *>(&craw);
#pragma unroll
    for (int q = 0; q < 8; ++q) cf[q] = to_f32<Tin>(e[q]);
  }
  if (tid < kChunks) {   // warp 0, lanes 0..15 hold C: fp32, and f16 scaled so that max |C| is in [2^14, 2^15)
#pragma unroll
    for (int q = 0; q < 8; ++q) sC[cch * 8 + q] = cf[q];
  }
  if (warp == 0) {
    float cm = 0.0f;
#pragma unroll
    for (int q = 0; q < 8; ++q) cm = fmaxf(cm, fabsf(cf[q]));
    cm = group_max<kChunks>(cm);   // lanes 16..31 hold the same chunks as 0..15
    const int e = cm > 0.0f ? 14 - ilogbf(cm) : 0;
    if (lane < kChunks) {
#pragma unroll
      for (int q = 0; q < 8; ++q) sCh[cch * 8 + q] = __float2half_rn(ldexpf(cf[q], e));
    }
    if (lane == 0) *sCinv = ldexpf(1.0f, -e);
  }
#pragma unroll
  for (int k = 0; k < kMaxB; ++k) {
    if (k < bpass) {   // uniform over the CTA: every lane takes part in the row reduction
      const int idx = tid + k * kRcThreads, i = idx / kChunks;
      const bool valid = idx < nbc;
      const Tin *e = reinterpret_cast<const Tin *>(&braw[k]);
      float dot = 0.0f;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const float v = to_f32<Tin>(e[q]);
        if (valid) sB[i * RN + cch * 8 + q] = v;
        dot = fmaf(v, cf[q], dot);
      }
#pragma unroll
      for (int o = kChunks / 2; o >= 1; o >>= 1) dot += __shfl_xor_sync(kFull, dot, o);
      if (valid && cch == 0) sBC[i] = dot;
      if (valid && i == n && chunk == 0) *reinterpret_cast<uint4 *>(Bring + (size_t)slot_new * RN + cch * 8) = braw[k];
    }
  }
#pragma unroll
  for (int k = 0; k < kMaxB + 1; ++k) {
    const int idx = tid + k * kRcThreads;
    if (k < dpass && idx < ndt) {
      const int jh = idx / (n + 1), i = idx - jh * (n + 1);
      sdt[jh * WM + i] = dtv[k];
      if (i == n) a.buf2[(bh0 + jh) * cap + slot_new] = dtv[k];
    }
  }
  cp_async_wait_all();
  __syncthreads();

  // Every CTA of sequence b has read its pointers once all of them have counted
  // in (this CTA's threads have: the barrier above), so the last to count in moves them.
  if (tid == 0 && atomicAdd(a.arrivals + b, 1) == a.G * nchunk - 1) {
    a.arrivals[b] = 0;
    int st2 = st, n2 = n, fl = a.flushes[b];
    if (pre) {
      st2 = (st + n) % cap;
      n2 = 0;
      ++fl;
    }
    n2 += 1;
    if (post) {
      st2 = (st2 + n2) % cap;
      n2 = 0;
      ++fl;
    }
    a.start[b] = st2;
    a.len[b] = n2;
    a.flushes[b] = fl;
  }

  // ---- heads: warp w takes heads w, w + 8, ...  The warp forms its head's
  //      window scalars itself: output coefficients e^{A seg(i, n)} dt_i (B_i . C)
  //      over [w0, n] and e^{A G}; fold weights e^{A seg(i, last)} dt_i and the
  //      decay of each folded window.  Segment sums are warp suffix sums of dt.
  const uint2 *cfrag = reinterpret_cast<const uint2 *>(sCh);   // C (f16): the B fragments, C[32 t4 + 4 ks .. + 3]
  const float cinv = *sCinv;
  for (int jh = warp; jh < hc; jh += kRcWarps) {
    const int h = h0 + jh;
    const size_t sbh = (size_t)rp.src * a.H + h, dbh = (size_t)rp.dst * a.H + h;
    const Stage stg{sX + (size_t)jh * WM * kXRow, 0, kXRow, n, L};
    const float Ah = sA[jh];
    const float Dh = __ldg(a.D + h);
    float *hs = ssc + jh * kHS;   // fold weights: [33, 65) the pre-fold, [65, 97) the window fold; decays 97, 98
    // output coefficients (lane i: entry w0 + i) and the decay from the checkpoint
    const int len = n - w0 + 1;
    float coef, dec;
    {
      const float v = lane < len ? sdt[jh * WM + w0 + lane] : 0.0f;
      float after, total;
      suffix_scan(v, lane, after, total);
      coef = lane < len ? expf(Ah * after) * v * sBC[w0 + lane] : 0.0f;
      dec = expf(Ah * total);
    }
    // fold weights e^{A seg(i, last)} dt_i of a folded window [i0, i0 + ne) and its decay
    auto fold_weights = [&](int q, int i0, int ne) {
      const float v = lane < ne ? sdt[jh * WM + i0 + lane] : 0.0f;
      float after, total;
      suffix_scan(v, lane, after, total);
      hs[33 + 32 * q + lane] = expf(Ah * after) * v;
      if (lane == 0) hs[97 + q] = expf(Ah * total);
      __syncwarp();
    };
    // fold entries [i0, i1) of the window into the fp32 checkpoint read at src,
    // store it and quantise the new copy, 4 rows at a time (a lane: 4 columns
    // of 4 rows)
    const int c0 = lane * 4;
    float *hc_dst = a.hc + dbh * RP * RN;
    uint8_t *rc_dst = a.rc_codes + dbh * TB;
    auto fold_rows = [&](const float *src, int i0, int i1, const float *fw, float fdec) {
#pragma unroll 1
      for (int vw = 0; vw < RP / T::RPW; ++vw) {
        const int row0 = vw * T::RPW;
        float4 f[T::NLD];
#pragma unroll
        for (int l = 0; l < T::NLD; ++l) f[l] = ld_stream(src + (size_t)(row0 + l) * RN + c0);
        fold_tile<RP, RN, 16, Tin>(f, fw, fdec, i0, i1, stg, sB, row0, c0);
#pragma unroll
        for (int l = 0; l < T::NLD; ++l) {
          const int row = row0 + l;
          st_stream(hc_dst + (size_t)row * RN + c0, f[l]);
          quantize4<RF, T::LPR>(f[l], rc_dst + (size_t)row * RB, a.rc_scales, dbh * RP + row, RN, c0, lane);
        }
      }
    };
    size_t cbh = sbh;   // the copy the outputs read
    if (pre) {
      // the token does not fit: fold the committed window first; the outputs
      // then read the copy this writes (the warp's own stores: fence, then sync)
      fold_weights(0, 0, n);
      fold_rows(a.hc + sbh * RP * RN, 0, n, hs + 33, hs[97]);
      __threadfence_block();
      __syncwarp();
      cbh = dbh;
      load_batch<RF>(cq, a.rc_codes + cbh * TB, a.rc_scales, cbh * RP, 0, lane);
    } else if (post && jh != warp) {   // after a fold the next head's codes are requested at its start
      load_batch<RF>(cq, a.rc_codes + cbh * TB, a.rc_scales, cbh * RP, 0, lane);
    }
    // ---- outputs: window terms of rows lane and lane + 32 (while the codes'
    //      loads are in flight), then the tensor-core read of the copy, batch by
    //      batch (NVFP4: two batches of two 16-row m-tiles; FP8: four of one);
    //      the next batch, or without a fold the next head's first, is requested
    //      as soon as this one's codes are used
    float ws[2] = {0.0f, 0.0f};
    for (int i = 0; i < len; ++i) {
      const float ci = __shfl_sync(kFull, coef, i);
#pragma unroll
      for (int q = 0; q < 2; ++q) ws[q] = fmaf(ci, stg.x<Tin>(w0 + i, lane + 32 * q), ws[q]);
    }
#pragma unroll
    for (int bi = 0; bi < Codes::kBatches; ++bi) {   // cq holds batch bi of this head's copy
      float hcv[Codes::kTiles];
#pragma unroll
      for (int k = 0; k < Codes::kTiles; ++k) hcv[k] = tile_hc<RF>(cq, k, cfrag, lane);
      if (bi + 1 < Codes::kBatches) {
        load_batch<RF>(cq, a.rc_codes + cbh * TB, a.rc_scales, cbh * RP, bi + 1, lane);
      } else if (!fold && jh + kRcWarps < hc) {
        const size_t nbh = sbh + kRcWarps;
        load_batch<RF>(cq, a.rc_codes + nbh * TB, a.rc_scales, nbh * RP, 0, lane);
      }
      if constexpr (Codes::kTiles == 2) {   // rows 32 bi + lane: m-tile 2 bi + (lane >= 16)
        const int row = 32 * bi + lane;
        const float hcr = lane < 16 ? hcv[0] : hcv[1];
        a.out[((size_t)b * a.H + h) * RP + row] = fmaf(Dh, stg.x<Tin>(n, row), fmaf(dec, hcr * cinv, ws[bi]));
      } else {   // rows 16 bi + (lane & 15), written by lanes 0..15
        const int row = 16 * bi + (lane & 15);
        const float wsr = __shfl_sync(kFull, ws[bi >> 1], row & 31);
        if (lane < 16)
          a.out[((size_t)b * a.H + h) * RP + row] = fmaf(Dh, stg.x<Tin>(n, row), fmaf(dec, hcv[0] * cinv, wsr));
      }
    }
    if (post) {   // the window is full: fold it (after a pre-fold, on top of what that stored)
      fold_weights(1, w0, n - w0 + 1);
      fold_rows(pre ? hc_dst : a.hc + sbh * RP * RN, w0, n + 1, hs + 65, hs[98]);
    }
  }
}

int rc_heads_per_cta(int hpg) {
  int hc = hpg < 16 ? hpg : 16;
  while (hpg % hc) --hc;
  return hc;
}

template <int RF>
cudaError_t launch_rc(const StepArgs &a, cudaStream_t s) {
  auto kern = m2_rc_decode_kernel<RF>;
  const int hc = rc_heads_per_cta(a.hpg);
  const size_t smem = RcSmem{a.L, hc}.bytes();
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const long long items = (long long)a.B * a.G * (a.hpg / hc);
  kern<<<dim3((unsigned)items), dim3(kRcThreads), smem, s>>>(a, hc);
  return cudaGetLastError();
}

}  // namespace

bool m2_rc_decode_path(const StepArgs &a, int in_dtype, int read_fmt) {
  return a.mode == kDecode && a.m == 1 && in_dtype == RSSM_BF16 && read_fmt != RSSM_READ_FP32 && a.R == RP &&
         a.C == RN;
}

cudaError_t m2_rc_decode_step(const StepArgs &a, int read_fmt, cudaStream_t s) {
  return read_fmt == RSSM_READ_FP8_E4M3_ROW ? launch_rc<RSSM_READ_FP8_E4M3_ROW>(a, s) : launch_rc<RSSM_READ_NVFP4>(a, s);
}

}  // namespace rssm
