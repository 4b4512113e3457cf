// Mamba-2 kernels: ReplaySSM replay step (decode / verify / flush) and the
// conventional per-token update used as the in-run baseline.
//
// Replay form (unrolled Mamba-2 SSD recurrence over the window, with
// a_r = dt_r A_h, seg(s,t) = sum_{s<r<=t} a_r, G_t = seg(w0-1, t)):
//   y_t = e^{G_t} h_c C_t + sum_{s<=t} e^{seg(s,t)} dt_s (B_s . C_t) x_s + D x_t
//   fold: h_c <- e^{G_l} h_c + sum_{s<=l} e^{seg(s,l)} dt_s x_s B_s^T
// "ReplaySSM: Rethinking State Storage for Faster Hybrid-Model Decoding"
// (deskofai.com summary, paragraphs 2-4): outputs are computed from the
// checkpoint and the buffered inputs without writing the state; the buffer is
// folded in when it fills; drafts are appended and rolled back by pointer; a
// low-precision copy of the checkpoint may serve the reads.
//
// One CTA owns one (sequence b, head h): its checkpoint tile [P, N] fp32 is
// streamed from HBM into registers with 128-bit loads (8 warps; a warp covers
// P/8 rows, a lane 4 consecutive columns of a row), the window's x / B / dt and
// the new tokens' C are staged in shared memory, and row dot products use a
// transposed warp reduction.  The tile is written back only when the row is
// folded (window full, or the new tokens would not fit).
#include <algorithm>

#include "rssm_device.cuh"

namespace rssm {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

template <int P, int N>
struct Tile {
  static constexpr int LPR = N / 4;     // lanes per state row
  static constexpr int RPI = 32 / LPR;  // rows covered by one warp instruction
  static constexpr int RPW = P / kWarps;
  static constexpr int NLD = RPW / RPI; // float4 per lane
  static_assert(N == 64 || N == 128, "dstate 64 or 128");
  static_assert(RPW % RPI == 0, "headdim must cover whole warp instructions");
};

template <int RF, int N>
constexpr int rc_row_bytes() { return RF == RSSM_READ_NVFP4 ? N / 2 : N; }

// t <- dec * t + sum_{i0 <= i < i1} fw[i] x_i[row] B_i[cols]   (rank-(i1-i0) fold)
template <int P, int N>
__device__ __forceinline__ void fold_tile(float4 (&t)[Tile<P, N>::NLD], const float *s_fw, float dec,
                                          int i0, int i1, const float *s_x, const float *s_B,
                                          int row0, int c0) {
  using T = Tile<P, N>;
#pragma unroll
  for (int l = 0; l < T::NLD; ++l) {
    t[l].x *= dec; t[l].y *= dec; t[l].z *= dec; t[l].w *= dec;
  }
  for (int i = i0; i < i1; ++i) {
    const float4 bv = *reinterpret_cast<const float4 *>(s_B + i * N + c0);
    const float fw = s_fw[i];
#pragma unroll
    for (int l = 0; l < T::NLD; ++l) {
      const float xr = fw * s_x[i * P + row0 + l * T::RPI];
      t[l].x = fmaf(xr, bv.x, t[l].x);
      t[l].y = fmaf(xr, bv.y, t[l].y);
      t[l].z = fmaf(xr, bv.z, t[l].z);
      t[l].w = fmaf(xr, bv.w, t[l].w);
    }
  }
}

// Outputs y_j for the m new tokens from the read view `v` (registers).
template <int P, int N, int MAXM>
__device__ __forceinline__ void outputs(const float4 (&v)[Tile<P, N>::NLD], const StepArgs &a,
                                        const float *s_C, const float *s_x, const float *s_coef,
                                        const float *s_dec, int b, int h, int n, int w0,
                                        int warp, int lane, int c0) {
  using T = Tile<P, N>;
  constexpr int NV = T::NLD * MAXM;
  float part[NV];
#pragma unroll
  for (int j = 0; j < MAXM; ++j) {
    const float4 cv = *reinterpret_cast<const float4 *>(s_C + j * N + c0);
#pragma unroll
    for (int l = 0; l < T::NLD; ++l)
      part[l * MAXM + j] = v[l].x * cv.x + v[l].y * cv.y + v[l].z * cv.z + v[l].w * cv.w;
  }
  tr_sum<NV, T::LPR / 2>(part, lane);
  const int base = tr_base<NV, T::LPR / 2>(lane);
  constexpr int R = NV >= T::LPR ? NV / T::LPR : 1;
  const bool writer = NV >= T::LPR || (lane & (T::LPR / NV - 1)) == 0;
  const float Dh = __ldg(a.D + h);
  const int cap = a.cap;
#pragma unroll
  for (int q = 0; q < R; ++q) {
    const int idx = base + q, l = idx / MAXM, j = idx % MAXM;
    if (writer && j < a.m) {
      const int row = warp * T::RPW + l * T::RPI + lane / T::LPR;
      const int e = n + j;
      float y = s_dec[j] * part[q];
      for (int i = w0; i <= e; ++i) y = fmaf(s_coef[j * cap + i], s_x[i * P + row], y);
      y = fmaf(Dh, s_x[e * P + row], y);
      a.out[(((size_t)b * a.m + j) * a.H + h) * P + row] = y;
    }
  }
}

template <int P, int N, typename Tin, int RF, int MAXM>
__global__ void __launch_bounds__(kThreads) m2_step_kernel(const StepArgs a) {
  using T = Tile<P, N>;
  extern __shared__ float4 smem4[];
  float *smem = reinterpret_cast<float *>(smem4);
  const int cap = a.cap;
  float *s_x = smem;                     // [cap][P]   window x (fp32)
  float *s_B = s_x + cap * P;            // [cap][N]   window B
  float *s_C = s_B + cap * N;            // [MAXM][N]  new tokens' C
  float *s_dt = s_C + MAXM * N;          // [cap]
  float *s_a = s_dt + cap;               // [cap]      dt * A
  float *s_bc = s_a + cap;               // [MAXM][cap] B_i . C_j
  float *s_coef = s_bc + MAXM * cap;     // [MAXM][cap] window coefficients
  float *s_fwpre = s_coef + MAXM * cap;  // [cap]      fold weights (pre-fold)
  float *s_fwpost = s_fwpre + cap;       // [cap]      fold weights (window-full fold)
  float *s_dec = s_fwpost + cap;         // [MAXM + 2] decays: outputs, pre, post
  __shared__ int s_book[3];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int b = blockIdx.x / a.H, h = blockIdx.x - b * a.H, g = h / a.hpg;
  if (tid == 0) {
    s_book[0] = a.start[b];
    s_book[1] = a.len[b];
    s_book[2] = a.pending[b];
  }
  __syncthreads();
  const int st = s_book[0], n = s_book[1], pend = s_book[2], m = a.m;

  // Row decisions; every CTA of sequence b takes the same ones.
  bool pre, post = false;
  if (a.mode == kFlush) {
    if (a.mask != nullptr && a.mask[b] == 0) return;
    if (pend != 0) {
      if (h == 0 && tid == 0) atomicOr(a.status, (unsigned)RSSM_STATUS_STATE);
      return;
    }
    if (n == 0) return;
    pre = true;
  } else {
    if (pend != 0) {
      if (h == 0 && tid == 0) atomicOr(a.status, (unsigned)RSSM_STATUS_STATE);
      return;
    }
    pre = n + m > a.L;
    if (pre && !a.auto_flush) {
      if (h == 0 && tid == 0) atomicOr(a.status, (unsigned)RSSM_STATUS_CAPACITY);
      return;
    }
    post = a.mode == kDecode && a.auto_flush && ((pre ? 0 : n) + 1 == a.L);
  }
  const int w0 = pre ? n : 0;  // first entry of the output window
  const int ntot = n + m;
  const bool need_f32 = (RF == RSSM_READ_FP32) || pre || post;

  const size_t bh = (size_t)b * a.H + h;
  float *hc = a.hc + bh * P * N;
  const int row0 = warp * T::RPW + lane / T::LPR;
  const int c0 = (lane % T::LPR) * 4;
  constexpr int RB = rc_row_bytes<RF, N>();
  uint8_t *rc = (RF != RSSM_READ_FP32) ? a.rc_codes + bh * P * RB : nullptr;

  // 1. Stream the checkpoint tile (and/or its read copy) into registers.
  float4 st4[T::NLD];
  float4 view[T::NLD];
  if (need_f32) {
#pragma unroll
    for (int l = 0; l < T::NLD; ++l) st4[l] = ld_stream(hc + (size_t)(row0 + l * T::RPI) * N + c0);
  }
  if constexpr (RF != RSSM_READ_FP32) {
    if (!pre && m > 0) {
#pragma unroll
      for (int l = 0; l < T::NLD; ++l) {
        const int row = row0 + l * T::RPI;
        view[l] = load_read_copy4<RF>(rc + (size_t)row * RB, a.rc_scales, bh * P + row, N, c0);
      }
    }
  }

  // 2. Stage the window (committed entries, then the new tokens) in shared
  //    memory and append the new tokens to the ring.
  constexpr int kPer = 16 / sizeof(Tin);
  constexpr int XV = P / kPer, BV = N / kPer;
  const Tin *xbuf = reinterpret_cast<const Tin *>(a.buf0) + bh * cap * P;
  const Tin *Bbuf = reinterpret_cast<const Tin *>(a.buf1) + ((size_t)b * a.G + g) * cap * N;
  for (int idx = tid; idx < n * (XV + BV); idx += kThreads) {
    const int i = idx / (XV + BV), r = idx - i * (XV + BV);
    const int slot = (st + i) % cap;
    const Tin *src = r < XV ? xbuf + slot * P + r * kPer : Bbuf + slot * N + (r - XV) * kPer;
    float *dst = r < XV ? s_x + i * P + r * kPer : s_B + i * N + (r - XV) * kPer;
    const uint4 raw = __ldg(reinterpret_cast<const uint4 *>(src));
    const Tin *e = reinterpret_cast<const Tin *>(&raw);
#pragma unroll
    for (int c = 0; c < kPer; ++c) dst[c] = to_f32<Tin>(e[c]);
  }
  for (int i = tid; i < n; i += kThreads) s_dt[i] = a.buf2[bh * cap + (st + i) % cap];
  {
    const Tin *xin = reinterpret_cast<const Tin *>(a.in[0]);
    const Tin *Bin = reinterpret_cast<const Tin *>(a.in[1]);
    const Tin *Cin = reinterpret_cast<const Tin *>(a.in[2]);
    const Tin *dtin = reinterpret_cast<const Tin *>(a.in[3]);
    Tin *xring = reinterpret_cast<Tin *>(a.buf0) + bh * cap * P;
    Tin *Bring = reinterpret_cast<Tin *>(a.buf1) + ((size_t)b * a.G + g) * cap * N;
    const bool group_writer = (h % a.hpg) == 0;
    for (int idx = tid; idx < m * (XV + 2 * BV); idx += kThreads) {
      const int j = idx / (XV + 2 * BV), r = idx - j * (XV + 2 * BV);
      const int slot = (st + n + j) % cap;   // same slot with or without a pre-fold
      const size_t tok = (size_t)b * m + j;
      const Tin *src;
      float *dst;
      Tin *ring = nullptr;
      if (r < XV) {
        src = xin + (tok * a.H + h) * P + r * kPer;
        dst = s_x + (n + j) * P + r * kPer;
        ring = xring + slot * P + r * kPer;
      } else if (r < XV + BV) {
        src = Bin + (tok * a.G + g) * N + (r - XV) * kPer;
        dst = s_B + (n + j) * N + (r - XV) * kPer;
        if (group_writer) ring = Bring + slot * N + (r - XV) * kPer;
      } else {
        src = Cin + (tok * a.G + g) * N + (r - XV - BV) * kPer;
        dst = s_C + j * N + (r - XV - BV) * kPer;
      }
      const uint4 raw = __ldg(reinterpret_cast<const uint4 *>(src));
      if (ring) *reinterpret_cast<uint4 *>(ring) = raw;
      const Tin *e = reinterpret_cast<const Tin *>(&raw);
#pragma unroll
      for (int c = 0; c < kPer; ++c) dst[c] = to_f32<Tin>(e[c]);
    }
    for (int j = tid; j < m; j += kThreads) {
      const float dtv = to_f32<Tin>(dtin[((size_t)b * m + j) * a.H + h]);
      s_dt[n + j] = dtv;
      a.buf2[bh * cap + (st + n + j) % cap] = dtv;
    }
    for (int idx = m * N + tid; idx < MAXM * N; idx += kThreads) s_C[idx] = 0.0f;
  }
  __syncthreads();

  // 3. Window scalars: a_i = dt_i A, B_i . C_j, coefficients and decays.
  //    Segment sums are direct sums of the a_r (never ratios of decays).
  const float Ah = __ldg(a.A + h);
  for (int i = tid; i < ntot; i += kThreads) s_a[i] = s_dt[i] * Ah;
  for (int p = warp; p < m * ntot; p += kWarps) {
    const int j = p / ntot, i = p - j * ntot;
    if (i < w0 || i > n + j) continue;
    float acc = 0.0f;
    for (int c = lane; c < N; c += 32) acc = fmaf(s_B[i * N + c], s_C[j * N + c], acc);
    acc = warp_sum(acc);
    if (lane == 0) s_bc[j * cap + i] = acc;
  }
  __syncthreads();
  for (int p = tid; p < m * ntot; p += kThreads) {
    const int j = p / ntot, i = p - j * ntot, e = n + j;
    if (i < w0 || i > e) continue;
    float sg = 0.0f;
    for (int r = i + 1; r <= e; ++r) sg += s_a[r];
    s_coef[j * cap + i] = expf(sg) * s_dt[i] * s_bc[j * cap + i];
  }
  for (int j = tid; j < m; j += kThreads) {
    float G = 0.0f;
    for (int r = w0; r <= n + j; ++r) G += s_a[r];
    s_dec[j] = expf(G);
  }
  if (pre) {
    for (int i = tid; i < n; i += kThreads) {
      float sg = 0.0f;
      for (int r = i + 1; r < n; ++r) sg += s_a[r];
      s_fwpre[i] = expf(sg) * s_dt[i];
    }
    if (tid == 0) {
      float G = 0.0f;
      for (int r = 0; r < n; ++r) G += s_a[r];
      s_dec[MAXM] = expf(G);
    }
  }
  if (post) {
    for (int i = w0 + tid; i <= n; i += kThreads) {
      float sg = 0.0f;
      for (int r = i + 1; r <= n; ++r) sg += s_a[r];
      s_fwpost[i] = expf(sg) * s_dt[i];
    }
    if (tid == 0) {
      float G = 0.0f;
      for (int r = w0; r <= n; ++r) G += s_a[r];
      s_dec[MAXM + 1] = expf(G);
    }
  }
  __syncthreads();

  // 4. New tokens do not fit: fold the committed window into the checkpoint
  //    first; its read copy is rebuilt from the folded fp32 values.
  if (pre) {
    fold_tile<P, N>(st4, s_fwpre, s_dec[MAXM], 0, n, s_x, s_B, row0, c0);
#pragma unroll
    for (int l = 0; l < T::NLD; ++l) {
      const int row = row0 + l * T::RPI;
      if constexpr (RF != RSSM_READ_FP32)
        view[l] = quantize4<RF, T::LPR>(st4[l], rc + (size_t)row * RB, a.rc_scales, bh * P + row, N, c0, lane);
      if (!post) st_stream(hc + (size_t)row * N + c0, st4[l]);
    }
  }

  // 5. Outputs of the new tokens, from the read view of the checkpoint.
  if (m > 0) {
    if constexpr (RF == RSSM_READ_FP32)
      outputs<P, N, MAXM>(st4, a, s_C, s_x, s_coef, s_dec, b, h, n, w0, warp, lane, c0);
    else
      outputs<P, N, MAXM>(view, a, s_C, s_x, s_coef, s_dec, b, h, n, w0, warp, lane, c0);
  }

  // 6. The decode filled the window: fold all of it.
  if (post) {
    fold_tile<P, N>(st4, s_fwpost, s_dec[MAXM + 1], w0, n + 1, s_x, s_B, row0, c0);
#pragma unroll
    for (int l = 0; l < T::NLD; ++l) {
      const int row = row0 + l * T::RPI;
      st_stream(hc + (size_t)row * N + c0, st4[l]);
      if constexpr (RF != RSSM_READ_FP32)
        quantize4<RF, T::LPR>(st4[l], rc + (size_t)row * RB, a.rc_scales, bh * P + row, N, c0, lane);
    }
  }

  // 7. The last CTA of sequence b moves its pointers.
  __syncthreads();
  if (last_arrival(a.arrivals + b, a.H)) {
    int st2 = st, n2 = n, fl = a.flushes[b];
    if (pre) {
      st2 = (st + n) % cap;
      n2 = 0;
      ++fl;
    }
    if (a.mode == kDecode) {
      n2 += 1;
      if (post) {
        st2 = (st2 + n2) % cap;
        n2 = 0;
        ++fl;
      }
    } else if (a.mode == kVerify) {
      a.pending[b] = m;
    }
    a.start[b] = st2;
    a.len[b] = n2;
    a.flushes[b] = fl;
  }
}

// Conventional update: h <- e^{dt A} h + dt x B^T ; y = h C + D x ; h written back.
template <int P, int N, typename Tin>
__global__ void __launch_bounds__(kThreads) m2_conv_kernel(const ConvArgs a) {
  using T = Tile<P, N>;
  __shared__ __align__(16) float s_x[P];
  __shared__ __align__(16) float s_B[N];
  __shared__ __align__(16) float s_C[N];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int b = blockIdx.x / a.H, h = blockIdx.x - b * a.H, g = h / a.hpg;
  const size_t bh = (size_t)b * a.H + h;
  const int row0 = warp * T::RPW + lane / T::LPR;
  const int c0 = (lane % T::LPR) * 4;
  float4 t[T::NLD];
#pragma unroll
  for (int l = 0; l < T::NLD; ++l)
    t[l] = ld_stream(a.state_in + bh * P * N + (size_t)(row0 + l * T::RPI) * N + c0);
  const Tin *xin = reinterpret_cast<const Tin *>(a.in[0]);
  const Tin *Bin = reinterpret_cast<const Tin *>(a.in[1]);
  const Tin *Cin = reinterpret_cast<const Tin *>(a.in[2]);
  const Tin *dtin = reinterpret_cast<const Tin *>(a.in[3]);
  stage_row<Tin>(s_x, xin + bh * P, P, tid, kThreads);
  stage_row<Tin>(s_B, Bin + ((size_t)b * a.G + g) * N, N, tid, kThreads);
  stage_row<Tin>(s_C, Cin + ((size_t)b * a.G + g) * N, N, tid, kThreads);
  __syncthreads();
  const float dt = to_f32<Tin>(dtin[bh]);
  const float dA = expf(dt * __ldg(a.A + h));
  const float4 bv = *reinterpret_cast<const float4 *>(s_B + c0);
  const float4 cv = *reinterpret_cast<const float4 *>(s_C + c0);
  float part[T::NLD];
#pragma unroll
  for (int l = 0; l < T::NLD; ++l) {
    const int row = row0 + l * T::RPI;
    const float xr = dt * s_x[row];
    t[l].x = fmaf(xr, bv.x, dA * t[l].x);
    t[l].y = fmaf(xr, bv.y, dA * t[l].y);
    t[l].z = fmaf(xr, bv.z, dA * t[l].z);
    t[l].w = fmaf(xr, bv.w, dA * t[l].w);
    st_stream(a.state_out + bh * P * N + (size_t)row * N + c0, t[l]);
    part[l] = t[l].x * cv.x + t[l].y * cv.y + t[l].z * cv.z + t[l].w * cv.w;
  }
  tr_sum<T::NLD, T::LPR / 2>(part, lane);
  const int base = tr_base<T::NLD, T::LPR / 2>(lane);
  constexpr int R = T::NLD >= T::LPR ? T::NLD / T::LPR : 1;
  const bool writer = T::NLD >= T::LPR || (lane & (T::LPR / T::NLD - 1)) == 0;
  const float Dh = __ldg(a.D + h);
#pragma unroll
  for (int q = 0; q < R; ++q) {
    const int row = warp * T::RPW + (base + q) * T::RPI + lane / T::LPR;
    if (writer) a.out[bh * P + row] = part[q] + Dh * s_x[row];
  }
}

size_t step_smem_bytes(int P, int N, int cap, int maxm) {
  return sizeof(float) * ((size_t)cap * (P + N) + (size_t)maxm * N + 2 * (size_t)cap +
                          2 * (size_t)maxm * cap + 2 * (size_t)cap + maxm + 2);
}

template <int P, int N, typename Tin, int RF, int MAXM>
cudaError_t launch_step(const StepArgs &a, cudaStream_t s) {
  auto kern = m2_step_kernel<P, N, Tin, RF, MAXM>;
  const size_t smem = step_smem_bytes(P, N, a.cap, MAXM);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  kern<<<dim3((unsigned)(a.B * a.H)), dim3(kThreads), smem, s>>>(a);
  return cudaGetLastError();
}

template <int P, int N, typename Tin, int RF>
cudaError_t dispatch_m(const StepArgs &a, cudaStream_t s) {
  if (a.mode != kVerify) return launch_step<P, N, Tin, RF, 1>(a, s);
  if (a.m <= 4) return launch_step<P, N, Tin, RF, 4>(a, s);
  return launch_step<P, N, Tin, RF, 8>(a, s);
}

template <int P, int N, typename Tin>
cudaError_t dispatch_rf(const StepArgs &a, int rf, cudaStream_t s) {
  switch (rf) {
    case RSSM_READ_FP32: return dispatch_m<P, N, Tin, RSSM_READ_FP32>(a, s);
    case RSSM_READ_FP8_E4M3_ROW: return dispatch_m<P, N, Tin, RSSM_READ_FP8_E4M3_ROW>(a, s);
    default: return dispatch_m<P, N, Tin, RSSM_READ_NVFP4>(a, s);
  }
}

template <int P, int N>
cudaError_t dispatch_dtype(const StepArgs &a, int in_dtype, int rf, cudaStream_t s) {
  if (in_dtype == RSSM_BF16) return dispatch_rf<P, N, __nv_bfloat16>(a, rf, s);
  return dispatch_rf<P, N, float>(a, rf, s);
}

template <int P, int N>
cudaError_t launch_conv(const ConvArgs &a, int in_dtype, cudaStream_t s) {
  if (in_dtype == RSSM_BF16)
    m2_conv_kernel<P, N, __nv_bfloat16><<<dim3((unsigned)(a.B * a.H)), dim3(kThreads), 0, s>>>(a);
  else
    m2_conv_kernel<P, N, float><<<dim3((unsigned)(a.B * a.H)), dim3(kThreads), 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace

bool mamba2_supported(int R, int C) { return R == 64 && (C == 64 || C == 128); }

cudaError_t mamba2_step(const StepArgs &a, int in_dtype, int read_fmt, cudaStream_t s) {
  if (a.R == 64 && a.C == 64) return dispatch_dtype<64, 64>(a, in_dtype, read_fmt, s);
  return dispatch_dtype<64, 128>(a, in_dtype, read_fmt, s);
}

cudaError_t mamba2_conventional(const ConvArgs &a, int in_dtype, cudaStream_t s) {
  if (a.R == 64 && a.C == 64) return launch_conv<64, 64>(a, in_dtype, s);
  return launch_conv<64, 128>(a, in_dtype, s);
}

}  // namespace rssm
