// Kimi Delta Attention (KDA) replay decode / flush and the conventional step.
//
// KDA is read as the gated delta rule with one gate per key channel
// ("ReplaySSM: Rethinking State Storage for Faster Hybrid-Model Decoding",
// babnews.org teaser, names the layer; no formula is given):
//   S_t = S_{t-1} Diag(alpha_t) + beta_t (v_t - S_{t-1} Diag(alpha_t) k_t) k_t^T,
//   o_t = out_scale S_t q_t,  S in R^{dv x dk}.
// Replay form over a window of entries 0..t on top of the checkpoint S_c, with
// g = ln alpha per channel, seg(s,t) = sum_{s<r<=t} g_r and G_t = sum_{r<=t} g_r.
// The ring keeps alpha itself, and e^{seg(s,t)} = prod_{s<r<=t} alpha_r is
// formed as a running product per channel (the same value as the exponential
// of the suffix sum, with no transcendental per entry):
//   w_t = beta_t (v_t - S_c (e^{G_t} . k_t) - sum_{s<t} ((k_s . e^{seg(s,t)}) . k_t) w_s)
//   o_t = out_scale (S_c (e^{G_t} . q_t) + sum_{s<=t} ((k_s . e^{seg(s,t)}) . q_t) w_s)
//   fold: S_c <- S_c Diag(e^{G_t}) + sum_{s<=t} w_s (k_s . e^{seg(s,t)})^T
// (. between vectors: elementwise).  The w_s of committed entries are kept in
// the ring, so a decode reads S_c once and does two matrix-vector products.
//
// A verify call runs its k drafts through the same solve in order (draft j is
// entry n + j, seeing S_c, the committed window and drafts 0 .. j-1) and leaves
// them in the ring as pending entries with their w rows; a rollback keeps the
// accepted prefix, whose w rows are then exactly those a decode of the same
// tokens would have written.
//
// One CTA of 256 threads per (sequence, head).  The 128 x 128 fp32 tile sits in
// registers: warp w holds rows 16w .. 16w+15, lane l columns 4l .. 4l+3.  The
// window's k rows, log gates, cached w rows and decays sit in shared memory.
#include "rssm_device.cuh"
#include "rssm_kda.h"

namespace rssm {
namespace {

constexpr int KD = 128;            // d_k = d_v
constexpr int kKdaThreads = 256;
constexpr int kRowsPerWarp = KD / (kKdaThreads / 32);   // 16

struct KdaSmem {
  int wmax;
  size_t floats() const { return (size_t)4 * wmax * KD + 5 * KD + 2 * wmax + 8; }
};

// S (registers) <- S Diag(e^{G}) + sum_{s<=t} w_s (k_s . dec_s)^T for this thread's
// 16 x 4 block.
__device__ __forceinline__ void kda_fold(float4 (&S)[kRowsPerWarp], const float *eG, const float *kw,
                                         const float *dec, const float *ww, int t, int row0, int c0) {
  const float4 e = *reinterpret_cast<const float4 *>(eG + c0);
#pragma unroll
  for (int i = 0; i < kRowsPerWarp; ++i) {
    S[i].x *= e.x;
    S[i].y *= e.y;
    S[i].z *= e.z;
    S[i].w *= e.w;
  }
  for (int s = 0; s <= t; ++s) {
    const float4 kk = *reinterpret_cast<const float4 *>(kw + s * KD + c0);
    const float4 dd = *reinterpret_cast<const float4 *>(dec + s * KD + c0);
    const float4 kd = make_float4(kk.x * dd.x, kk.y * dd.y, kk.z * dd.z, kk.w * dd.w);
#pragma unroll
    for (int i = 0; i < kRowsPerWarp; ++i) {
      const float wv = ww[s * KD + row0 + i];
      S[i].x = fmaf(wv, kd.x, S[i].x);
      S[i].y = fmaf(wv, kd.y, S[i].y);
      S[i].z = fmaf(wv, kd.z, S[i].z);
      S[i].w = fmaf(wv, kd.w, S[i].w);
    }
  }
}

// dec[s][c] = e^{seg(s,t)}, eG[c] = e^{G_t} from the gates aw[0..t] (threads < KD, one channel each).
__device__ __forceinline__ void kda_decays(const float *aw, float *dec, float *eG, int t) {
  const int c = threadIdx.x;
  if (c < KD) {
    float acc = 1.0f;
    for (int s = t; s >= 0; --s) {
      dec[s * KD + c] = acc;
      acc *= aw[s * KD + c];
    }
    eG[c] = acc;
  }
}

template <typename Tin, int RF>
__global__ void __launch_bounds__(kKdaThreads, 2) kda_replay_kernel(const StepArgs a) {
  constexpr int RB = RF == RSSM_READ_NVFP4 ? KD / 2 : KD;   // bytes of a read-copy row
  extern __shared__ __align__(16) float sm[];
  const int bh = blockIdx.x, b = bh / a.H, h = bh - b * a.H;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int L = a.L, cap = a.cap, wmax = L + (a.m > 1 ? a.m : 1);
  float *kw = sm;                   // [wmax][KD]  window k rows (fp32)
  float *gw = kw + wmax * KD;       // [wmax][KD]  gates alpha
  float *ww = gw + wmax * KD;       // [wmax][KD]  w rows
  float *dec = ww + wmax * KD;      // [wmax][KD]  e^{seg(s, t)}
  float *qv = dec + wmax * KD, *vv = qv + KD, *eG = vv + KD, *uu = eG + KD, *yy = uu + KD;
  float *Adot = yy + KD, *Bdot = Adot + wmax;   // window dot products

  // the checkpoint tile is requested first: its address needs nothing but the
  // sequence's slot (b itself unless the layer branches)
  const int row0 = warp * kRowsPerWarp, c0 = lane * 4;
  const int src_slot = a.slot ? a.slot[b] : b;
  const float *src = a.hc + ((size_t)src_slot * a.H + h) * KD * KD;
  float4 S[kRowsPerWarp];
  auto load_fp32 = [&](const float *from) {
#pragma unroll
    for (int i = 0; i < kRowsPerWarp; ++i) S[i] = ld_stream(from + (size_t)(row0 + i) * KD + c0);
  };
  if constexpr (RF == RSSM_READ_FP32) {
    load_fp32(src);
  } else {   // a read-copy layer's reads see the copy; a fold reloads the fp32 rows
    const size_t rbase = ((size_t)src_slot * a.H + h) * KD;
#pragma unroll
    for (int i = 0; i < kRowsPerWarp; ++i)
      S[i] = load_read_copy4<RF>(a.rc_codes + (rbase + row0 + i) * RB, a.rc_scales, rbase + row0 + i, KD, c0);
  }
  // and the first new token's inputs (thread c < KD: channel / value row c)
  Tin kr{}, vr{}, qr{};
  float ar = 1.0f;
  auto load_token = [&](int j) {   // token j of this call (decode: j = 0; verify: draft j)
    if (tid < KD) {
      const size_t tix = ((size_t)b * a.m + j) * a.H + h;
      kr = reinterpret_cast<const Tin *>(a.in[1])[tix * KD + tid];
      vr = reinterpret_cast<const Tin *>(a.in[2])[tix * KD + tid];
      qr = reinterpret_cast<const Tin *>(a.in[0])[tix * KD + tid];
      ar = reinterpret_cast<const float *>(a.in[3])[tix * KD + tid];
    }
  };
  if (a.m >= 1) load_token(0);

  const RowPlan rp = plan_row(a, b);
  if (rp.refuse) {
    if (rp.bit && h == 0 && tid == 0) atomicOr(a.status, rp.bit);
    return;
  }
  // Every CTA of sequence b has read its pointers once all of them have counted
  // in, so the last to count in moves them now (its own threads have read them:
  // the barrier below), off the end of the kernel.
  __syncthreads();
  if (tid == 0 && atomicAdd(a.arrivals + b, 1) == a.H - 1) {
    a.arrivals[b] = 0;
    int st2 = rp.st, n2 = rp.n, fl = a.flushes[b];
    if (rp.pre) {
      st2 = (rp.st + rp.n) % a.cap;
      n2 = 0;
      ++fl;
    }
    if (a.mode == kDecode) {
      n2 += 1;
      if (rp.post) {
        st2 = (st2 + n2) % a.cap;
        n2 = 0;
        ++fl;
      }
    } else if (a.mode == kVerify) {
      a.pending[b] = a.m;   // the drafts are appended as pending entries
    }
    a.start[b] = st2;
    a.len[b] = n2;
    a.flushes[b] = fl;
  }
  const int m = a.m, st = rp.st;
  int n = rp.n;
  const bool pre = rp.pre, post = rp.post;
  const Tin *kring = reinterpret_cast<const Tin *>(a.buf0) + (size_t)bh * cap * KD;
  Tin *kring_w = reinterpret_cast<Tin *>(a.buf0) + (size_t)bh * cap * KD;
  Tin *vring = reinterpret_cast<Tin *>(a.buf1) + (size_t)bh * cap * KD;
  float *gring = a.buf2 + (size_t)bh * cap * KD;   // alpha per channel
  float *bring = a.buf3 + (size_t)bh * cap;
  float *wring = a.buf4 + (size_t)bh * cap * KD;   // [2 halves][cap][KD / 2]
  auto wslot = [&](size_t slot, int i) -> size_t { return ((size_t)(i / (KD / 2)) * cap + slot) * (KD / 2) + i % (KD / 2); };

  float *dst = a.hc + ((size_t)rp.dst * a.H + h) * KD * KD;   // where a fold writes

  // Read-copy layers: the w rows cached while decoding were solved against the
  // copy, so a fold first solves its entries 0..tl again against the fp32 tile
  // in S (the same forward substitution; entry t in ring slot (st_e + t) % cap),
  // leaving dec / eG of t = tl for the fold.  The cached rows are not rewritten:
  // the fold empties the window.
  auto resolve = [&](int tl, int st_e) {
    for (int t = 0; t <= tl; ++t) {
      const size_t slot = (size_t)((st_e + t) % cap);
      kda_decays(gw, dec, eG, t);
      __syncthreads();
      for (int s2 = warp; s2 < t; s2 += kKdaThreads / 32) {
        float acc = 0.0f;
#pragma unroll
        for (int jj = 0; jj < KD / 32; ++jj) {
          const int c = lane + 32 * jj;
          acc = fmaf(kw[s2 * KD + c] * dec[s2 * KD + c], kw[t * KD + c], acc);
        }
        acc = warp_sum(acc);
        if (lane == 0) Adot[s2] = acc;
      }
      {   // u = S (e^{G_t} . k_t)
        const float4 e = *reinterpret_cast<const float4 *>(eG + c0);
        const float4 kk = *reinterpret_cast<const float4 *>(kw + t * KD + c0);
        const float4 gk = make_float4(e.x * kk.x, e.y * kk.y, e.z * kk.z, e.w * kk.w);
        float p[kRowsPerWarp];
#pragma unroll
        for (int i = 0; i < kRowsPerWarp; ++i) p[i] = S[i].x * gk.x + S[i].y * gk.y + S[i].z * gk.z + S[i].w * gk.w;
        tr_sum<kRowsPerWarp, 16>(p, lane);   // lanes 2j, 2j + 1 hold the sum of row tr_base
        if ((lane & 1) == 0) uu[row0 + tr_base<kRowsPerWarp, 16>(lane)] = p[0];
      }
      __syncthreads();
      if (tid < KD) {
        float r = to_f32<Tin>(vring[slot * KD + tid]) - uu[tid];
        for (int s2 = 0; s2 < t; ++s2) r = fmaf(-Adot[s2], ww[s2 * KD + tid], r);
        ww[t * KD + tid] = bring[slot] * r;
      }
      __syncthreads();
    }
  };
  // Store the folded fp32 rows; a read-copy layer also quantises them into its
  // copy and reads the copy back into S (the reads that follow see the new copy).
  auto store_fold = [&]() {
#pragma unroll
    for (int i = 0; i < kRowsPerWarp; ++i) st_stream(dst + (size_t)(row0 + i) * KD + c0, S[i]);
    if constexpr (RF != RSSM_READ_FP32) {
      const size_t dbase = ((size_t)rp.dst * a.H + h) * KD;
#pragma unroll
      for (int i = 0; i < kRowsPerWarp; ++i)
        S[i] = quantize4<RF, 32>(S[i], a.rc_codes + (dbase + row0 + i) * RB, a.rc_scales, dbase + row0 + i, KD, c0,
                                 lane);
    }
  };

  // committed window rows into shared memory
  for (int idx = tid; idx < n * KD; idx += kKdaThreads) {
    const int e = idx / KD, c = idx - e * KD;
    const size_t slot = (size_t)((st + e) % cap);
    kw[idx] = to_f32<Tin>(kring[slot * KD + c]);
    gw[idx] = gring[slot * KD + c];
    ww[idx] = wring[wslot(slot, c)];
  }
  __syncthreads();

  if (pre) {   // the committed window is folded first (flush, or a token that does not fit)
    if constexpr (RF == RSSM_READ_FP32) {
      kda_decays(gw, dec, eG, n - 1);
      __syncthreads();
      kda_fold(S, eG, kw, dec, ww, n - 1, row0, c0);
      if (!post && m == 0) {
#pragma unroll
        for (int i = 0; i < kRowsPerWarp; ++i) st_stream(dst + (size_t)(row0 + i) * KD + c0, S[i]);
      }
    } else {
      load_fp32(src);
      resolve(n - 1, st);
      kda_fold(S, eG, kw, dec, ww, n - 1, row0, c0);
      store_fold();
    }
    __syncthreads();   // the window arrays are reused below
  }
  int st_new = st;
  if (pre) {
    st_new = (st + n) % cap;
    n = 0;
  }

  for (int j = 0; j < m; ++j) {
    // ---- new token j (decode: the token; verify: draft j): entry t = n + j of the
    //      window, ring slot (st_new + t) % cap; each solved against S_c and the
    //      window entries before it
    const int t = n + j;
    const size_t slot = (size_t)((st_new + t) % cap);
    const size_t tix = ((size_t)b * m + j) * a.H + h;
    const float beta = reinterpret_cast<const float *>(a.in[4])[tix];
    if (j > 0) load_token(j);   // registers: the previous token ended on a barrier
    if (tid < KD) {
      const float g = ar;
      kw[t * KD + tid] = to_f32<Tin>(kr);
      gw[t * KD + tid] = g;
      qv[tid] = to_f32<Tin>(qr);
      vv[tid] = to_f32<Tin>(vr);
      kring_w[slot * KD + tid] = kr;
      vring[slot * KD + tid] = vr;
      gring[slot * KD + tid] = g;
    }
    if (tid == 0) bring[slot] = beta;
    __syncthreads();
    kda_decays(gw, dec, eG, t);
    __syncthreads();
    // window dots: Adot[s] = (k_s . dec_s) . k_t (s < t), Bdot[s] = (k_s . dec_s) . q_t (s <= t)
    for (int task = warp; task < 2 * (t + 1); task += kKdaThreads / 32) {
      const int s = task >> 1;
      const bool isq = task & 1;
      if (!isq && s == t) continue;
      const float *other = isq ? qv : kw + t * KD;
      float acc = 0.0f;
#pragma unroll
      for (int jj = 0; jj < KD / 32; ++jj) {
        const int c = lane + 32 * jj;
        acc = fmaf(kw[s * KD + c] * dec[s * KD + c], other[c], acc);
      }
      acc = warp_sum(acc);
      if (lane == 0) (isq ? Bdot : Adot)[s] = acc;
    }
    // u = S_c (e^{G_t} . k_t), y = S_c (e^{G_t} . q_t) from the register tile
    {
      const float4 e = *reinterpret_cast<const float4 *>(eG + c0);
      const float4 kk = *reinterpret_cast<const float4 *>(kw + t * KD + c0);
      const float4 qq = *reinterpret_cast<const float4 *>(qv + c0);
      const float4 gk = make_float4(e.x * kk.x, e.y * kk.y, e.z * kk.z, e.w * kk.w);
      const float4 gq = make_float4(e.x * qq.x, e.y * qq.y, e.z * qq.z, e.w * qq.w);
      float p[2 * kRowsPerWarp];   // this lane's partial sums: u rows, then y rows
#pragma unroll
      for (int i = 0; i < kRowsPerWarp; ++i) {
        p[i] = S[i].x * gk.x + S[i].y * gk.y + S[i].z * gk.z + S[i].w * gk.w;
        p[kRowsPerWarp + i] = S[i].x * gq.x + S[i].y * gq.y + S[i].z * gq.z + S[i].w * gq.w;
      }
      tr_sum<2 * kRowsPerWarp, 16>(p, lane);   // 31 shuffles: lane ends with one complete sum
      const int idx = tr_base<2 * kRowsPerWarp, 16>(lane);
      (idx < kRowsPerWarp ? uu : yy)[row0 + (idx & (kRowsPerWarp - 1))] = p[0];
    }
    __syncthreads();
    // w_t and the output, one value row per thread
    if (tid < KD) {
      const int i = tid;
      float r = vv[i] - uu[i];
      for (int s = 0; s < t; ++s) r = fmaf(-Adot[s], ww[s * KD + i], r);
      const float w = beta * r;
      ww[t * KD + i] = w;
      wring[wslot(slot, i)] = w;
      float o = yy[i];
      for (int s = 0; s <= t; ++s) o = fmaf(Bdot[s], ww[s * KD + i], o);
      a.out[tix * KD + i] = a.out_scale * o;
    }
    __syncthreads();
  }
  if (m >= 1) {
    if (post) {   // the decode filled the window: fold all of it
      if constexpr (RF == RSSM_READ_FP32) {
        kda_fold(S, eG, kw, dec, ww, n, row0, c0);
#pragma unroll
        for (int i = 0; i < kRowsPerWarp; ++i) st_stream(dst + (size_t)(row0 + i) * KD + c0, S[i]);
      } else {   // from the fp32 rows (those a pre-fold of this call stored, if any)
        load_fp32(pre ? dst : src);
        resolve(n, st_new);
        kda_fold(S, eG, kw, dec, ww, n, row0, c0);
        store_fold();
      }
    } else if (pre && RF == RSSM_READ_FP32) {   // (a read-copy layer stored its pre-fold already)
#pragma unroll
      for (int i = 0; i < kRowsPerWarp; ++i) st_stream(dst + (size_t)(row0 + i) * KD + c0, S[i]);
    }
  }
}

// Conventional step: S <- S Diag(alpha); u = S k; S <- S + beta (v - u) k^T;
// o = out_scale S q; S written back.  One CTA per (sequence, head), tile in registers.
template <typename Tin>
__global__ void __launch_bounds__(kKdaThreads, 2) kda_conv_kernel(const ConvArgs a) {
  __shared__ __align__(16) float kv[KD], qv[KD], al[KD], uu[KD];
  const int bh = blockIdx.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int row0 = warp * kRowsPerWarp, c0 = lane * 4;
  const float *src = a.state_in + (size_t)bh * KD * KD;
  float *dst = a.state_out + (size_t)bh * KD * KD;
  float4 S[kRowsPerWarp];
#pragma unroll
  for (int i = 0; i < kRowsPerWarp; ++i) S[i] = ld_stream(src + (size_t)(row0 + i) * KD + c0);
  if (tid < KD) {
    kv[tid] = to_f32<Tin>(reinterpret_cast<const Tin *>(a.in[1])[(size_t)bh * KD + tid]);
    qv[tid] = to_f32<Tin>(reinterpret_cast<const Tin *>(a.in[0])[(size_t)bh * KD + tid]);
    al[tid] = reinterpret_cast<const float *>(a.in[3])[(size_t)bh * KD + tid];
  }
  __syncthreads();
  const float beta = reinterpret_cast<const float *>(a.in[4])[bh];
  const float4 e = *reinterpret_cast<const float4 *>(al + c0);
  const float4 kk = *reinterpret_cast<const float4 *>(kv + c0);
  const float4 qq = *reinterpret_cast<const float4 *>(qv + c0);
  float p[kRowsPerWarp];
#pragma unroll
  for (int i = 0; i < kRowsPerWarp; ++i) {
    S[i].x *= e.x;
    S[i].y *= e.y;
    S[i].z *= e.z;
    S[i].w *= e.w;
    p[i] = S[i].x * kk.x + S[i].y * kk.y + S[i].z * kk.z + S[i].w * kk.w;
  }
  tr_sum<kRowsPerWarp, 16>(p, lane);   // lanes 2j, 2j + 1 hold the sum of row tr_base
  if ((lane & 1) == 0) uu[row0 + tr_base<kRowsPerWarp, 16>(lane)] = p[0];
  __syncwarp();
  const Tin *vin = reinterpret_cast<const Tin *>(a.in[2]) + (size_t)bh * KD;
#pragma unroll
  for (int i = 0; i < kRowsPerWarp; ++i) {
    const int row = row0 + i;
    const float r = beta * (to_f32<Tin>(vin[row]) - uu[row]);
    S[i].x = fmaf(r, kk.x, S[i].x);
    S[i].y = fmaf(r, kk.y, S[i].y);
    S[i].z = fmaf(r, kk.z, S[i].z);
    S[i].w = fmaf(r, kk.w, S[i].w);
    p[i] = S[i].x * qq.x + S[i].y * qq.y + S[i].z * qq.z + S[i].w * qq.w;
    st_stream(dst + (size_t)row * KD + c0, S[i]);
  }
  tr_sum<kRowsPerWarp, 16>(p, lane);
  if ((lane & 1) == 0) a.out[(size_t)bh * KD + row0 + tr_base<kRowsPerWarp, 16>(lane)] = a.out_scale * p[0];
}

template <typename Tin, int RF>
cudaError_t launch_kda_step(const StepArgs &a, cudaStream_t s) {
  auto kern = kda_replay_kernel<Tin, RF>;
  const KdaSmem y{a.L + (a.m > 1 ? a.m : 1)};   // the window and the new tokens
  const size_t smem = y.floats() * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  kern<<<dim3((unsigned)((size_t)a.B * a.H)), dim3(kKdaThreads), smem, s>>>(a);
  return cudaGetLastError();
}

template <typename Tin>
cudaError_t dispatch_rf(const StepArgs &a, int read_fmt, cudaStream_t s) {
  switch (read_fmt) {
    case RSSM_READ_FP32: return launch_kda_step<Tin, RSSM_READ_FP32>(a, s);
    case RSSM_READ_FP8_E4M3_ROW: return launch_kda_step<Tin, RSSM_READ_FP8_E4M3_ROW>(a, s);
    default: return launch_kda_step<Tin, RSSM_READ_NVFP4>(a, s);
  }
}

}  // namespace

bool kda_supported(int R, int C) { return R == KD && C == KD; }

cudaError_t kda_step(const StepArgs &a, int in_dtype, int read_fmt, cudaStream_t s) {
  if (kda_decode_fast_path(a, in_dtype)) return kda_decode_step(a, s);
  return in_dtype == RSSM_BF16 ? dispatch_rf<__nv_bfloat16>(a, read_fmt, s) : dispatch_rf<float>(a, read_fmt, s);
}

cudaError_t kda_conventional(const ConvArgs &a, int in_dtype, cudaStream_t s) {
  const dim3 grid((unsigned)((size_t)a.B * a.H));
  if (in_dtype == RSSM_BF16)
    kda_conv_kernel<__nv_bfloat16><<<grid, dim3(kKdaThreads), 0, s>>>(a);
  else
    kda_conv_kernel<float><<<grid, dim3(kKdaThreads), 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace rssm
