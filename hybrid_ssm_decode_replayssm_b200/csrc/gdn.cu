// Gated DeltaNet kernels: ReplaySSM replay step (decode / verify / flush) in
// the WY/UT form, and the conventional per-token update (in-run baseline).
//
// Gated delta rule, S in R^{dv x dk}: S_t = a_t S_{t-1} (I - b_t k_t k_t^T) + b_t v_t k_t^T,
// o_t = out_scale S_t q_t.  On top of a checkpoint S_c, over window entries s,
// with g_r = ln a_r, seg(s,t) = sum_{s<r<=t} g_r and G_t the sum from the
// window start to t:
//   S_t = e^{G_t} S_c + sum_{s<=t} e^{seg(s,t)} w_s k_s^T
//   w_t = b_t (v_t - e^{G_t} S_c k_t - sum_{s<t} e^{seg(s,t)} (k_s . k_t) w_s)
//   o_t = out_scale (e^{G_t} S_c q_t + sum_{s<=t} e^{seg(s,t)} (k_s . q_t) w_s)
// -- a unit lower-triangular system for the w_s, solved by forward
// substitution (the UT form of the WY representation).  The w_s depend only on
// S_c and entries <= s, so a decode step solves for its own w only and keeps it
// in the ring (w_buf) for the reads of later steps.  "ReplaySSM: Rethinking
// State Storage for Faster Hybrid-Model Decoding" (deskofai.com summary,
// paragraphs 2-4): outputs come from the checkpoint and the buffered inputs,
// the buffer is folded in when it fills, drafts are appended and rolled back
// by pointer, and a low-precision copy may serve the reads while the
// recurrence stays in high precision.  So a fold never uses the cached w: it
// solves the window again from the fp32 checkpoint.
//
// Work unit: half a head (64 of the 128 value rows, 32 KiB of fp32 state).  A
// persistent CTA has one producer warp, which streams units into a ring of
// shared-memory stages with 1-D TMA bulk copies, and two consumer groups of 8
// warps taking alternate items (item = one sequence and a chunk of heads).
// Per head the group first computes the head's scalars (k.k and k.q products
// and decays) from the stage, then each warp handles 8 rows of each half.
#include "rssm_device.cuh"

namespace rssm {
namespace {

constexpr int DK = 128, DV = 128, HALF = 64;
constexpr int kGroupWarps = 8;
constexpr int kGroups = 2;
constexpr int kGroupThreads = kGroupWarps * 32;
constexpr int kConsumers = kGroups * kGroupThreads;
constexpr int kReplayThreads = kConsumers + 32;
constexpr int kMaxStages = 16;
constexpr int RPW = HALF / kGroupWarps;   // rows of a unit per warp (8)
constexpr int kMaxW = 32;                 // longest window a scan or fold covers

template <int RF> constexpr int tile_bytes() {
  return RF == RSSM_READ_FP32 ? HALF * DK * 4 : RF == RSSM_READ_FP8_E4M3_ROW ? HALF * DK : HALF * DK / 2;
}
template <int RF> constexpr int scale_bytes() {
  return RF == RSSM_READ_FP32 ? 0 : RF == RSSM_READ_FP8_E4M3_ROW ? HALF * 4 : HALF * (DK / 16);
}
template <int RF> constexpr int rc_row_bytes() { return RF == RSSM_READ_NVFP4 ? DK / 2 : DK; }
template <int RF> constexpr int rc_scale_row_bytes() { return RF == RSSM_READ_NVFP4 ? DK / 16 : 4; }

template <typename Tin>
__device__ __forceinline__ float4 ld4(const Tin *p) {
  if constexpr (sizeof(Tin) == 4) {
    return *reinterpret_cast<const float4 *>(p);
  } else {
    const uint2 raw = *reinterpret_cast<const uint2 *>(p);
    const Tin *e = reinterpret_cast<const Tin *>(&raw);
    return make_float4(to_f32<Tin>(e[0]), to_f32<Tin>(e[1]), to_f32<Tin>(e[2]), to_f32<Tin>(e[3]));
  }
}
template <typename Tin>
__device__ __forceinline__ void ld8(const Tin *p, float (&o)[8]) {
  if constexpr (sizeof(Tin) == 4) {
    const float4 a = reinterpret_cast<const float4 *>(p)[0], b = reinterpret_cast<const float4 *>(p)[1];
    o[0] = a.x; o[1] = a.y; o[2] = a.z; o[3] = a.w; o[4] = b.x; o[5] = b.y; o[6] = b.z; o[7] = b.w;
  } else {
    const uint4 raw = *reinterpret_cast<const uint4 *>(p);
    const Tin *e = reinterpret_cast<const Tin *>(&raw);
#pragma unroll
    for (int q = 0; q < 8; ++q) o[q] = to_f32<Tin>(e[q]);
  }
}
__device__ __forceinline__ float dot4(const float4 a, const float4 b) {
  return a.x * b.x + a.y * b.y + a.z * b.z + a.w * b.w;
}
__device__ __forceinline__ void fma4(float4 &t, float c, const float4 k) {
  t.x = fmaf(c, k.x, t.x); t.y = fmaf(c, k.y, t.y); t.z = fmaf(c, k.z, t.z); t.w = fmaf(c, k.w, t.w);
}
__device__ __forceinline__ void scale4(float4 &t, float c) { t.x *= c; t.y *= c; t.z *= c; t.w *= c; }

// Stage layout of one unit: [read tile | scales | k rows | q rows | v half rows | w half rows].
// k and v rows: committed entries at rows [0, n), new tokens at rows L + j.
template <typename Tin>
struct GStage {
  uint8_t *base;
  int koff, qoff, voff, woff, n, L;
  __device__ __forceinline__ int slot_row(int i) const { return i < n ? i : L + (i - n); }
  __device__ __forceinline__ const Tin *k(int i) const {
    return reinterpret_cast<const Tin *>(base + koff) + (size_t)slot_row(i) * DK;
  }
  __device__ __forceinline__ const Tin *q(int j) const {
    return reinterpret_cast<const Tin *>(base + qoff) + (size_t)j * DK;
  }
  __device__ __forceinline__ const Tin *v(int i) const {
    return reinterpret_cast<const Tin *>(base + voff) + (size_t)slot_row(i) * HALF;
  }
  __device__ __forceinline__ const float *w(int i) const {
    return reinterpret_cast<const float *>(base + woff) + (size_t)i * HALF;
  }
};

struct RowPlan {
  int st, n;
  bool refuse, pre, post;
  unsigned bit;
};
__device__ __forceinline__ RowPlan plan_row(const StepArgs &a, int b) {
  RowPlan r;
  r.st = a.start[b];
  r.n = a.len[b];
  const int pend = a.pending[b];
  r.refuse = r.pre = r.post = false;
  r.bit = 0;
  if (a.mode == kFlush) {
    if (a.mask != nullptr && a.mask[b] == 0) r.refuse = true;
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

// Per-group shared scalars of the current head.
template <int MAXM>
struct HeadScalars {
  static constexpr int kOut = MAXM + 2 * MAXM * 32;             // per head: dec, Mk, Mq
  static constexpr int kFold = kMaxW + 2 * kMaxW * kMaxW + kMaxW + 4; // decf, A, T, fw, decF, 1-entry fold
  static constexpr int kDots = 0;
  static constexpr int kWarp = kMaxW * RPW + 2 * MAXM * RPW;     // U/W fold scratch, reductions
};

// Fold of the window entries [i0, i0 + nf) into the fp32 rows t (8 rows of this
// warp, 4 columns of this lane), by the UT transform of the window: with
// u_i = t k_i (matvecs in chunks of 4 keys), r_i = beta_i (v_i - e^{G_i} u_i)
// and T = (I + A)^{-1}, A[i][i'] = beta_i e^{seg(i',i)} k_i'.k_i (i' < i), the
// solved values are w = T r (forward substitution done once per head in T),
// then t <- decF t + sum_i fw_i w_i k_i^T.
template <typename Tin>
__device__ void fold_rows(float4 (&t)[RPW], const GStage<Tin> &stg, int i0, int nf, const float *decf,
                          const float *Tm, const float *fw, float decF, const float *beta, int urow0,
                          float *U, int lane, int c0) {
  for (int ch = 0; ch < nf; ch += 4) {
    float part[RPW * 4];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int i = ch + c;
      const float4 kc = i < nf ? ld4<Tin>(stg.k(i0 + i) + c0) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int r = 0; r < RPW; ++r) part[r * 4 + c] = dot4(t[r], kc);
    }
    tr_sum<RPW * 4, 16>(part, lane);
    const int idx = tr_base<RPW * 4, 16>(lane), r = idx / 4, i = ch + idx % 4;
    if (i < nf) U[i * RPW + r] = part[0];
  }
  __syncwarp();
  for (int p = lane; p < nf * RPW; p += 32) {   // r_i per (entry, row); U[i][r] layout
    const int i = p / RPW, r = p - i * RPW;
    U[p] = beta[i0 + i] * fmaf(-decf[i], U[p], to_f32<Tin>(stg.v(i0 + i)[urow0 + r]));
  }
  __syncwarp();
  constexpr int kPer = kMaxW * RPW / 32;
  float wv[kPer];
#pragma unroll
  for (int q = 0; q < kPer; ++q) {
    const int p = lane + 32 * q, i = p / RPW, r = p - i * RPW;
    float acc = 0.0f;
    if (i < nf)
      for (int ip = 0; ip <= i; ++ip) acc = fmaf(Tm[i * kMaxW + ip], U[ip * RPW + r], acc);
    wv[q] = acc;
  }
  __syncwarp();
#pragma unroll
  for (int q = 0; q < kPer; ++q)
    if (lane + 32 * q < nf * RPW) U[lane + 32 * q] = wv[q];
  __syncwarp();
#pragma unroll
  for (int r = 0; r < RPW; ++r) scale4(t[r], decF);
  for (int i = 0; i < nf; ++i) {
    const float4 kc = ld4<Tin>(stg.k(i0 + i) + c0);
    const float f = fw[i];
#pragma unroll
    for (int r = 0; r < RPW; ++r) fma4(t[r], f * U[i * RPW + r], kc);
  }
  __syncwarp();
}

template <typename Tin, int RF, int MAXM>
__global__ void __launch_bounds__(kReplayThreads, 1)
    gdn_replay_kernel(const StepArgs a, const int hc, const int stages) {
  using HS = HeadScalars<MAXM>;
  constexpr int KROW = DK * (int)sizeof(Tin);
  constexpr int VHROW = HALF * (int)sizeof(Tin);
  constexpr int TB = tile_bytes<RF>();
  constexpr int SB = scale_bytes<RF>();
  constexpr int RB = rc_row_bytes<RF>();
  constexpr int SR = rc_scale_row_bytes<RF>();
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ uint64_t full[kMaxStages], empty[kMaxStages];
  __shared__ int stage_use[kMaxStages];   // see the Mamba-2 kernel: gates parity waits
  __shared__ int abort_flag;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int L = a.L, cap = a.cap, m = a.m, WMAX = L + MAXM;
  const int nchunk = a.H / hc;
  const int nitems = a.B * nchunk;
  const int my_items = (int)blockIdx.x < nitems ? (nitems - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
  const int total_seq = my_items * hc * 2;
  const int KOFF = TB + SB;
  const int QOFF = KOFF + (L + MAXM) * KROW;
  const int VOFF = QOFF + MAXM * KROW;
  const int WOFF = VOFF + (L + MAXM) * VHROW;
  const size_t stage_bytes = ((size_t)WOFF + (size_t)L * HALF * 4 + 127) & ~(size_t)127;
  const int group_floats = (2 * hc * WMAX + hc * HS::kOut + HS::kFold + kGroupWarps * HS::kWarp + 31) & ~31;

  const Tin *qin = reinterpret_cast<const Tin *>(a.in[0]);
  const Tin *kin = reinterpret_cast<const Tin *>(a.in[1]);
  const Tin *vin = reinterpret_cast<const Tin *>(a.in[2]);
  const float *alin = reinterpret_cast<const float *>(a.in[3]);
  const float *bein = reinterpret_cast<const float *>(a.in[4]);
  Tin *kring = reinterpret_cast<Tin *>(a.buf0);
  Tin *vring = reinterpret_cast<Tin *>(a.buf1);
  float *gring = a.buf2, *bring = a.buf3, *wring = a.buf4;
  volatile int *abort = &abort_flag;

  if (tid == 0) {
    for (int s = 0; s < stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kGroupWarps);
      stage_use[s] = -1;
    }
    abort_flag = 0;
    mbar_fence_init();
  }
  __syncthreads();

  auto item_of = [&](int k, int &b, int &chunk) {
    const int item = (int)blockIdx.x + k * (int)gridDim.x;
    b = item / nchunk;
    chunk = item - b * nchunk;
  };

  if (warp == kConsumers / 32) {
    // ------------------------------------------------------------ producer
    if (lane != 0) return;
    // Issue order: the units of items 2p and 2p+1 interleaved (unit u of 2p, unit
    // u of 2p+1, unit u+1 of 2p, ...), so both consumer groups work at once.
    int b2[2] = {0, 0}, chunk2[2] = {0, 0}, s = 0, u = 0, cur_pair = -1;
    RowPlan rp2[2] = {};
    int issued = 0;
    for (int seq = 0; seq < total_seq; ++seq) {
      if (u > 0 && !mbar_wait_bounded(&empty[s], (uint32_t)((u - 1) & 1), abort)) {
        atomicOr(a.status, (unsigned)RSSM_STATUS_TIMEOUT);
        break;
      }
      const int p = seq / (4 * hc), within = seq - p * 4 * hc;
      const bool paired = 2 * p + 1 < my_items;
      const int gsel = paired ? (within & 1) : 0;
      const int unit = paired ? (within >> 1) : within;
      if (p != cur_pair) {
        cur_pair = p;
        for (int g2 = 0; g2 < (paired ? 2 : 1); ++g2) {
          item_of(2 * p + g2, b2[g2], chunk2[g2]);
          rp2[g2] = plan_row(a, b2[g2]);
        }
      }
      const int b = b2[gsel], chunk = chunk2[gsel];
      const RowPlan &rp = rp2[gsel];
      issued = seq + 1;
      if (rp.refuse) {
        mbar_arrive(&full[s]);
      } else {
        const int jh = unit >> 1, hf = unit & 1;
        const int h = chunk * hc + jh;
        const size_t bh = (size_t)b * a.H + h;
        const bool fold = rp.pre || rp.post;
        const int nk = fold ? rp.n : 0;                // committed k rows (fold passes)
        const int nv = fold ? rp.n : 0;                // committed v rows
        const int nw = rp.pre ? 0 : rp.n;              // committed w rows
        uint8_t *dst = smem + s * stage_bytes;
        mbar_arrive_expect_tx(&full[s], (uint32_t)(TB + SB + (nk + 2 * m) * KROW + (nv + m) * VHROW + nw * HALF * 4));
        if constexpr (RF == RSSM_READ_FP32) {
          bulk_g2s(dst, a.hc + (bh * DV + hf * HALF) * DK, TB, &full[s]);
        } else {
          bulk_g2s(dst, a.rc_codes + (bh * DV + hf * HALF) * RB, TB, &full[s]);
          bulk_g2s(dst + TB, reinterpret_cast<const uint8_t *>(a.rc_scales) + (bh * DV + hf * HALF) * SR, SB, &full[s]);
        }
        const int c1 = rp.n < cap - rp.st ? rp.n : cap - rp.st;   // ring segment lengths
        if (nk > 0) {
          const Tin *src = kring + bh * cap * DK;
          bulk_g2s(dst + KOFF, src + (size_t)rp.st * DK, c1 * KROW, &full[s]);
          if (nk > c1) bulk_g2s(dst + KOFF + c1 * KROW, src, (nk - c1) * KROW, &full[s]);
        }
        if (nv > 0) {
          const Tin *src = vring + (bh * 2 + hf) * cap * HALF;
          bulk_g2s(dst + VOFF, src + (size_t)rp.st * HALF, c1 * VHROW, &full[s]);
          if (nv > c1) bulk_g2s(dst + VOFF + c1 * VHROW, src, (nv - c1) * VHROW, &full[s]);
        }
        if (nw > 0) {
          const float *src = wring + (bh * 2 + hf) * cap * HALF;
          bulk_g2s(dst + WOFF, src + (size_t)rp.st * HALF, c1 * HALF * 4, &full[s]);
          if (nw > c1) bulk_g2s(dst + WOFF + c1 * HALF * 4, src, (nw - c1) * HALF * 4, &full[s]);
        }
        for (int j = 0; j < m; ++j) {
          const size_t tok = ((size_t)b * m + j) * a.H + h;
          bulk_g2s(dst + KOFF + (L + j) * KROW, kin + tok * DK, KROW, &full[s]);
          bulk_g2s(dst + QOFF + j * KROW, qin + tok * DK, KROW, &full[s]);
          bulk_g2s(dst + VOFF + (L + j) * VHROW, vin + tok * DV + hf * HALF, VHROW, &full[s]);
        }
      }
      *reinterpret_cast<volatile int *>(&stage_use[s]) = u;
      if (++s == stages) {
        s = 0;
        ++u;
      }
    }
    if (*abort) {
      for (int q = issued - stages > 0 ? issued - stages : 0; q < issued; ++q)
        mbar_wait_bounded(&full[q % stages], (uint32_t)((q / stages) & 1), nullptr, 200000000LL);
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  const int gi = warp / kGroupWarps, gw = warp % kGroupWarps, gt = tid - gi * kGroupThreads;
  const int bar_id = 1 + gi;
  float *gbase = reinterpret_cast<float *>(smem + stages * stage_bytes) + gi * group_floats;
  float *sg = gbase;                          // [hc][WMAX]  ln alpha
  float *sbeta = sg + hc * WMAX;              // [hc][WMAX]
  float *hso = sbeta + hc * WMAX;             // per head: dec[MAXM] | Mk[MAXM][32] | Mq[MAXM][32]
  float *hsf = hso + hc * HS::kOut;           // decf[32] | A[32][32] | T[32][32] | fw[32] | decF | one[3]
  float *wscr = hsf + HS::kFold + gw * HS::kWarp;
  float *U = wscr, *red = wscr + kMaxW * RPW;
  float *odec = hso, *Mk = hso + MAXM, *Mq = Mk + MAXM * 32;   // repointed per head
  float *decf = hsf, *Mf = hsf + kMaxW, *Tm = Mf + kMaxW * kMaxW, *fw = Tm + kMaxW * kMaxW;
  float *decF = fw + kMaxW;
  float *one = decF + 1;   // window-full fold of a 1-entry window after a pre-fold (L = 1):
                           // one[0] = e^{g} (its decf and decF), one[1] = 1 (fw), one[2] = 1 (T)
  const int c0 = lane * 4;
  const int urow0 = gw * RPW;   // first row of this warp inside a unit

  for (int k = gi; k < my_items; k += kGroups) {
    int b, chunk;
    item_of(k, b, chunk);
    const int h0 = chunk * hc;
    const size_t bh0 = (size_t)b * a.H + h0;
    const RowPlan rp = plan_row(a, b);
    const int st = rp.st, n = rp.n;
    const bool pre = rp.pre, post = rp.post;
    if (rp.refuse && rp.bit && chunk == 0 && gt == 0) atomicOr(a.status, rp.bit);
    const int w0 = pre ? n : 0;
    const int ntot = n + m;
    // fold window [f0, f0 + nf): the committed entries (pre) or the full window (post)
    const int f0 = pre ? 0 : w0, nf = pre ? n : n - w0 + 1;

    if (!rp.refuse) {
      // ---- gates and betas of the item's heads; ring appends of new tokens
      for (int idx = gt; idx < hc * ntot; idx += kGroupThreads) {
        const int jh = idx / ntot, i = idx - jh * ntot;
        const size_t bh = bh0 + jh;
        const int slot = (st + i) % cap;
        float g, be;
        if (i < n) {
          g = gring[bh * cap + slot];
          be = bring[bh * cap + slot];
        } else {
          const size_t tok = ((size_t)b * m + (i - n)) * a.H + h0 + jh;
          g = logf(alin[tok]);
          be = bein[tok];
          gring[bh * cap + slot] = g;
          bring[bh * cap + slot] = be;
        }
        sg[jh * WMAX + i] = g;
        sbeta[jh * WMAX + i] = be;
      }
      constexpr int kPer = 16 / sizeof(Tin);
      for (int idx = gt; idx < hc * m * 2 * (DK / kPer); idx += kGroupThreads) {
        const int per = 2 * (DK / kPer);
        const int r = idx / per, c = (idx - r * per) * kPer;   // c in [0, 2*DK): k row then v row
        const int jh = r / m, j = r - jh * m;
        const size_t bh = bh0 + jh;
        const size_t tok = ((size_t)b * m + j) * a.H + h0 + jh;
        const int slot = (st + n + j) % cap;
        if (c < DK) {
          const uint4 raw = __ldg(reinterpret_cast<const uint4 *>(kin + tok * DK + c));
          *reinterpret_cast<uint4 *>(kring + (bh * cap + slot) * DK + c) = raw;
        } else {
          const int cv = c - DK, hf = cv / HALF;
          const uint4 raw = __ldg(reinterpret_cast<const uint4 *>(vin + tok * DV + cv));
          *reinterpret_cast<uint4 *>(vring + ((bh * 2 + hf) * cap + slot) * HALF + (cv - hf * HALF)) = raw;
        }
      }
      named_sync(bar_id, kGroupThreads);
      // ---- output scalars of every head (one warp per head), from the k rows of
      //      the ring and the inputs: for output j (e = n + j) and window entry
      //      i in [w0, e]: Mq_ji = e^{seg(i,e)} k_i.q_j, Mk_ji = e^{seg(i,e)} k_i.k_e
      //      (i < e), 0 elsewhere; dec_j = e^{G}, G the g summed over [w0, e].
      if (m > 0) {
        constexpr int CE = MAXM == 1 ? 8 : 4;   // window entries per reduction
        constexpr int NV = CE * 2 * MAXM;
        for (int jh = gw; jh < hc; jh += kGroupWarps) {
          const size_t bh = bh0 + jh;
          float *hs = hso + jh * HS::kOut;
          float *hMk = hs + MAXM, *hMq = hMk + MAXM * 32;
          float4 qv[MAXM], kv[MAXM];
#pragma unroll
          for (int j = 0; j < MAXM; ++j) {
            const size_t tok = ((size_t)b * m + j) * a.H + h0 + jh;
            qv[j] = j < m ? ld4<Tin>(qin + tok * DK + c0) : make_float4(0.f, 0.f, 0.f, 0.f);
            kv[j] = j < m ? ld4<Tin>(kin + tok * DK + c0) : make_float4(0.f, 0.f, 0.f, 0.f);
          }
          for (int i0 = w0; i0 < ntot; i0 += CE) {
            float part[NV];
#pragma unroll
            for (int c = 0; c < CE; ++c) {
              const int i = i0 + c;
              float4 ki = make_float4(0.f, 0.f, 0.f, 0.f);
              if (i < n)
                ki = ld4<Tin>(kring + (bh * cap + (st + i) % cap) * DK + c0);
              else if (i < ntot)
                ki = ld4<Tin>(kin + (((size_t)b * m + (i - n)) * a.H + h0 + jh) * DK + c0);
#pragma unroll
              for (int j = 0; j < MAXM; ++j) {
                part[(c * MAXM + j) * 2 + 0] = dot4(ki, qv[j]);
                part[(c * MAXM + j) * 2 + 1] = dot4(ki, kv[j]);
              }
            }
            tr_sum<NV, 16>(part, lane);
            const int base = tr_base<NV, 16>(lane);
            constexpr int R = NV >= 32 ? NV / 32 : 1;
            constexpr int DUP = NV >= 32 ? 1 : 32 / NV;
            if ((lane & (DUP - 1)) == 0) {
#pragma unroll
              for (int q = 0; q < R; ++q) {   // raw dots, scaled below by their decays
                const int idx = base + q, which = idx & 1, j = (idx >> 1) % MAXM, c = (idx >> 1) / MAXM;
                const int l = i0 - w0 + c;
                if (l < 32) (which == 0 ? hMq : hMk)[j * 32 + l] = part[q];
              }
            }
          }
          __syncwarp();
          const int l = lane, i = w0 + l;
#pragma unroll
          for (int j = 0; j < MAXM; ++j) {
            const int e = n + j, len = e - w0 + 1;
            const float v = (j < m && l < len) ? sg[jh * WMAX + i] : 0.0f;
            float after, total;
            suffix_scan(v, lane, after, total);
            const float ex = expf(after);
            const bool in = j < m && l < len;
            hMq[j * 32 + l] = in ? ex * hMq[j * 32 + l] : 0.0f;
            hMk[j * 32 + l] = (in && l < len - 1) ? ex * hMk[j * 32 + l] : 0.0f;
            if (lane == 0) hs[j] = j < m ? expf(total) : 0.0f;
          }
        }
      }
      named_sync(bar_id, kGroupThreads);
    }

    // sequence number of this item's unit `unit` in the producer's issue order
    const int pair = k >> 1;
    const bool paired = 2 * pair + 1 < my_items;
    const int seq0 = pair * 4 * hc + (paired ? (k & 1) : 0), step = paired ? 2 : 1;
    int s = seq0 % stages, use = seq0 / stages;   // stage and use of the current unit
    auto wait_stage = [&]() -> bool {
      if (!wait_flag_at_least(&stage_use[s], use, abort)) return false;
      return mbar_wait_bounded(&full[s], (uint32_t)(use & 1), abort);
    };
    auto release_stage = [&]() {
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
    };
    auto next_unit = [&]() {
      s += step;
      if (s >= stages) {
        s -= stages;
        ++use;
      }
    };

    // A failed wait (bounded, or another warp's abort) does not leave the loop:
    // the warp skips its work but passes every group barrier, whose OR
    // reduction spreads the failure, so all warps keep the same barrier sequence.
    bool failed = false;
    for (int jh = 0; jh < hc; ++jh) {
      const int h = h0 + jh;
      const size_t bh = bh0 + jh;
      const float *gw_ = sg + jh * WMAX, *bw_ = sbeta + jh * WMAX;
      odec = hso + jh * HS::kOut;
      Mk = odec + MAXM;
      Mq = Mk + MAXM * 32;
      for (int hf = 0; hf < 2; ++hf, next_unit()) {
        if (rp.refuse) {
          if (!failed && wait_stage()) release_stage();
          else failed = true;
          continue;
        }
        const size_t row_base = bh * DV + hf * HALF;   // first state row of this unit
        float *hc_rows = a.hc + row_base * DK;
        uint8_t *rc = (RF != RSSM_READ_FP32) ? a.rc_codes + row_base * RB : nullptr;
        float4 f[RPW];    // fp32 checkpoint rows for a fold (read-copy layers)
        if constexpr (RF != RSSM_READ_FP32) {
          if (pre || post) {
#pragma unroll
            for (int r = 0; r < RPW; ++r) f[r] = ld_stream(hc_rows + (size_t)(urow0 + r) * DK + c0);
          }
        }
        // fold scalars are single-buffered: all warps must be done with the previous head's
        if (hf == 0 && (pre || post) && named_sync_or(bar_id, kGroupThreads, failed)) failed = true;
        const bool have = !failed && wait_stage();
        if (!have) failed = true;
        const GStage<Tin> stg{smem + s * stage_bytes, KOFF, QOFF, VOFF, WOFF, n, L};

        if (hf == 0 && (pre || post)) {
          // ---- fold scalars (fold heads only): Gram dots k_i'.k_i in 4 x 4 blocks.
          if (have) {
            const int nb = (nf + 3) / 4;
            for (int blk = gw; blk < nb * nb; blk += kGroupWarps) {
              const int bi = blk / nb, bj = blk - bi * nb;
              if (bj > bi) continue;
              float part[16];
              float4 ka[4], kb[4];
#pragma unroll
              for (int c = 0; c < 4; ++c) {
                const int ia = 4 * bi + c, ib = 4 * bj + c;
                ka[c] = ia < nf ? ld4<Tin>(stg.k(f0 + ia) + c0) : make_float4(0.f, 0.f, 0.f, 0.f);
                kb[c] = ib < nf ? ld4<Tin>(stg.k(f0 + ib) + c0) : make_float4(0.f, 0.f, 0.f, 0.f);
              }
#pragma unroll
              for (int ca = 0; ca < 4; ++ca)
#pragma unroll
                for (int cb = 0; cb < 4; ++cb) part[ca * 4 + cb] = dot4(ka[ca], kb[cb]);
              tr_sum<16, 16>(part, lane);
              const int idx = tr_base<16, 16>(lane);
              const int ia = 4 * bi + idx / 4, ib = 4 * bj + idx % 4;
              if ((lane & 1) == 0 && ib < ia && ia < nf) {
                // A[i][i'] = beta_i e^{seg(i', i)} k_i'.k_i (direct sums)
                float sgm = 0.0f;
                for (int r = ib + 1; r <= ia; ++r) sgm += gw_[f0 + r];
                Mf[ia * kMaxW + ib] = bw_[f0 + ia] * expf(sgm) * part[0];
              }
            }
            if (gw == 1 % kGroupWarps) {   // fold weights
              const float v = lane < nf ? gw_[f0 + lane] : 0.0f;
              float after, total;
              suffix_scan(v, lane, after, total);
              fw[lane] = expf(after);
              if (lane == 0) decF[0] = expf(total);
              float pre_sum = 0.0f;   // e^{G_i}: g summed from the window start to entry i
              for (int r = 0; r <= lane && r < nf; ++r) pre_sum += gw_[f0 + r];
              decf[lane] = expf(pre_sum);
              if (pre && post && lane == 0) {   // L = 1: then fold the new entry alone
                one[0] = expf(gw_[n]);
                one[1] = 1.0f;
                one[2] = 1.0f;
              }
            }
          }
          if (named_sync_or(bar_id, kGroupThreads, failed)) failed = true;
          if (!failed && gw == 0) {
            // T = (I + A)^{-1}: unit lower triangular, lane c computes column c
            // by forward substitution (it reads only its own column of T).
            const int c = lane;
            for (int i = 0; i < nf; ++i) {
              float v = i == c ? 1.0f : 0.0f;
              if (i > c) {
                float acc = 0.0f;
                for (int ip = c; ip < i; ++ip) acc = fmaf(Mf[i * kMaxW + ip], Tm[ip * kMaxW + c], acc);
                v = -acc;
              }
              if (c < nf) Tm[i * kMaxW + c] = v;
            }
          }
          if (named_sync_or(bar_id, kGroupThreads, failed)) failed = true;
        }
        if (failed) {
          if (have) release_stage();
          continue;
        }

        // ---- the read view of this warp's 8 rows
        float4 vw[RPW];
        if (pre) {   // new tokens do not fit: fold the committed window first
          if constexpr (RF == RSSM_READ_FP32) {
#pragma unroll
            for (int r = 0; r < RPW; ++r)
              f[r] = *reinterpret_cast<const float4 *>(stg.base + ((size_t)(urow0 + r) * DK + c0) * 4);
          }
          fold_rows<Tin>(f, stg, f0, nf, decf, Tm, fw, decF[0], bw_, urow0, U, lane, c0);
#pragma unroll
          for (int r = 0; r < RPW; ++r) {
            const int row = urow0 + r;
            if (!post) st_stream(hc_rows + (size_t)row * DK + c0, f[r]);
            if constexpr (RF == RSSM_READ_FP32)
              vw[r] = f[r];
            else
              vw[r] = quantize4<RF, 32>(f[r], rc + (size_t)row * RB, a.rc_scales, row_base + row, DK, c0, lane);
          }
        } else {
#pragma unroll
          for (int r = 0; r < RPW; ++r) {
            const int row = urow0 + r;
            if constexpr (RF == RSSM_READ_FP32) {
              vw[r] = *reinterpret_cast<const float4 *>(stg.base + ((size_t)row * DK + c0) * 4);
            } else if constexpr (RF == RSSM_READ_FP8_E4M3_ROW) {
              const uint32_t w = *reinterpret_cast<const uint32_t *>(stg.base + (size_t)row * RB + c0);
              dec_e4m3x4(w, reinterpret_cast<const float *>(stg.base + TB)[row], vw[r]);
            } else {
              const uint32_t w = *reinterpret_cast<const uint16_t *>(stg.base + (size_t)row * RB + c0 / 2);
              const float sc = dec_e4m3(stg.base[TB + row * (DK / 16) + c0 / 16]);
              dec_e2m1x4(w, sc, vw[r]);
            }
          }
        }

        // ---- outputs.  Per row: z_j = dec_j (S k_ej) + sum_{committed i} Mk_ji w_i,
        //      a_j = dec_j (S q_j) + sum_{committed i} Mq_ji w_i, reduced across
        //      the row's lanes; then per row the new w and o in draft order.
        if (m > 0) {
          constexpr int NV = RPW * 2 * MAXM;
          float part[NV];
#pragma unroll
          for (int j = 0; j < MAXM; ++j) {
            const float4 ke = j < m ? ld4<Tin>(stg.k(n + j) + c0) : make_float4(0.f, 0.f, 0.f, 0.f);
            const float4 qj = j < m ? ld4<Tin>(stg.q(j) + c0) : make_float4(0.f, 0.f, 0.f, 0.f);
            const float dj = odec[j < m ? j : 0];
#pragma unroll
            for (int r = 0; r < RPW; ++r) {
              part[(r * MAXM + j) * 2 + 0] = dj * dot4(vw[r], ke);
              part[(r * MAXM + j) * 2 + 1] = dj * dot4(vw[r], qj);
            }
          }
          if (!pre && lane < n) {   // committed entry i = lane (w0 = 0)
            float w8[RPW];
            const float4 wa = reinterpret_cast<const float4 *>(stg.w(lane) + urow0)[0];
            const float4 wb = reinterpret_cast<const float4 *>(stg.w(lane) + urow0)[1];
            w8[0] = wa.x; w8[1] = wa.y; w8[2] = wa.z; w8[3] = wa.w;
            w8[4] = wb.x; w8[5] = wb.y; w8[6] = wb.z; w8[7] = wb.w;
#pragma unroll
            for (int j = 0; j < MAXM; ++j) {
              const float mk = Mk[j * 32 + lane], mq = Mq[j * 32 + lane];
#pragma unroll
              for (int r = 0; r < RPW; ++r) {
                part[(r * MAXM + j) * 2 + 0] = fmaf(mk, w8[r], part[(r * MAXM + j) * 2 + 0]);
                part[(r * MAXM + j) * 2 + 1] = fmaf(mq, w8[r], part[(r * MAXM + j) * 2 + 1]);
              }
            }
          }
          tr_sum<NV, 16>(part, lane);
          const int base = tr_base<NV, 16>(lane);
          constexpr int R = NV >= 32 ? NV / 32 : 1;
          constexpr int DUP = NV >= 32 ? 1 : 32 / NV;
          if constexpr (MAXM == 1) {
            // one token: the lane holds z or a of its row; the other sits in lane ^ 2
            const float other = __shfl_xor_sync(kFull, part[0], 2);
            const int r = base >> 1, which = base & 1, row = urow0 + r, e = n;
            const float z = which == 0 ? part[0] : other, av = which == 0 ? other : part[0];
            const float wv = bw_[e] * (to_f32<Tin>(stg.v(e)[row]) - z);
            if ((lane & 1) == 0) {
              if (which == 0) wring[((bh * 2 + hf) * cap + (st + e) % cap) * HALF + row] = wv;
              else a.out[((size_t)b * a.H + h) * DV + hf * HALF + row] = a.out_scale * fmaf(Mq[e - w0], wv, av);
            }
          } else {
          if ((lane & (DUP - 1)) == 0) {
#pragma unroll
            for (int q = 0; q < R; ++q) red[base + q] = part[q];
          }
          __syncwarp();
          if (lane < RPW) {
            const int r = lane, row = urow0 + r;
            float wn[MAXM];
            for (int j = 0; j < m; ++j) {
              const int e = n + j;
              float acc = to_f32<Tin>(stg.v(e)[row]) - red[(r * MAXM + j) * 2 + 0];
              for (int jp = 0; jp < j; ++jp) acc = fmaf(-Mk[j * 32 + (n + jp - w0)], wn[jp], acc);
              wn[j] = bw_[e] * acc;
              float o = red[(r * MAXM + j) * 2 + 1];
              for (int jp = 0; jp <= j; ++jp) o = fmaf(Mq[j * 32 + (n + jp - w0)], wn[jp], o);
              a.out[(((size_t)b * m + j) * a.H + h) * DV + hf * HALF + row] = a.out_scale * o;
              wring[((bh * 2 + hf) * cap + (st + e) % cap) * HALF + row] = wn[j];
            }
          }
          __syncwarp();
          }
        }

        if (post) {   // the decode filled the window: fold all of it (from fp32)
          if constexpr (RF == RSSM_READ_FP32) {
#pragma unroll
            for (int r = 0; r < RPW; ++r) f[r] = vw[r];
          }
          if (pre)   // L = 1: the window is the new entry alone
            fold_rows<Tin>(f, stg, n, 1, one, one + 2, one + 1, one[0], bw_, urow0, U, lane, c0);
          else
            fold_rows<Tin>(f, stg, f0, nf, decf, Tm, fw, decF[0], bw_, urow0, U, lane, c0);
#pragma unroll
          for (int r = 0; r < RPW; ++r) {
            const int row = urow0 + r;
            st_stream(hc_rows + (size_t)row * DK + c0, f[r]);
            if constexpr (RF != RSSM_READ_FP32)
              quantize4<RF, 32>(f[r], rc + (size_t)row * RB, a.rc_scales, row_base + row, DK, c0, lane);
          }
        }
        release_stage();
      }
    }

    const bool any_abort = named_sync_or(bar_id, kGroupThreads, failed || *abort != 0);
    if (any_abort) {
      if (gt == 0) atomicOr(a.status, (unsigned)RSSM_STATUS_TIMEOUT);
      return;
    }
    if (!rp.refuse && gt == 0) {
      __threadfence();
      if (atomicAdd(a.arrivals + b, 1) == nchunk - 1) {
        a.arrivals[b] = 0;
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
  }
}

// Conventional gated delta rule: per row i of S (16 warps x 8 rows, a lane owns
// 4 columns): u_i = alpha S_i.k, o_i = out_scale (alpha S_i.q + c_i (k.q)),
// S_i <- alpha S_i + c_i k with c_i = beta (v_i - u_i); S written back.
template <typename Tin>
__global__ void __launch_bounds__(512) gdn_conv_kernel(const ConvArgs a) {
  constexpr int R8 = DV / 16;
  __shared__ float s_c[DV], s_kq;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const size_t bh = blockIdx.x;
  const int b = (int)(bh / a.H);
  (void)b;
  const int c0 = lane * 4, row0 = warp * R8;
  const float *S = a.state_in + bh * DV * DK;
  float4 t[R8];
#pragma unroll
  for (int r = 0; r < R8; ++r) t[r] = ld_stream(S + (size_t)(row0 + r) * DK + c0);
  const Tin *q = reinterpret_cast<const Tin *>(a.in[0]) + bh * DK;
  const Tin *k = reinterpret_cast<const Tin *>(a.in[1]) + bh * DK;
  const Tin *v = reinterpret_cast<const Tin *>(a.in[2]) + bh * DV;
  const float alpha = reinterpret_cast<const float *>(a.in[3])[bh];
  const float beta = reinterpret_cast<const float *>(a.in[4])[bh];
  const float4 kc = ld4<Tin>(k + c0), qc = ld4<Tin>(q + c0);
  if (warp == 0) {
    const float kq = warp_sum(dot4(kc, qc));
    if (lane == 0) s_kq = kq;
  }
  float part[R8 * 2];
#pragma unroll
  for (int r = 0; r < R8; ++r) {
    part[r * 2 + 0] = dot4(t[r], kc);
    part[r * 2 + 1] = dot4(t[r], qc);
  }
  tr_sum<R8 * 2, 16>(part, lane);
  const int idx = tr_base<R8 * 2, 16>(lane);
  __syncthreads();   // s_kq
  // lanes holding (row, S.k) compute c; lanes holding (row, S.q) write o
  {
    const int r = idx / 2, which = idx & 1, row = row0 + r;
    const bool writer = (lane & 1) == 0;   // 16 values over 32 lanes: pairs hold copies
    const float dk_ = part[0];
    const float other = __shfl_xor_sync(kFull, dk_, 2);   // partner holding the other value of the row
    const float sk = which == 0 ? dk_ : other, sq = which == 0 ? other : dk_;
    const float u = alpha * sk;
    const float c = beta * (to_f32<Tin>(v[row]) - u);
    if (writer && which == 0) s_c[row] = c;
    if (writer && which == 1) a.out[bh * DV + row] = a.out_scale * (alpha * sq + c * s_kq);
  }
  __syncthreads();
#pragma unroll
  for (int r = 0; r < R8; ++r) {
    scale4(t[r], alpha);
    fma4(t[r], s_c[row0 + r], kc);
    st_stream(a.state_out + bh * DV * DK + (size_t)(row0 + r) * DK + c0, t[r]);
  }
}

template <typename Tin, int RF, int MAXM>
cudaError_t launch_step(const StepArgs &a, cudaStream_t s) {
  using HS = HeadScalars<MAXM>;
  auto kern = gdn_replay_kernel<Tin, RF, MAXM>;
  const size_t esz = sizeof(Tin);
  const size_t krow = DK * esz, vhrow = HALF * esz;
  const size_t stage = ((size_t)tile_bytes<RF>() + scale_bytes<RF>() + (a.L + MAXM) * krow + MAXM * krow +
                        (a.L + MAXM) * vhrow + (size_t)a.L * HALF * 4 + 127) & ~(size_t)127;
  const size_t wmax = a.L + MAXM;
  int dev = 0, sms = 0, max_smem = 0;
  cudaError_t e;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&max_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev)) != cudaSuccess) return e;
  const size_t budget = (size_t)max_smem - 2048;
  // heads per item: the largest divisor of H (at most 16) whose per-head scalars
  // leave room for at least two stages
  int hc = a.H < 16 ? a.H : 16;
  size_t fixed = 0;
  for (;; --hc) {
    if (hc < 1) return cudaErrorInvalidConfiguration;
    if (a.H % hc) continue;
    const size_t group_floats = (2 * hc * wmax + (size_t)hc * HS::kOut + HS::kFold + kGroupWarps * HS::kWarp + 31) & ~(size_t)31;
    fixed = kGroups * sizeof(float) * group_floats;
    if (fixed + 2 * stage <= budget) break;
  }
  int stages = (int)((budget - fixed) / stage);
  if (stages > kMaxStages) stages = kMaxStages;
  const size_t smem = fixed + (size_t)stages * stage;
  if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) != cudaSuccess) return e;
  int per_sm = 0;
  if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kReplayThreads, smem)) != cudaSuccess) return e;
  if (per_sm < 1) return cudaErrorInvalidConfiguration;
  const long long items = (long long)a.B * (a.H / hc);
  const long long slots = (long long)sms * per_sm;
  const unsigned grid = (unsigned)(items < slots ? items : slots);
  kern<<<dim3(grid), dim3(kReplayThreads), smem, s>>>(a, hc, stages);
  return cudaGetLastError();
}

template <typename Tin, int RF>
cudaError_t dispatch_m(const StepArgs &a, cudaStream_t s) {
  if (a.mode != kVerify) return launch_step<Tin, RF, 1>(a, s);
  if (a.m <= 4) return launch_step<Tin, RF, 4>(a, s);
  return launch_step<Tin, RF, 8>(a, s);
}

template <typename Tin>
cudaError_t dispatch_rf(const StepArgs &a, int rf, cudaStream_t s) {
  switch (rf) {
    case RSSM_READ_FP32: return dispatch_m<Tin, RSSM_READ_FP32>(a, s);
    case RSSM_READ_FP8_E4M3_ROW: return dispatch_m<Tin, RSSM_READ_FP8_E4M3_ROW>(a, s);
    default: return dispatch_m<Tin, RSSM_READ_NVFP4>(a, s);
  }
}

}  // namespace

bool gdn_supported(int R, int C) { return R == DV && C == DK; }

cudaError_t gdn_step(const StepArgs &a, int in_dtype, int read_fmt, cudaStream_t s) {
  if (in_dtype == RSSM_BF16) return dispatch_rf<__nv_bfloat16>(a, read_fmt, s);
  return dispatch_rf<float>(a, read_fmt, s);
}

cudaError_t gdn_conventional(const ConvArgs &a, int in_dtype, cudaStream_t s) {
  if (in_dtype == RSSM_BF16)
    gdn_conv_kernel<__nv_bfloat16><<<dim3((unsigned)(a.B * a.H)), dim3(512), 0, s>>>(a);
  else
    gdn_conv_kernel<float><<<dim3((unsigned)(a.B * a.H)), dim3(512), 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace rssm
