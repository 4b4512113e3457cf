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
// recurrence stays in high precision.  A layer that reads the fp32 checkpoint
// solved its cached w against that checkpoint, so its fold is the rank-l
// update with them; a layer that reads a low-precision copy solved its cached
// w against the copy, so its fold solves the window again from the fp32
// checkpoint (UT transform) and the copy's rounding never enters the state.
//
// Work unit: half a head (64 of the 128 value rows, 32 KiB of fp32 state).  A
// persistent CTA has one producer warp, which streams units into rings of
// shared-memory stages with 1-D TMA bulk copies (the read tile and the cached
// w rows; fold units of re-solving layers also the v rows), and two consumer
// groups of 8 warps taking alternate items (item = one sequence and a chunk of
// heads).  Each group has its own ring; the producer serves whichever group
// has a free stage, so one group's item prologue overlaps the other's stream.
// An item's prologue copies the committed window k rows of its heads into
// shared memory (cp.async), loads the gates, converts the new q, k, v rows to
// fp32, appends to the ring and computes every head's window scalars.  Per
// unit each warp owns 8 state rows; a row is spread over 8 lanes (4 chunks of
// 4 columns each), so its dot products reduce in three shuffle steps.
#include "rssm_device.cuh"
#include "umma.cuh"

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
constexpr int kMaxW = 32;                 // window positions a scalar array covers

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
__device__ __forceinline__ float dot4(const float4 a, const float4 b) {
  return a.x * b.x + a.y * b.y + a.z * b.z + a.w * b.w;
}
__device__ __forceinline__ void fma4(float4 &t, float c, const float4 k) {
  t.x = fmaf(c, k.x, t.x); t.y = fmaf(c, k.y, t.y); t.z = fmaf(c, k.z, t.z); t.w = fmaf(c, k.w, t.w);
}
__device__ __forceinline__ void scale4(float4 &t, float c) { t.x *= c; t.y *= c; t.z *= c; t.w *= c; }

// Shared-memory layout of a replay launch (the host sizes the launch with the
// same function).  Stage, in bytes: [read tile | scales | cached w rows (L) |
// v half rows (L + MAXM, fold units of re-solving layers; committed entries
// at rows [0, n), new tokens at L + j)].  Group region, in floats: gates and
// betas of the item's heads, fp32 k/q/v of the new tokens, the committed
// window k rows of the item's heads (input dtype), per-head output scalars,
// fold scalars, per-warp scratch.
// Folds of layers that read the fp32 checkpoint with bf16 inputs run on the
// tensor cores (tcgen05): the rank-l update of a unit, D^T[c][r] =
// sum_i k_i[c] (fw_i w_i[r]), is one M = 128 (key columns) x N = 64 (value
// rows) x K = l bf16 MMA chain per unit with an fp32 accumulator in TMEM.  The
// k rows are bf16 already (exact); each weighted w value is split into three
// bf16 parts (hi, mid, lo; their sum is the fp32 value to 2^-24), so the
// products are exact and only the fp32 accumulation rounds, as on the CUDA
// cores.  The epilogue adds e^{G} S from the stage and stores.
template <typename Tin, int RF>
constexpr bool umma_fold() { return RF == RSSM_READ_FP32 && sizeof(Tin) == 2; }

struct Layout {
  int woff, voff, stage_bytes;
  int sg, sbeta, kqv, kbuf, hso, fold, warp, warp_floats, umma, umma_kg, group_floats;
};
template <typename Tin, int RF, int MAXM>
__host__ __device__ inline Layout make_layout(int L, int hc) {
  constexpr bool kResolve = RF != RSSM_READ_FP32;
  Layout y;
  const int vhrow = HALF * (int)sizeof(Tin);
  y.woff = tile_bytes<RF>() + scale_bytes<RF>();
  y.voff = y.woff + L * HALF * 4;
  y.stage_bytes = (y.voff + (kResolve ? (L + MAXM) * vhrow : 0) + 127) & ~127;
  const int wmax = L + MAXM;
  y.sg = 0;
  y.sbeta = hc * wmax;
  y.kqv = (2 * hc * wmax + 3) & ~3;
  y.kbuf = y.kqv + hc * 3 * MAXM * DK;   // [hc][L][DK] input dtype, 16-byte aligned
  y.hso = y.kbuf + hc * L * DK * (int)sizeof(Tin) / 4;
  y.fold = y.hso + hc * (MAXM + 2 * MAXM * kMaxW);
  // fw[2][kMaxW + 1] | decF[2] | decf[2][kMaxW + 1] | A[L][L] | T[L][L] (A, T: re-solving layers)
  const int fold_floats = 4 * (kMaxW + 1) + 2 + (kResolve ? 2 * L * L : 0);
  y.warp = (y.fold + fold_floats + 3) & ~3;
  // per warp: red[8][MAXM][2] | win[8][MAXM][2] | wnew[MAXM][8] | U[L][8] (re-solving layers)
  y.warp_floats = (5 * MAXM * RPW + (kResolve ? L * RPW : 0) + 3) & ~3;
  // tensor-core fold operands (MN-major bf16 tiles, 128-byte aligned) for one
  // block of 16 window entries: A = their k rows [DK columns x 16], B = three
  // parts of the weighted w [HALF rows x 16]; longer windows go block by block
  y.umma_kg = 2;
  y.umma = (y.warp + kGroupWarps * y.warp_floats + 31) & ~31;
  const int umma_floats = umma_fold<Tin, RF>() ? (DK / 8 + 3 * HALF / 8) * y.umma_kg * 128 / 4 : 0;
  y.group_floats = (y.umma + umma_floats + 31) & ~31;
  return y;
}


// Quantise two state rows held in the 8-lane row mapping (lane j of the row's
// lane group holds columns 32 c + 4 j .. + 3, c = 0..3) into the read copy,
// returning the dequantised values.  FP8: one fp32 scale per row; NVFP4: one
// E4M3 scale per 16 columns (4 lanes of one chunk).
template <int RF>
__device__ __forceinline__ void quantize_rows(const float4 (&x)[2][4], float4 (&out)[2][4], uint8_t *rc,
                                              void *scales, size_t row_base, int row_a, int row_b, int j,
                                              int lane) {
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int row = r == 0 ? row_a : row_b;
    uint8_t *crow = rc + (size_t)row * rc_row_bytes<RF>();
    if constexpr (RF == RSSM_READ_FP8_E4M3_ROW) {
      float am = 0.0f;
#pragma unroll
      for (int c = 0; c < 4; ++c)
        am = fmaxf(am, fmaxf(fmaxf(fabsf(x[r][c].x), fabsf(x[r][c].y)), fmaxf(fabsf(x[r][c].z), fabsf(x[r][c].w))));
      am = group_max<8>(am);
      const float s = am / 448.0f;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t w = 0;
        if (s != 0.0f)
          w = enc_e4m3(x[r][c].x / s) | (enc_e4m3(x[r][c].y / s) << 8) | (enc_e4m3(x[r][c].z / s) << 16) |
              (enc_e4m3(x[r][c].w / s) << 24);
        *reinterpret_cast<uint32_t *>(crow + 32 * c + 4 * j) = w;
        dec_e4m3x4(w, s, out[r][c]);
      }
      if (j == 0) reinterpret_cast<float *>(scales)[row_base + row] = s;
    } else {
#pragma unroll
      for (int c = 0; c < 4; ++c)
        out[r][c] = quantize4<RSSM_READ_NVFP4, 8>(x[r][c], crow, scales, row_base + row, DK, 32 * c + 4 * j, lane);
    }
  }
}

template <typename Tin, int RF, int MAXM>
__global__ void __launch_bounds__(kReplayThreads, 1)
    gdn_replay_kernel(const StepArgs a, const int hc, const int stages) {
  constexpr bool kResolve = RF != RSSM_READ_FP32;
  constexpr int VHROW = HALF * (int)sizeof(Tin);
  constexpr int TB = tile_bytes<RF>();
  constexpr int SB = scale_bytes<RF>();
  constexpr int RB = rc_row_bytes<RF>();
  constexpr int SR = rc_scale_row_bytes<RF>();
  constexpr int HSO = MAXM + 2 * MAXM * kMaxW;   // per head: dec[MAXM] | Mk[MAXM][32] | Mq[MAXM][32]
  constexpr bool kUmma = umma_fold<Tin, RF>();
  constexpr uint32_t kTmemCols = 2 * HALF;        // one 64-column fp32 accumulator per consumer group
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ uint64_t full[kMaxStages], empty[kMaxStages];
  __shared__ uint64_t mma_bar[kGroups];           // tensor-core fold completion, one per group
  __shared__ uint32_t tmem_base;
  __shared__ int abort_flag;
  __shared__ int never_set;                       // the timeout self-test waits for it

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int L = a.L, cap = a.cap, m = a.m, WMAX = L + MAXM;
  const Layout Y = make_layout<Tin, RF, MAXM>(L, hc);
  const int nchunk = a.H / hc;
  const int nitems = a.B * nchunk;
  const int my_items = (int)blockIdx.x < nitems ? (nitems - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;

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
    }
    for (int g = 0; g < kGroups; ++g) mbar_init(&mma_bar[g], 1);
    abort_flag = 0;
    never_set = 0;
    mbar_fence_init();
  }
  if constexpr (kUmma) {
    if (warp == 0) {   // TMEM for both groups' fold accumulators; freed by warp 0 at the end
      umma::alloc(&tmem_base, kTmemCols);
      umma::relinquish();
    }
    umma::fence_before_sync();
  }
  __syncthreads();
  if constexpr (kUmma) umma::fence_after_sync();

  auto item_of = [&](int k, int &b, int &chunk) {
    const int item = (int)blockIdx.x + k * (int)gridDim.x;
    b = item / nchunk;
    chunk = item - b * nchunk;
  };

  if (warp == kConsumers / 32) {
    // ------------------------------------------------------------ producer
    if (lane != 0) return;
    // Each consumer group has its own ring (group 0: stages 0 .. R0 - 1, group 1:
    // stages R0 .. stages - 1; R0 = ceil(stages / 2)) and consumes its units in
    // order: unit t of group g (its item t / 2hc, unit t mod 2hc) uses stage
    // base_g + t mod R_g for the (t / R_g)-th time.  The producer serves
    // whichever group has a free stage, so a group busy in its item prologue
    // holds back only its own ring while the other group's stream goes on.
    const int R0 = (stages + 1) / 2, R1 = stages - R0;
    const int T0 = ((my_items + 1) / 2) * 2 * hc, T1 = (my_items / 2) * 2 * hc;
    int t0 = 0, t1 = 0, pref = 0;
    int b_0 = 0, b_1 = 0, chunk_0 = 0, chunk_1 = 0, cur_0 = -1, cur_1 = -1;
    RowPlan rp_0{}, rp_1{};
    long long idle_since = clock64();
    bool timed_out = false;
    while (t0 < T0 || t1 < T1) {
      // the group to serve: the preferred one if its next stage is free, else the other
      int g = -1;
      for (int q = 0; q < 2 && g < 0; ++q) {
        const int c = pref ^ q;
        const int t = c ? t1 : t0;
        if (t >= (c ? T1 : T0)) continue;
        const int Rc = c ? R1 : R0;
        const int s_ = (c ? R0 : 0) + t % Rc, u_ = t / Rc;
        if (u_ == 0 || mbar_test_wait(&empty[s_], (uint32_t)((u_ - 1) & 1))) g = c;
      }
      if (g < 0) {   // neither group has released a stage yet
        if (*abort || clock64() - idle_since > a.wait_limit) {
          timed_out = true;
          break;
        }
        __nanosleep(20);
        continue;
      }
      idle_since = clock64();
      pref = g ^ 1;   // alternate when both can go
      const int t = g ? t1 : t0;
      const int s = (g ? R0 : 0) + t % (g ? R1 : R0);
      const int kk = t / (2 * hc), unit = t - kk * 2 * hc, kc = 2 * kk + g;
      if (g) {
        ++t1;
        if (kc != cur_1) {
          cur_1 = kc;
          item_of(kc, b_1, chunk_1);
          rp_1 = plan_row(a, b_1);
        }
      } else {
        ++t0;
        if (kc != cur_0) {
          cur_0 = kc;
          item_of(kc, b_0, chunk_0);
          rp_0 = plan_row(a, b_0);
        }
      }
      const int b = g ? b_1 : b_0, chunk = g ? chunk_1 : chunk_0;
      const RowPlan rp = g ? rp_1 : rp_0;
      if (rp.refuse) {
        mbar_arrive(&full[s]);
      } else {
        const int jh = unit >> 1, hf = unit & 1;
        const int h = chunk * hc + jh;
        const size_t bh = (size_t)b * a.H + h, sbh = (size_t)rp.src * a.H + h;
        const bool fold = rp.pre || rp.post;
        // cached w rows: the reads of the committed entries, and the folds of
        // layers that fold with them
        const int nw = (kResolve && rp.pre) ? 0 : rp.n;
        const int nv = (kResolve && fold) ? rp.n : 0;         // v rows of re-solving folds
        const int mv = (kResolve && fold) ? m : 0;
        uint8_t *dst = smem + s * Y.stage_bytes;
        mbar_arrive_expect_tx(&full[s], (uint32_t)(TB + SB + nw * HALF * 4 + (nv + mv) * VHROW));
        if constexpr (RF == RSSM_READ_FP32) {
          bulk_g2s(dst, a.hc + (sbh * DV + hf * HALF) * DK, TB, &full[s]);
        } else {
          bulk_g2s(dst, a.rc_codes + (sbh * DV + hf * HALF) * RB, TB, &full[s]);
          bulk_g2s(dst + TB, reinterpret_cast<const uint8_t *>(a.rc_scales) + (sbh * DV + hf * HALF) * SR, SB, &full[s]);
        }
        const int c1 = rp.n < cap - rp.st ? rp.n : cap - rp.st;   // ring segment lengths
        if (nw > 0) {
          const float *src = wring + (bh * 2 + hf) * cap * HALF;
          const int w1 = nw < c1 ? nw : c1;
          bulk_g2s(dst + Y.woff, src + (size_t)rp.st * HALF, w1 * HALF * 4, &full[s]);
          if (nw > w1) bulk_g2s(dst + Y.woff + w1 * HALF * 4, src, (nw - w1) * HALF * 4, &full[s]);
        }
        if (nv > 0) {
          const Tin *src = vring + (bh * 2 + hf) * cap * HALF;
          bulk_g2s(dst + Y.voff, src + (size_t)rp.st * HALF, c1 * VHROW, &full[s]);
          if (nv > c1) bulk_g2s(dst + Y.voff + c1 * VHROW, src, (nv - c1) * VHROW, &full[s]);
        }
        for (int j = 0; j < mv; ++j) {
          const size_t tok = ((size_t)b * m + j) * a.H + h;
          bulk_g2s(dst + Y.voff + (L + j) * VHROW, vin + tok * DV + hf * HALF, VHROW, &full[s]);
        }
      }
    }
    if (timed_out) {
      *abort = 1;
      atomicOr(a.status, (unsigned)RSSM_STATUS_TIMEOUT);
    }
    if (*abort) {   // let the copies requested on every stage land (bounded) before the CTA retires
      for (int c = 0; c < 2; ++c) {
        const int t = c ? t1 : t0, Rc = c ? R1 : R0;
        for (int q = t - Rc > 0 ? t - Rc : 0; q < t; ++q)
          mbar_wait_bounded(&full[(c ? R0 : 0) + q % Rc], (uint32_t)((q / Rc) & 1), nullptr, 200000000LL);
      }
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  const int gi = warp / kGroupWarps, gw = warp % kGroupWarps, gt = tid - gi * kGroupThreads;
  const int bar_id = 1 + gi;
  float *G = reinterpret_cast<float *>(smem + stages * Y.stage_bytes) + gi * Y.group_floats;
  float *sg = G + Y.sg;          // [hc][WMAX]  ln alpha of the window entries
  float *sbeta = G + Y.sbeta;    // [hc][WMAX]
  float *kqv = G + Y.kqv;        // [hc][k | q | v][MAXM][128]  new tokens, fp32
  Tin *kbuf = reinterpret_cast<Tin *>(G + Y.kbuf);   // [hc][L][128]  committed window k rows
  float *hso = G + Y.hso;        // [hc][HSO]
  float *fw = G + Y.fold;        // [2][kMaxW + 1]  fold weights e^{seg(i, last)}: pre-fold, window-full fold
  float *decF = fw + 2 * (kMaxW + 1);   // [2]  decay over each fold window
  float *decf = decF + 2;        // [2][kMaxW + 1]  e^{G_i} within each fold window (re-solving layers)
  float *Am = decf + 2 * (kMaxW + 1), *Tm = Am + L * L;   // re-solving layers
  float *wscr = G + Y.warp + gw * Y.warp_floats;
  float *red = wscr;                    // [8][MAXM][2]  reduced S.k_e and S.q per row
  float *win = red + 2 * MAXM * RPW;    // [8][MAXM][2]  window sums per row
  float *wnew = win + 2 * MAXM * RPW;   // [MAXM][8]     solved w of the new tokens
  float *U = wnew + MAXM * RPW;         // [L][8]        re-solving folds
  const int c0 = lane * 4;              // full-row mapping (scalars): 4 columns per lane
  const int g8 = lane >> 3, j8 = lane & 7;   // state mapping: rows g8, g8 + 4 of the warp; lane j8 of the row
  const int urow0 = gw * RPW;           // first row of this warp inside a unit
  const int row_a = urow0 + g8, row_b = urow0 + g8 + 4;
  if (a.stall_test && blockIdx.x == 0) {   // the timeout self-test: this CTA's waits run out
    stall_on_unset_flag(&never_set, abort, a.wait_limit);
    if (gt == 0) atomicOr(a.status, (unsigned)RSSM_STATUS_TIMEOUT);
  }


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
    const int slot_n = (st + n) % cap;   // ring slot of the first new entry

    if (!rp.refuse) {
      // ---- committed window k rows of the item's heads into shared memory
      //      (asynchronous copies, in flight while the loads below are made)
      constexpr int kChunks = DK * (int)sizeof(Tin) / 16;   // 16-byte chunks per row
      for (int idx = gt; idx < hc * n * kChunks; idx += kGroupThreads) {
        const int c = idx % kChunks, r = idx / kChunks;
        const int i = r % n, jh = r / n;
        const int slot = (st + i) % cap;
        cp_async16(reinterpret_cast<uint8_t *>(kbuf + ((size_t)jh * L + i) * DK) + 16 * c,
                   reinterpret_cast<const uint8_t *>(kring + ((bh0 + jh) * cap + slot) * DK) + 16 * c);
      }
      // ---- gates and betas of the item's heads (committed from the ring, new
      //      from the inputs: raw alpha, its log is taken below), also in flight
      for (int idx = gt; idx < hc * ntot; idx += kGroupThreads) {
        const int jh = idx / ntot, i = idx - jh * ntot;
        const size_t bh = bh0 + jh;
        const float *gsrc, *bsrc;
        if (i < n) {
          const size_t o = bh * cap + (st + i) % cap;
          gsrc = gring + o;
          bsrc = bring + o;
        } else {
          const size_t tok = ((size_t)b * m + (i - n)) * a.H + h0 + jh;
          gsrc = alin + tok;
          bsrc = bein + tok;
        }
        cp_async4(sg + jh * WMAX + i, gsrc);
        cp_async4(sbeta + jh * WMAX + i, bsrc);
      }
      // ---- new tokens: k, q, v rows to fp32 in shared memory; k and v appended
      //      to the ring.  A thread's 16-byte loads (up to kBatch) are issued before any is used.
      constexpr int kPer = 16 / sizeof(Tin);
      constexpr int kLoads = DK / kPer;   // 16-byte loads per row
      const int ntok = hc * m * 3 * kLoads;
      constexpr int kBatch = MAXM == 1 ? 1 : 4;
      for (int base = 0; base < ntok; base += kBatch * kGroupThreads) {
        uint4 raw[kBatch];
#pragma unroll
        for (int q = 0; q < kBatch; ++q) {
          const int idx = base + q * kGroupThreads + gt;
          if (idx < ntok) {
            const int c = (idx % kLoads) * kPer, r = idx / kLoads, which = r % 3, j = (r / 3) % m, jh = r / 3 / m;
            const size_t tok = ((size_t)b * m + j) * a.H + h0 + jh;
            raw[q] = __ldg(reinterpret_cast<const uint4 *>((which == 0 ? kin : which == 1 ? qin : vin) + tok * DK + c));
          }
        }
#pragma unroll
        for (int q = 0; q < kBatch; ++q) {
          const int idx = base + q * kGroupThreads + gt;
          if (idx >= ntok) continue;
          const int c = (idx % kLoads) * kPer, r = idx / kLoads, which = r % 3, j = (r / 3) % m, jh = r / 3 / m;
          const Tin *e = reinterpret_cast<const Tin *>(&raw[q]);
          float *dst = kqv + ((size_t)(jh * 3 + which) * MAXM + j) * DK + c;
#pragma unroll
          for (int u = 0; u < kPer; u += 4)
            *reinterpret_cast<float4 *>(dst + u) =
                make_float4(to_f32<Tin>(e[u]), to_f32<Tin>(e[u + 1]), to_f32<Tin>(e[u + 2]), to_f32<Tin>(e[u + 3]));
          const size_t bh = bh0 + jh;
          const int slot = (slot_n + j) % cap;
          if (which == 0) {
            *reinterpret_cast<uint4 *>(kring + (bh * cap + slot) * DK + c) = raw[q];
          } else if (which == 2) {
            const int hf = c / HALF;
            *reinterpret_cast<uint4 *>(vring + ((bh * 2 + hf) * cap + slot) * HALF + (c - hf * HALF)) = raw[q];
          }
        }
      }
      cp_async_wait_all();
      named_sync(bar_id, kGroupThreads);
      // ---- the new gates: ln alpha, appended with the betas to the ring (read
      //      by the decays after the next group barrier)
      for (int idx = gt; idx < hc * m; idx += kGroupThreads) {
        const int jh = idx / m, j = idx - jh * m, i = n + j;
        const size_t o = (bh0 + jh) * cap + (slot_n + j) % cap;
        const float g = logf(sg[jh * WMAX + i]);
        sg[jh * WMAX + i] = g;
        gring[o] = g;
        bring[o] = sbeta[jh * WMAX + i];
      }
      // ---- raw dots k_i.q_j and k_i.k_ej of every head and window entry i in
      //      [w0, n + j], in tasks (head, batch of CE entries) over the warps
      if (m > 0) {
        constexpr int CE = MAXM == 1 ? 8 : 4;   // window entries per reduction
        constexpr int NV = CE * 2 * MAXM;
        const int nbatch = (ntot - w0 + CE - 1) / CE;
        for (int t = gw; t < hc * nbatch; t += kGroupWarps) {
          const int jh = t % hc, i0 = w0 + (t / hc) * CE;
          float *hMk = hso + jh * HSO + MAXM, *hMq = hMk + MAXM * kMaxW;
          const float *hk = kqv + (size_t)jh * 3 * MAXM * DK, *hq = hk + MAXM * DK;
          const Tin *kb = kbuf + (size_t)jh * L * DK;
          float part[NV];
#pragma unroll
          for (int c = 0; c < CE; ++c) {
            const int i = i0 + c;
            float4 ki = make_float4(0.f, 0.f, 0.f, 0.f);
            if (i < n)
              ki = ld4<Tin>(kb + (size_t)i * DK + c0);
            else if (i < ntot)
              ki = *reinterpret_cast<const float4 *>(hk + (i - n) * DK + c0);
#pragma unroll
            for (int j = 0; j < MAXM; ++j) {
              const float4 qv = j < m ? *reinterpret_cast<const float4 *>(hq + j * DK + c0) : make_float4(0.f, 0.f, 0.f, 0.f);
              const float4 kv = j < m ? *reinterpret_cast<const float4 *>(hk + j * DK + c0) : make_float4(0.f, 0.f, 0.f, 0.f);
              part[(c * MAXM + j) * 2 + 0] = dot4(ki, qv);
              part[(c * MAXM + j) * 2 + 1] = dot4(ki, kv);
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
              if (l < kMaxW) (which == 0 ? hMq : hMk)[j * kMaxW + l] = part[q];
            }
          }
        }
        named_sync(bar_id, kGroupThreads);
        // ---- decays (one warp per head and token): for output j (e = n + j) and
        //      window entry i in [w0, e]: Mq_ji = e^{seg(i,e)} k_i.q_j, Mk_ji =
        //      e^{seg(i,e)} k_i.k_e (i < e), 0 elsewhere; dec_j = e^{G}, G the g
        //      summed over [w0, e].
        for (int t = gw; t < hc * MAXM; t += kGroupWarps) {
          const int jh = t / MAXM, j = t - jh * MAXM;
          float *hs = hso + jh * HSO;
          float *hMk = hs + MAXM, *hMq = hMk + MAXM * kMaxW;
          const int l = lane, e = n + j, len = e - w0 + 1;
          const bool in = j < m && l < len;
          const float v = in ? sg[jh * WMAX + w0 + l] : 0.0f;
          float after, total;
          suffix_scan(v, lane, after, total);
          const float ex = expf(after);
          hMq[j * kMaxW + l] = in ? ex * hMq[j * kMaxW + l] : 0.0f;
          hMk[j * kMaxW + l] = (in && l < len - 1) ? ex * hMk[j * kMaxW + l] : 0.0f;
          if (lane == 0) hs[j] = j < m ? expf(total) : 0.0f;
        }
        named_sync(bar_id, kGroupThreads);
      }
    }

    // stage and use of unit 2 jh + hf of this item in the group's own ring (the
    // group's units in order: t = (k / 2) 2hc + 2 jh + hf)
    const int R0 = (stages + 1) / 2, Rg = gi ? stages - R0 : R0, base = gi ? R0 : 0;
    int s = 0, use = 0;
    auto locate = [&](int jh, int hf) {
      const int t = (k >> 1) * 2 * hc + 2 * jh + hf;
      s = base + t % Rg;
      use = t / Rg;
    };
    auto wait_stage = [&]() -> bool { return warp_all(mbar_wait_bounded(&full[s], (uint32_t)(use & 1), abort, a.wait_limit)); };
    auto release_stage = [&]() {
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
    };
    // fold windows: pre-fold = committed entries [0, n); window-full fold = [w0, n]
    const int nf0 = n, nf1 = n - w0 + 1;

    // A failed wait (bounded, or another warp's abort) does not leave the loop:
    // the warp skips its work but passes every group barrier, whose OR
    // reduction spreads the failure, so all warps keep the same barrier sequence.
    bool failed = false;
    int mma_uses = 0;   // completed tensor-core folds of this group (parity of mma_bar[gi])
    for (int jh = 0; jh < hc; ++jh) {
      const int h = h0 + jh;
      const size_t bh = bh0 + jh;
      const float *gw_ = sg + jh * WMAX, *bw_ = sbeta + jh * WMAX;
      const float *odec = hso + jh * HSO, *Mk = odec + MAXM, *Mq = Mk + MAXM * kMaxW;
      const float *hk = kqv + (size_t)jh * 3 * MAXM * DK, *hq = hk + MAXM * DK, *hv = hq + MAXM * DK;
      for (int hf = 0; hf < 2; ++hf) {
        locate(jh, hf);
        if (rp.refuse) {
          if (!failed && wait_stage()) release_stage();
          else failed = true;
          continue;
        }
        // first state row of this unit in the checkpoint slot read (src) and in
        // the one a fold writes (dst)
        const size_t src_base = ((size_t)rp.src * a.H + h) * DV + hf * HALF;
        const size_t row_base = ((size_t)rp.dst * a.H + h) * DV + hf * HALF;
        const float *hc_src = a.hc + src_base * DK;
        float *hc_rows = a.hc + row_base * DK;
        uint8_t *rc = kResolve ? a.rc_codes + row_base * RB : nullptr;
        float4 f[2][4];   // fp32 state rows (fp32 layers: the tile; re-solving layers: fold units)
        if constexpr (kResolve) {
          if (pre || post) {
#pragma unroll
            for (int r = 0; r < 2; ++r)
#pragma unroll
              for (int c = 0; c < 4; ++c)
                f[r][c] = ld_stream(hc_src + (size_t)(r == 0 ? row_a : row_b) * DK + 32 * c + 4 * j8);
          }
        }
        // fold scalars are single-buffered: all warps must be done with the previous head's
        if (hf == 0 && (pre || post) && named_sync_or(bar_id, kGroupThreads, failed)) failed = true;
        const bool have = !failed && wait_stage();
        if (!have) failed = true;
        // a tensor-core fold has group barriers inside: every warp must agree on doing it
        if (kUmma && hf == 1 && (pre || post) && named_sync_or(bar_id, kGroupThreads, failed)) failed = true;
        bool released = false;
        const uint8_t *sb = smem + s * Y.stage_bytes;
        const float *wst = reinterpret_cast<const float *>(sb + Y.woff);   // cached w, committed entries
        const Tin *kb = kbuf + (size_t)jh * L * DK;
        // k_i[col .. col + 3]: committed entries from the item's k rows, new ones (fp32)
        auto kval4 = [&](int i, int col) -> float4 {
          return i < n ? ld4<Tin>(kb + (size_t)i * DK + col) : *reinterpret_cast<const float4 *>(hk + (i - n) * DK + col);
        };
        auto vrow = [&](int i) -> const Tin * {
          return reinterpret_cast<const Tin *>(sb + Y.voff) + (size_t)(i < n ? i : L + (i - n)) * HALF;
        };

        if (hf == 0 && (pre || post)) {
          // ---- fold scalars of this head: weights and decays of both fold
          //      windows, and the Gram dots of a re-solved window
          if (have) {
            if (gw == 1 && pre) {   // pre-fold window [0, n)
              const float v = lane < nf0 ? gw_[lane] : 0.0f;
              float after, total;
              suffix_scan(v, lane, after, total);
              fw[lane] = expf(after);
              if (lane == 0) decF[0] = expf(total);
              if constexpr (kResolve) {
                float ps = 0.0f;   // e^{G_i}: g summed from the window start through entry i
                for (int r = 0; r <= lane && r < nf0; ++r) ps += gw_[r];
                decf[lane] = expf(ps);
              }
            }
            if (gw == 2 && post) {   // window-full fold [w0, n]
              const float v = lane < nf1 ? gw_[w0 + lane] : 0.0f;
              float after, total;
              suffix_scan(v, lane, after, total);
              fw[kMaxW + 1 + lane] = expf(after);
              if (lane == 0) decF[1] = expf(total);
              if constexpr (kResolve) {
                float ps = 0.0f;
                for (int r = 0; r <= lane && r < nf1; ++r) ps += gw_[w0 + r];
                decf[kMaxW + 1 + lane] = expf(ps);
              }
            }
            if constexpr (kResolve) {
              // Gram dots of the re-solved window in 4 x 4 blocks:
              // A[i][i'] = beta_i e^{seg(i', i)} k_i'.k_i (i' < i, direct sums).  A
              // decode that folds twice (L = 1) re-solves two 1-entry windows (T = 1).
              const int rf0 = pre ? 0 : w0, rnf = pre ? nf0 : nf1;
              const int nb = (rnf + 3) / 4;
              for (int blk = gw; blk < nb * nb; blk += kGroupWarps) {
                const int bi = blk / nb, bj = blk - bi * nb;
                if (bj > bi) continue;
                float part[16];
                float4 ka[4], kb_[4];
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                  const int ia = 4 * bi + c, ib = 4 * bj + c;
                  ka[c] = ia < rnf ? kval4(rf0 + ia, c0) : make_float4(0.f, 0.f, 0.f, 0.f);
                  kb_[c] = ib < rnf ? kval4(rf0 + ib, c0) : make_float4(0.f, 0.f, 0.f, 0.f);
                }
#pragma unroll
                for (int ca = 0; ca < 4; ++ca)
#pragma unroll
                  for (int cb = 0; cb < 4; ++cb) part[ca * 4 + cb] = dot4(ka[ca], kb_[cb]);
                tr_sum<16, 16>(part, lane);
                const int idx = tr_base<16, 16>(lane);
                const int ia = 4 * bi + idx / 4, ib = 4 * bj + idx % 4;
                if ((lane & 1) == 0 && ib < ia && ia < rnf) {
                  float sgm = 0.0f;
                  for (int r = ib + 1; r <= ia; ++r) sgm += gw_[rf0 + r];
                  Am[ia * L + ib] = bw_[rf0 + ia] * expf(sgm) * part[0];
                }
              }
            }
          }
          if (named_sync_or(bar_id, kGroupThreads, failed)) failed = true;
          if constexpr (kResolve) {
            if (!failed && gw == 0) {
              // T = (I + A)^{-1}: unit lower triangular, lane c computes column c
              // by forward substitution (it reads only its own column of T).
              const int rnf = pre ? nf0 : nf1, c = lane;
              for (int i = 0; i < rnf; ++i) {
                float v = i == c ? 1.0f : 0.0f;
                if (i > c) {
                  float acc = 0.0f;
                  for (int ip = c; ip < i; ++ip) acc = fmaf(Am[i * L + ip], Tm[ip * L + c], acc);
                  v = -acc;
                }
                if (c < rnf) Tm[i * L + c] = v;
              }
            }
            if (named_sync_or(bar_id, kGroupThreads, failed)) failed = true;
          }
        }
        if (failed) {
          if (have) release_stage();
          continue;
        }

        // ---- folds.  x <- decF x + sum_i fw_i w_i[row] k_i^T over the window
        //      [i0, i0 + nf).  Layers that read the fp32 checkpoint take the w
        //      cached in the ring (the new entry's from this warp's scratch);
        //      re-solving layers first solve w from x by the UT transform:
        //      u_i = x k_i, r_i = beta_i (v_i - e^{G_i} u_i), w = T r.
        auto fold = [&](float4 (&x)[2][4], int i0, int nf, int which) {
          const float *fwv = fw + which * (kMaxW + 1);
          if constexpr (kResolve) {
            const float *dfv = decf + which * (kMaxW + 1);
            for (int ch = 0; ch < nf; ch += 4) {   // U[i][row] = x_row . k_i, 4 entries per reduction
              float part[8];
#pragma unroll
              for (int c = 0; c < 4; ++c) {
                const int i = ch + c;
                float za = 0.0f, zb = 0.0f;
                if (i < nf) {
#pragma unroll
                  for (int cc = 0; cc < 4; ++cc) {
                    const float4 k4 = kval4(i0 + i, 32 * cc + 4 * j8);
                    za += dot4(x[0][cc], k4);
                    zb += dot4(x[1][cc], k4);
                  }
                }
                part[c] = za;
                part[4 + c] = zb;
              }
              tr_sum<8, 4>(part, lane);
              const int idx = tr_base<8, 4>(lane), r = idx >> 2, i = ch + (idx & 3);
              if (i < nf) U[i * RPW + g8 + 4 * r] = part[0];
            }
            __syncwarp();
            for (int p = lane; p < nf * RPW; p += 32) {   // r_i per (entry, row); U[i][r] layout
              const int i = p / RPW, r8 = p - i * RPW;
              U[p] = bw_[i0 + i] * fmaf(-dfv[i], U[p], to_f32<Tin>(vrow(i0 + i)[urow0 + r8]));
            }
            __syncwarp();
            constexpr int kPer = kMaxW * RPW / 32;
            float wv[kPer];
            const float *Tw = (pre && post && which == 1) ? fwv : Tm;   // L = 1: T = 1 (= fw_0)
#pragma unroll
            for (int q = 0; q < kPer; ++q) {
              const int p = lane + 32 * q, i = p / RPW, r8 = p - i * RPW;
              float acc = 0.0f;
              if (i < nf)
                for (int ip = 0; ip <= i; ++ip) acc = fmaf(Tw[i * L + ip], U[ip * RPW + r8], acc);
              wv[q] = acc;
            }
            __syncwarp();
#pragma unroll
            for (int q = 0; q < kPer; ++q)
              if (lane + 32 * q < nf * RPW) U[lane + 32 * q] = wv[q];
            __syncwarp();
          }
          const float dF = decF[which];
#pragma unroll
          for (int r = 0; r < 2; ++r)
#pragma unroll
            for (int c = 0; c < 4; ++c) scale4(x[r][c], dF);
          for (int i = 0; i < nf; ++i) {
            const int e = i0 + i;
            float wa, wb;
            if constexpr (kResolve) {
              wa = U[i * RPW + g8];
              wb = U[i * RPW + g8 + 4];
            } else if (e < n) {
              wa = wst[e * HALF + row_a];
              wb = wst[e * HALF + row_b];
            } else {
              wa = wnew[(e - n) * RPW + g8];
              wb = wnew[(e - n) * RPW + g8 + 4];
            }
            const float cf = fwv[i];
            wa *= cf;
            wb *= cf;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              const float4 k4 = kval4(e, 32 * c + 4 * j8);
              fma4(x[0][c], wa, k4);
              fma4(x[1][c], wb, k4);
            }
          }
          if constexpr (kResolve) __syncwarp();   // U is reused by the next fold
        };

        // ---- tensor-core fold of the unit's 64 rows by the whole group: x <- decF x +
        //      sum_i fw_i w_i[row] k_i^T over the window [i0, i0 + nf), as D^T[c][r] =
        //      sum_i k_i[c] (fw_i w_i[r]) (M = 128 key columns, N = 64 rows, K = the
        //      entries, zero padded to 16 per MMA step).  Operands: A = the k rows
        //      (bf16, exact), B = three bf16 parts of fw_i w_i[r], each warp writing its
        //      own 8 rows.  The epilogue thread of key column c adds decF S[r][c] from
        //      the stage for 32 rows r and stores the result to the stage (to_stage:
        //      a pre-fold whose result the outputs read) and/or to the checkpoint.
        auto fold_tc = [&](int i0, int nf, int which, bool to_stage, bool to_global) {
          const float *fwv = fw + which * (kMaxW + 1);
          constexpr int KG = 2, KE = 16;
          uint8_t *uA = reinterpret_cast<uint8_t *>(G + Y.umma);
          uint8_t *uB = uA + (DK / 8) * KG * 128;
          constexpr int partB = (HALF / 8) * KG * 128;
          const uint32_t tm = tmem_base + (uint32_t)(gi * HALF);
          for (int blk = 0; blk < nf; blk += KE) {   // blocks of 16 entries, accumulated in TMEM
            for (int idx = gt; idx < KE * (DK / 8); idx += kGroupThreads) {
              const int i = idx / (DK / 8), cc = idx - i * (DK / 8);
              uint4 val = make_uint4(0u, 0u, 0u, 0u);
              if (blk + i < nf) {
                const int e = i0 + blk + i;
                if (e < n) {
                  val = *reinterpret_cast<const uint4 *>(kb + (size_t)e * DK + 8 * cc);
                } else {   // a new token's k (bf16 values widened exactly): back to bf16
                  const float4 lo4 = *reinterpret_cast<const float4 *>(hk + (e - n) * DK + 8 * cc);
                  const float4 hi4 = *reinterpret_cast<const float4 *>(hk + (e - n) * DK + 8 * cc + 4);
                  const __nv_bfloat162 p0 = __floats2bfloat162_rn(lo4.x, lo4.y), p1 = __floats2bfloat162_rn(lo4.z, lo4.w);
                  const __nv_bfloat162 p2 = __floats2bfloat162_rn(hi4.x, hi4.y), p3 = __floats2bfloat162_rn(hi4.z, hi4.w);
                  val = make_uint4(*reinterpret_cast<const uint32_t *>(&p0), *reinterpret_cast<const uint32_t *>(&p1),
                                   *reinterpret_cast<const uint32_t *>(&p2), *reinterpret_cast<const uint32_t *>(&p3));
                }
              }
              *reinterpret_cast<uint4 *>(uA + umma::mn_offset(8 * cc, i, KG)) = val;
            }
            for (int p = lane; p < KE * RPW; p += 32) {
              const int i = p >> 3, r8 = p & 7;
              float x = 0.0f;
              if (blk + i < nf) {
                const int e = i0 + blk + i;
                x = fwv[blk + i] * (e < n ? wst[e * HALF + urow0 + r8] : wnew[(e - n) * RPW + r8]);
              }
              uint16_t xh, xm, xl;
              umma::split3_bf16(x, xh, xm, xl);
              const uint32_t off = umma::mn_offset(urow0 + r8, i, KG);
              *reinterpret_cast<uint16_t *>(uB + off) = xh;
              *reinterpret_cast<uint16_t *>(uB + partB + off) = xm;
              *reinterpret_cast<uint16_t *>(uB + 2 * partB + off) = xl;
            }
            fence_proxy_async();   // operands written by this thread -> visible to the tensor core
            umma::fence_before_sync();
            named_sync(bar_id, kGroupThreads);
            if (gt == 0) {
              umma::fence_after_sync();
              constexpr uint32_t idesc = umma::idesc_bf16_f32_mn(DK, HALF);
              const uint64_t ad = umma::smem_desc_mn(smem_u32(uA), 128, KG * 128);
              for (int part = 0; part < 3; ++part)
                umma::mma_bf16(tm, ad, umma::smem_desc_mn(smem_u32(uB + part * partB), 128, KG * 128), idesc,
                               part > 0 || blk > 0);
              umma::commit(&mma_bar[gi]);
            }
            // the MMAs always complete: wait without the abort flag (bounded), so
            // that TMEM and the operands are never reused under a running MMA
            const bool ok = warp_all(mbar_wait_bounded(&mma_bar[gi], (uint32_t)(mma_uses & 1), nullptr, kDefaultWaitLimit));
            ++mma_uses;
            umma::fence_after_sync();
            if (!ok) {
              *abort = 1;
              failed = true;
              return;
            }
          }
          const int q = gw & 3, c = 32 * q + lane, rh = (gw >> 2) * 32;
          float d[32];
          umma::ld_32x32b_x32(tm + ((uint32_t)(32 * q) << 16) + (uint32_t)rh, d);
          umma::fence_before_sync();
          const float dF = decF[which];
          float *tile = reinterpret_cast<float *>(const_cast<uint8_t *>(sb));
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int r = rh + j;
            const float val = fmaf(dF, tile[r * DK + c], d[j]);
            if (to_stage) tile[r * DK + c] = val;
            if (to_global) __stcs(hc_rows + (size_t)r * DK + c, val);
          }
        };

        // ---- the read view of this warp's rows, after a pre-fold if one is due
        float4 v[2][4];   // read view (re-solving layers); fp32 layers read f
        if constexpr (kUmma) {
          if (pre) {   // the new tokens do not fit: fold the committed window first, into the stage
            fold_tc(0, nf0, 0, true, !post);
            if (named_sync_or(bar_id, kGroupThreads, failed)) failed = true;   // the folded tile is complete
            if (failed) {
              if (have) release_stage();
              continue;
            }
          }
        }
        if constexpr (!kResolve) {
          const float *tile = reinterpret_cast<const float *>(sb);
#pragma unroll
          for (int r = 0; r < 2; ++r)
#pragma unroll
            for (int c = 0; c < 4; ++c)
              f[r][c] = *reinterpret_cast<const float4 *>(tile + (size_t)(r == 0 ? row_a : row_b) * DK + 32 * c + 4 * j8);
        }
        if (!kUmma && pre) {   // the new tokens do not fit: fold the committed window first
          fold(f, 0, nf0, 0);
#pragma unroll
          for (int r = 0; r < 2; ++r)
#pragma unroll
            for (int c = 0; c < 4; ++c)
              if (!post) st_stream(hc_rows + (size_t)(r == 0 ? row_a : row_b) * DK + 32 * c + 4 * j8, f[r][c]);
          if constexpr (kResolve) quantize_rows<RF>(f, v, rc, a.rc_scales, row_base, row_a, row_b, j8, lane);
        } else if constexpr (kResolve) {
#pragma unroll
          for (int r = 0; r < 2; ++r) {
            const int row = r == 0 ? row_a : row_b;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              if constexpr (RF == RSSM_READ_FP8_E4M3_ROW) {
                const uint32_t w = *reinterpret_cast<const uint32_t *>(sb + (size_t)row * RB + 32 * c + 4 * j8);
                dec_e4m3x4(w, reinterpret_cast<const float *>(sb + TB)[row], v[r][c]);
              } else {
                const uint32_t w = *reinterpret_cast<const uint16_t *>(sb + (size_t)row * RB + 16 * c + 2 * j8);
                dec_e2m1x4(w, dec_e4m3(sb[TB + row * (DK / 16) + 2 * c + (j8 >> 2)]), v[r][c]);
              }
            }
          }
        }

        // ---- outputs.  Per row and token j: z = dec_j (S k_ej) + sum_i Mk_ji w_i,
        //      a = dec_j (S q_j) + sum_i Mq_ji w_i over the committed entries i;
        //      then per row the new w and o in draft order.
        if (m > 0) {
          float wz[MAXM], wa[MAXM];   // window sums: lane = (entry group lane >> 3, row lane & 7)
#pragma unroll
          for (int j = 0; j < MAXM; ++j) wz[j] = wa[j] = 0.0f;
          if (!pre) {
            for (int i = lane >> 3; i < n; i += 4) {
              const float wv = wst[i * HALF + urow0 + (lane & 7)];
#pragma unroll
              for (int j = 0; j < MAXM; ++j) {
                wz[j] = fmaf(Mk[j * kMaxW + i], wv, wz[j]);
                wa[j] = fmaf(Mq[j * kMaxW + i], wv, wa[j]);
              }
            }
          }
          if (!post) {   // the last read of the stage: hand it back to the producer
            release_stage();
            released = true;
          }
          constexpr int NV = 4 * MAXM;   // (row r, token j, z|a) -> (r * MAXM + j) * 2 + which
          float part[NV];
#pragma unroll
          for (int j = 0; j < MAXM; ++j) {
            float za = 0.0f, zb = 0.0f, aa = 0.0f, ab = 0.0f;
            if (j < m) {
#pragma unroll
              for (int c = 0; c < 4; ++c) {
                const float4 k4 = *reinterpret_cast<const float4 *>(hk + j * DK + 32 * c + 4 * j8);
                const float4 q4 = *reinterpret_cast<const float4 *>(hq + j * DK + 32 * c + 4 * j8);
                if constexpr (kResolve) {
                  za += dot4(v[0][c], k4); zb += dot4(v[1][c], k4);
                  aa += dot4(v[0][c], q4); ab += dot4(v[1][c], q4);
                } else {
                  za += dot4(f[0][c], k4); zb += dot4(f[1][c], k4);
                  aa += dot4(f[0][c], q4); ab += dot4(f[1][c], q4);
                }
              }
            }
            part[j * 2 + 0] = za;
            part[j * 2 + 1] = aa;
            part[(MAXM + j) * 2 + 0] = zb;
            part[(MAXM + j) * 2 + 1] = ab;
          }
#pragma unroll
          for (int j = 0; j < MAXM; ++j) {   // sum the window terms over the 4 entry groups
            wz[j] += __shfl_xor_sync(kFull, wz[j], 8);
            wa[j] += __shfl_xor_sync(kFull, wa[j], 8);
            wz[j] += __shfl_xor_sync(kFull, wz[j], 16);
            wa[j] += __shfl_xor_sync(kFull, wa[j], 16);
          }
          tr_sum<NV, 4>(part, lane);   // over the 8 lanes of each row
          {
            const int base = tr_base<NV, 4>(lane);
            constexpr int R = NV >= 8 ? NV / 8 : 1;
            constexpr int DUP = NV >= 8 ? 1 : 8 / NV;
            if ((lane & (DUP - 1)) == 0) {
#pragma unroll
              for (int q = 0; q < R; ++q) {
                const int idx = base + q, r = idx / (2 * MAXM), jw = idx - r * 2 * MAXM;
                red[(g8 + 4 * r) * 2 * MAXM + jw] = part[q];
              }
            }
            if (lane < RPW) {
#pragma unroll
              for (int j = 0; j < MAXM; ++j) {
                win[lane * 2 * MAXM + 2 * j + 0] = wz[j];
                win[lane * 2 * MAXM + 2 * j + 1] = wa[j];
              }
            }
          }
          __syncwarp();
          if (lane < RPW) {
            const int r8 = lane, row = urow0 + r8;
            float wn[MAXM];
#pragma unroll
            for (int j = 0; j < MAXM; ++j) {
              if (j >= m) break;
              const int e = n + j;
              const float dj = odec[j];
              const float z = fmaf(dj, red[r8 * 2 * MAXM + 2 * j], win[r8 * 2 * MAXM + 2 * j]);
              float acc = hv[j * DK + hf * HALF + row] - z;
              for (int jp = 0; jp < j; ++jp) acc = fmaf(-Mk[j * kMaxW + (n + jp - w0)], wn[jp], acc);
              wn[j] = bw_[e] * acc;
              float o = fmaf(dj, red[r8 * 2 * MAXM + 2 * j + 1], win[r8 * 2 * MAXM + 2 * j + 1]);
              for (int jp = 0; jp <= j; ++jp) o = fmaf(Mq[j * kMaxW + (n + jp - w0)], wn[jp], o);
              a.out[(((size_t)b * m + j) * a.H + h) * DV + hf * HALF + row] = a.out_scale * o;
              int slot = slot_n + j;
              if (slot >= cap) slot -= cap;
              wring[((bh * 2 + hf) * cap + slot) * HALF + row] = wn[j];
              wnew[j * RPW + r8] = wn[j];
            }
          }
          __syncwarp();
        }

        if (kUmma && post) {   // the decode filled the window: fold all of it (tensor cores)
          fold_tc(w0, nf1, 1, false, true);
        } else if (post) {   // the decode filled the window: fold all of it
          fold(f, w0, nf1, 1);
#pragma unroll
          for (int r = 0; r < 2; ++r)
#pragma unroll
            for (int c = 0; c < 4; ++c)
              st_stream(hc_rows + (size_t)(r == 0 ? row_a : row_b) * DK + 32 * c + 4 * j8, f[r][c]);
          if constexpr (kResolve) quantize_rows<RF>(f, v, rc, a.rc_scales, row_base, row_a, row_b, j8, lane);
        }
        if (!released) release_stage();
      }
    }

    const bool any_abort = named_sync_or(bar_id, kGroupThreads, failed || *abort != 0);
    if (any_abort) {
      if (gt == 0) atomicOr(a.status, (unsigned)RSSM_STATUS_TIMEOUT);
      break;   // every consumer thread still meets the others at the TMEM release below
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
  if constexpr (kUmma) {   // both groups are done with their accumulators
    umma::fence_before_sync();
    named_sync(3, kConsumers);
    if (warp == 0) {
      umma::fence_after_sync();
      umma::dealloc(tmem_base, kTmemCols);
    }
  }
}

// Conventional gated delta rule: per row i of S (16 warps x 8 rows, a lane owns
// 4 columns): u_i = alpha S_i.k, o_i = out_scale (alpha S_i.q + c_i (k.q)),
// S_i <- alpha S_i + c_i k with c_i = beta (v_i - u_i); S written back.  SF
// (state format): fp32, or a state kept in low precision (FP8 row / NVFP4,
// read-copy layout), decoded, updated in fp32 and rounded again every token
// (o comes from the updated fp32 values before that rounding).
template <typename Tin, int SF>
__global__ void __launch_bounds__(512) gdn_conv_kernel(const ConvArgs a) {
  constexpr int R8 = DV / 16;
  __shared__ float s_c[DV], s_kq;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const size_t bh = blockIdx.x;
  const int b = (int)(bh / a.H);
  (void)b;
  const int c0 = lane * 4, row0 = warp * R8;
  constexpr int RB = rc_row_bytes<SF>();
  float4 t[R8];
#pragma unroll
  for (int r = 0; r < R8; ++r) {
    const size_t row = bh * DV + row0 + r;
    if constexpr (SF == RSSM_READ_FP32)
      t[r] = ld_stream(a.state_in + row * DK + c0);
    else
      t[r] = load_read_copy4<SF>(a.codes_in + row * RB, a.scales_in, row, DK, c0);
  }
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
    const size_t row = bh * DV + row0 + r;
    if constexpr (SF == RSSM_READ_FP32)
      st_stream(a.state_out + row * DK + c0, t[r]);
    else
      quantize4<SF, 32>(t[r], a.codes_out + row * RB, a.scales_out, row, DK, c0, lane);
  }
}

template <typename Tin, int RF, int MAXM>
cudaError_t launch_step(const StepArgs &a, cudaStream_t s) {
  auto kern = gdn_replay_kernel<Tin, RF, MAXM>;
  int dev = 0, sms = 0, max_smem = 0;
  cudaError_t e;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&max_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev)) != cudaSuccess) return e;
  const size_t budget = (size_t)max_smem - 2048;
  // Heads per item: the divisor of H (at most 8) with the lowest cost on the
  // busiest CTA (one CTA per SM): its items times (2 units per head + about 4
  // units' worth of item prologue, which both consumer groups run at the same
  // time), raised when the layout leaves fewer than 4 stages (fp32 reads at
  // L = 16: 4 heads per item with 4 stages; measured against 2 heads per item
  // at L = 32, 4 heads with 3 stages was 11% faster).
  int hc = 0, stages = 0;
  double best_cost = 0.0;
  for (int c = a.H < 8 ? a.H : 8; c >= 1; --c) {
    if (a.H % c) continue;
    const Layout y = make_layout<Tin, RF, MAXM>(a.L, c);
    const size_t fixed = (size_t)kGroups * sizeof(float) * y.group_floats;
    if (fixed + 2 * (size_t)y.stage_bytes > budget) continue;   // at least one stage per group ring
    int st = (int)((budget - fixed) / y.stage_bytes);
    if (st > kMaxStages) st = kMaxStages;
    const long long items = (long long)a.B * (a.H / c);
    double cost = (double)((items + sms - 1) / sms) * (2 * c + 4);
    if (st < 4) cost *= 4.0 / st;
    if (hc == 0 || cost < best_cost) {
      hc = c;
      stages = st;
      best_cost = cost;
    }
  }
  if (hc == 0) return cudaErrorInvalidConfiguration;
  const Layout y = make_layout<Tin, RF, MAXM>(a.L, hc);
  const size_t smem = (size_t)kGroups * sizeof(float) * y.group_floats + (size_t)stages * y.stage_bytes;
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

template <int SF>
cudaError_t launch_conv(const ConvArgs &a, int in_dtype, cudaStream_t s) {
  if (in_dtype == RSSM_BF16)
    gdn_conv_kernel<__nv_bfloat16, SF><<<dim3((unsigned)(a.B * a.H)), dim3(512), 0, s>>>(a);
  else
    gdn_conv_kernel<float, SF><<<dim3((unsigned)(a.B * a.H)), dim3(512), 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace

bool gdn_supported(int R, int C) { return R == DV && C == DK; }

cudaError_t gdn_step(const StepArgs &a, int in_dtype, int read_fmt, cudaStream_t s) {
  if (gdn_decode_fast_path(a, in_dtype, read_fmt)) return gdn_decode_step(a, s);
  if (in_dtype == RSSM_BF16) return dispatch_rf<__nv_bfloat16>(a, read_fmt, s);
  return dispatch_rf<float>(a, read_fmt, s);
}

cudaError_t gdn_conventional(const ConvArgs &a, int in_dtype, int state_fmt, cudaStream_t s) {
  switch (state_fmt) {
    case RSSM_READ_FP32: return launch_conv<RSSM_READ_FP32>(a, in_dtype, s);
    case RSSM_READ_FP8_E4M3_ROW: return launch_conv<RSSM_READ_FP8_E4M3_ROW>(a, in_dtype, s);
    default: return launch_conv<RSSM_READ_NVFP4>(a, in_dtype, s);
  }
}

}  // namespace rssm
