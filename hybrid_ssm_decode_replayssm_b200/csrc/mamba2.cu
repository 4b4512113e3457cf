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
// The replay kernel streams each head's checkpoint tile (or its read copy)
// through shared memory with 1-D TMA bulk copies, several heads in flight per
// CTA; see m2_replay_kernel.  The conventional kernel keeps one CTA per
// (sequence, head) and holds the tile in registers.
#include <algorithm>

#include "m2_common.cuh"
#include "rssm_device.cuh"
#include "umma.cuh"

namespace rssm {
namespace {

// Decode heads of read-copy layers (bf16 inputs, headdim 64, dstate 128) take
// the tensor-core path: y = h C as mma.sync m16n8k16 (f16 x f16 -> fp32), one
// warp per 16-row tile, four warps per head.  The dequantised codes are exact
// in f16 (an E2M1 value times an E4M3 scale has at most 6 significant bits and
// lies in [2^-10, 2688]; an E4M3 code is exact and its fp32 row scale is
// applied to the result); C is scaled by a power of two so that max |C| lies
// in [2^14, 2^15) before rounding to f16, which keeps every bf16 bit of the
// values within 2^15 of the largest.  The products are exact in fp32.
template <int P, int N, typename Tin, int RF, int MAXM>
constexpr bool mma_read() {
  return RF != RSSM_READ_FP32 && sizeof(Tin) == 2 && MAXM == 1 && P == 64 && N == 128;
}
template <int P, int N, typename Tin, int RF, int MAXM>
constexpr int mma_floats() { return mma_read<P, N, Tin, RF, MAXM>() ? N / 2 + 4 : 0; }   // C as f16, 1/scale

// Folds of layers that read the fp32 checkpoint with bf16 inputs (headdim 64,
// dstate 128) run on the tensor cores (tcgen05): the rank-l update of a head,
// D^T[n][p] = sum_i B_i[n] (fw_i x_i[p]), is an M = 128 (dstate) x N = 64
// (headdim) x K = l bf16 MMA chain with an fp32 accumulator in TMEM, 16 window
// entries per block.  B rows are bf16 already (exact); each weighted x value
// is split into three bf16 parts (hi, mid, lo; their sum is the fp32 value to
// 2^-24), so the products are exact and only the fp32 accumulation rounds, as
// on the CUDA cores.  The epilogue adds e^{G} h from the stage and stores.
template <int P, int N, typename Tin, int RF>
constexpr bool umma_fold() { return RF == RSSM_READ_FP32 && sizeof(Tin) == 2 && P == 64 && N == 128; }
template <int P, int N, typename Tin, int RF>
constexpr int umma_floats() { return umma_fold<P, N, Tin, RF>() ? (N / 8 + 3 * P / 8) * 2 * 128 / 4 : 0; }

// Floats of one consumer group's shared-memory region (host and device agree):
// B window and C rows, dt windows, B.C, per-head scalars, the f16 C of the
// read-copy tensor-core path, then the fold operands (128-byte aligned).
template <int P, int N, typename Tin, int RF, int MAXM>
__host__ __device__ constexpr int group_mma_off(int L, int hc) {
  return ((L + MAXM) * N + MAXM * N + hc * (L + MAXM) + MAXM * (L + MAXM) + hc * (MAXM * 32 + MAXM + 64 + 2) + 3) & ~3;
}

constexpr int kGroupWarps = 8;                  // consumer warps sharing one head
constexpr int kGroups = 2;                      // consumer groups, alternating items
constexpr int kGroupThreads = kGroupWarps * 32;
constexpr int kConsumers = kGroups * kGroupThreads;
constexpr int kReplayThreads = kConsumers + 32; // + one producer warp
constexpr int kMaxStages = 16;
constexpr int kPairSlots = 32;                  // > 1 + kMaxStages / 2 pairs in flight

// The replay kernel: persistent and warp-specialised.  CTA c works through the
// items c, c + grid, ... where an item is one (sequence b, group g, chunk of
// `hc` heads); consumer group k % 2 takes item k.  The heads of the CTA's
// items are numbered in the producer's issue order (seq: pairs of items, see
// the producer), stage = seq % stages, use u = seq / stages.
//  * Producer warp (one lane): for each head in sequence, waits until the
//    consumers have released its stage (empty barrier, phase u - 1), then
//    requests with 1-D TMA bulk copies the head's read tile (fp32, or FP8/NVFP4
//    codes and scales), its committed window rows of x and the new tokens' x
//    rows, all completing on the stage's full barrier.  It reads each item's
//    ring pointers itself, ahead of the consumers.
//  * Two consumer groups of 8 warps take alternate items, so that one group's
//    item prologue (pointers, B window, C rows, B.C products, dt windows, every
//    head's window scalars) overlaps the other group's heads.  Per head, each
//    warp of the group takes P/8 rows: optional pre-fold, outputs (window
//    terms merged into the row reductions), optional window-full fold; then it
//    releases the stage.  There is no block-wide barrier after the start.
template <int P, int N, typename Tin, int RF, int MAXM>
__global__ void __launch_bounds__(kReplayThreads, 1)
    m2_replay_kernel(const StepArgs a, const int hc, const int stages) {
  using T = Tile<P, N, kGroupWarps>;
  constexpr int XROW = P * (int)sizeof(Tin);
  constexpr int TB = tile_bytes<RF, P, N>();
  constexpr int SB = scale_bytes<RF, P, N>();
  constexpr int RB = rc_row_bytes<RF, N>();
  constexpr int HS = MAXM * 32 + MAXM + 64 + 2;   // per-head scalars
  constexpr bool kUmma = umma_fold<P, N, Tin, RF>();
  constexpr uint32_t kTmemCols = kGroups * P;     // one P-column fp32 accumulator per consumer group
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ uint64_t full[kMaxStages], empty[kMaxStages];
  __shared__ uint64_t mma_bar[kGroups];           // tensor-core fold completion, one per group
  __shared__ uint32_t tmem_base;
  // stage_use[s] = the use index u the producer last requested on stage s.  A
  // parity wait is exact only when the waiter is at most one phase ahead of
  // the barrier; a consumer group that skips the other group's item could be
  // further ahead, so it first waits for stage_use[s] == u.
  __shared__ int stage_use[kMaxStages];
  __shared__ int abort_flag;
  __shared__ int never_set;                       // the timeout self-test waits for it
  // pair_inter[p % kPairSlots]: the heads of the CTA's items 2p and 2p + 1
  // alternate in the issue order (both items fold).  The producer decides it
  // before issuing the pair's first head, when no item of the pair has been
  // processed (so the pair's ring pointers cannot have moved), and publishes
  // it before that head's stage_use; a consumer reads it after seeing that
  // stage_use.  The producer cannot run kPairSlots pairs ahead of a reader:
  // it stays within `stages` heads of the oldest unreleased one.
  __shared__ int pair_inter[kPairSlots];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int L = a.L, cap = a.cap, m = a.m, WMAX = L + MAXM;
  const int nchunk = a.hpg / hc;
  const int nitems = a.B * a.G * nchunk;
  const int my_items = (int)blockIdx.x < nitems ? (nitems - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
  const int total_seq = my_items * hc;
  const int XOFF = TB + SB;
  const size_t stage_bytes = ((size_t)XOFF + (size_t)(L + MAXM) * XROW + 127) & ~(size_t)127;
  // each group's region starts on a 128-byte boundary (float4 reads of B and C rows)
  constexpr bool kMma = mma_read<P, N, Tin, RF, MAXM>();
  constexpr int kUnitWarps = kMma ? 4 : kGroupWarps;   // warps that work on (and release) one head
  const int mma_off = group_mma_off<P, N, Tin, RF, MAXM>(L, hc);
  const int umma_off = (mma_off + mma_floats<P, N, Tin, RF, MAXM>() + 31) & ~31;
  const int group_floats = (umma_off + umma_floats<P, N, Tin, RF>() + 31) & ~31;

  const Tin *xin = reinterpret_cast<const Tin *>(a.in[0]);
  const Tin *Bin = reinterpret_cast<const Tin *>(a.in[1]);
  const Tin *Cin = reinterpret_cast<const Tin *>(a.in[2]);
  const Tin *dtin = reinterpret_cast<const Tin *>(a.in[3]);
  Tin *xring = reinterpret_cast<Tin *>(a.buf0);
  volatile int *abort = &abort_flag;

  auto item_of = [&](int k, int &b, int &g, int &chunk) {
    const int item = (int)blockIdx.x + k * (int)gridDim.x;
    b = item / (a.G * nchunk);
    const int rem = item - b * a.G * nchunk;
    g = rem / nchunk;
    chunk = rem - g * nchunk;
  };
  if (tid == 0) {
    for (int s = 0; s < stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kUnitWarps);
      stage_use[s] = -1;
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

  if (warp == kConsumers / 32) {
    // ------------------------------------------------------------ producer
    if (lane != 0) return;
    // Issue order, per pair of items (2p, 2p + 1): the heads of item 2p, then of
    // item 2p + 1 (one group's item prologue overlaps the other group's heads);
    // when both items fold, their heads alternate so that both groups compute.
    int p = 0, w = 0;   // pair and position in the pair of unit seq
    int cur_p = -1, b = 0, g = 0, chunk = 0, jh = 0, s = 0, u = 0, b_o = 0, g_o = 0, chunk_o = 0;
    bool inter = false;
    RowPlan rp{}, rp_e{}, rp_o{};   // current item; the pair's even and odd items
    int b_e = 0, g_e = 0, chunk_e = 0;
    int issued = 0;
    for (int seq = 0; seq < total_seq; ++seq) {
      if (u > 0 && !mbar_wait_bounded(&empty[s], (uint32_t)((u - 1) & 1), abort, a.wait_limit)) {
        atomicOr(a.status, (unsigned)RSSM_STATUS_TIMEOUT);
        break;
      }
      if (w == 2 * hc) {   // next pair
        w = 0;
        ++p;
      }
      if (p != cur_p) {
        cur_p = p;
        item_of(2 * p, b_e, g_e, chunk_e);
        rp_e = plan_row(a, b_e);
        const bool has_odd = 2 * p + 1 < my_items;
        if (has_odd) {
          item_of(2 * p + 1, b_o, g_o, chunk_o);
          rp_o = plan_row(a, b_o);
        }
        inter = has_odd && (rp_e.pre || rp_e.post) && (rp_o.pre || rp_o.post);
        *reinterpret_cast<volatile int *>(&pair_inter[p % kPairSlots]) = inter ? 1 : 0;
        __threadfence_block();   // visible before this head's stage_use
      }
      const bool odd = inter ? (w & 1) != 0 : w >= hc;
      jh = inter ? (w >> 1) : (odd ? w - hc : w);
      b = odd ? b_o : b_e;
      g = odd ? g_o : g_e;
      chunk = odd ? chunk_o : chunk_e;
      rp = odd ? rp_o : rp_e;
      issued = seq + 1;
      if (rp.refuse) {
        mbar_arrive(&full[s]);
      } else {
        const int h = g * a.hpg + chunk * hc + jh;
        const size_t bh = (size_t)b * a.H + h, sbh = (size_t)rp.src * a.H + h;
        uint8_t *dst = smem + s * stage_bytes;
        mbar_arrive_expect_tx(&full[s], (uint32_t)(TB + SB + (m + rp.n) * XROW));
        if constexpr (RF == RSSM_READ_FP32) {
          bulk_g2s(dst, a.hc + sbh * P * N, TB, &full[s]);
        } else {
          bulk_g2s(dst, a.rc_codes + sbh * TB, TB, &full[s]);
          bulk_g2s(dst + TB, reinterpret_cast<const uint8_t *>(a.rc_scales) + sbh * SB, SB, &full[s]);
        }
        if (rp.n > 0) {
          const Tin *src = xring + bh * cap * P;
          const int c1 = rp.n < cap - rp.st ? rp.n : cap - rp.st;
          bulk_g2s(dst + XOFF, src + (size_t)rp.st * P, c1 * XROW, &full[s]);
          if (rp.n > c1) bulk_g2s(dst + XOFF + c1 * XROW, src, (rp.n - c1) * XROW, &full[s]);
        }
        for (int j = 0; j < m; ++j)
          bulk_g2s(dst + XOFF + (L + j) * XROW, xin + (((size_t)b * m + j) * a.H + h) * P, XROW, &full[s]);
      }
      *reinterpret_cast<volatile int *>(&stage_use[s]) = u;
      ++w;
      if (++s == stages) {
        s = 0;
        ++u;
      }
    }
    if (*abort) {   // let requested copies land (bounded) before the CTA can retire
      for (int q = issued - stages > 0 ? issued - stages : 0; q < issued; ++q)
        mbar_wait_bounded(&full[q % stages], (uint32_t)((q / stages) & 1), nullptr, 200000000LL);
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  const int gi = warp / kGroupWarps, gw = warp % kGroupWarps, gt = tid - gi * kGroupThreads;
  const int bar_id = 1 + gi;
  float *sB = reinterpret_cast<float *>(smem + stages * stage_bytes) + gi * group_floats;  // [WMAX][N]
  float *sC = sB + WMAX * N;                                           // [MAXM][N]
  float *sdt = sC + MAXM * N;                                          // [hc][WMAX]
  float *sBC = sdt + hc * WMAX;                                        // [MAXM][WMAX]
  float *ssc = sBC + MAXM * WMAX;                                      // [hc][HS]
  __half *sCh = reinterpret_cast<__half *>(sB + mma_off);              // [N] C as f16 (tensor-core path)
  float *sCinv = sB + mma_off + N / 2;                                 // 1 / its power-of-two scale
  const int sub = kMma ? (gw >> 2) : 0;   // tensor-core path: 4-warp half of the group, alternate heads
  const int c0 = (lane % T::LPR) * 4;
  int mma_uses = 0;   // completed tensor-core folds of this group (parity of mma_bar[gi])
  if (a.stall_test && blockIdx.x == 0) {   // the timeout self-test: this CTA's waits run out
    stall_on_unset_flag(&never_set, abort, a.wait_limit);
    if (gt == 0) atomicOr(a.status, (unsigned)RSSM_STATUS_TIMEOUT);
  }
  for (int k = gi; k < my_items; k += kGroups) {
    int b, g, chunk;
    item_of(k, b, g, chunk);
    const int h0 = g * a.hpg + chunk * hc;
    const size_t bh0 = (size_t)b * a.H + h0;
    Tin *Bring = reinterpret_cast<Tin *>(a.buf1) + ((size_t)b * a.G + g) * cap * N;
    const RowPlan rp = plan_row(a, b);
    const int st = rp.st, n = rp.n;
    const bool pre = rp.pre, post = rp.post;
    if (rp.refuse && rp.bit && g == 0 && chunk == 0 && gt == 0) atomicOr(a.status, rp.bit);
    const int w0 = pre ? n : 0;
    const int ntot = n + m;

    if (!rp.refuse) {
      // ---- group data: B window and C rows (fp32), dt windows, ring appends
      constexpr int kPer = 16 / sizeof(Tin);
      for (int idx = gt; idx < ntot * (N / kPer); idx += kGroupThreads) {
        const int i = idx / (N / kPer), c = (idx - i * (N / kPer)) * kPer;
        const Tin *src = i < n ? Bring + (size_t)((st + i) % cap) * N + c
                               : Bin + (((size_t)b * m + (i - n)) * a.G + g) * N + c;
        const uint4 raw = __ldg(reinterpret_cast<const uint4 *>(src));
        const Tin *e = reinterpret_cast<const Tin *>(&raw);
#pragma unroll
        for (int q = 0; q < kPer; ++q) sB[i * N + c + q] = to_f32<Tin>(e[q]);
        if (i >= n && chunk == 0)
          *reinterpret_cast<uint4 *>(Bring + (size_t)((st + i) % cap) * N + c) = raw;
      }
      for (int idx = gt; idx < MAXM * N; idx += kGroupThreads) {
        const int j = idx / N, c = idx - j * N;
        sC[idx] = j < m ? to_f32<Tin>(Cin[(((size_t)b * m + j) * a.G + g) * N + c]) : 0.0f;
      }
      for (int idx = gt; idx < hc * ntot; idx += kGroupThreads) {
        const int jh = idx / ntot, i = idx - jh * ntot;
        const size_t bh = bh0 + jh;
        float v;
        if (i < n) {
          v = a.buf2[bh * cap + (st + i) % cap];
        } else {
          v = to_f32<Tin>(dtin[((size_t)b * m + (i - n)) * a.H + h0 + jh]);
          a.buf2[bh * cap + (st + i) % cap] = v;
        }
        sdt[jh * WMAX + i] = v;
      }
      for (int idx = gt; idx < hc * m * (P / kPer); idx += kGroupThreads) {
        const int jh = idx / (m * (P / kPer)), r = idx - jh * (m * (P / kPer));
        const int j = r / (P / kPer), c = (r - j * (P / kPer)) * kPer;
        const uint4 raw = __ldg(reinterpret_cast<const uint4 *>(xin + (((size_t)b * m + j) * a.H + h0 + jh) * P + c));
        *reinterpret_cast<uint4 *>(xring + ((bh0 + jh) * cap + (st + n + j) % cap) * P + c) = raw;
      }
      named_sync(bar_id, kGroupThreads);
      for (int p = gw; p < m * ntot; p += kGroupWarps) {
        const int j = p / ntot, i = p - j * ntot;
        if (i < w0 || i > n + j) continue;
        float acc = 0.0f;
        for (int c = lane; c < N; c += 32) acc = fmaf(sB[i * N + c], sC[j * N + c], acc);
        acc = warp_sum(acc);
        if (lane == 0) sBC[j * WMAX + i] = acc;
      }
      if constexpr (kMma) {
        if (gw == kGroupWarps - 1) {   // C as f16, scaled so that max |C| is in [2^14, 2^15)
          float cm = 0.0f;
          for (int c = lane; c < N; c += 32) cm = fmaxf(cm, fabsf(sC[c]));
          cm = group_max<32>(cm);
          const int e = cm > 0.0f ? 14 - ilogbf(cm) : 0;
          for (int c = lane; c < N; c += 32) sCh[c] = __float2half_rn(ldexpf(sC[c], e));
          if (lane == 0) *sCinv = ldexpf(1.0f, -e);
        }
      }
      named_sync(bar_id, kGroupThreads);
      // ---- window scalars of every head: per (head, task) one warp.  Output j:
      //      coef_ji = e^{A seg(i, e_j)} dt_i (B_i . C_j) for i in [w0, e_j] (0
      //      after e_j), dec_j = e^{A G_j}.  Folds: weights e^{A seg(i, last)} dt_i.
      //      Segment sums are warp suffix sums of the dt (direct sums).
      for (int t = gw; t < hc * (MAXM + 2); t += kGroupWarps) {
        const int jh = t / (MAXM + 2), task = t - jh * (MAXM + 2);
        float *hs = ssc + jh * HS;
        int i0, len;
        if (task < MAXM) {
          if (task >= m) {   // unused output slot: zero coefficients and decay
            hs[task * 32 + lane] = 0.0f;
            if (lane == 0) hs[MAXM * 32 + task] = 0.0f;
            continue;
          }
          i0 = w0; len = n + task - w0 + 1;
        } else if (task == MAXM) {
          if (!pre) continue;
          i0 = 0; len = n;
        } else {
          if (!post) continue;
          i0 = w0; len = n - w0 + 1;
        }
        const float Ah = __ldg(a.A + h0 + jh);
        const float v = lane < len ? sdt[jh * WMAX + i0 + lane] : 0.0f;
        float after, total;
        suffix_scan(v, lane, after, total);
        const float wgt = expf(Ah * after) * v;
        if (task < MAXM) {
          hs[task * 32 + lane] = lane < len ? wgt * sBC[task * WMAX + i0 + lane] : 0.0f;
          if (lane == 0) hs[MAXM * 32 + task] = expf(Ah * total);
        } else {
          const int q = task - MAXM;
          hs[MAXM * 32 + MAXM + q * 32 + lane] = wgt;
          if (lane == 0) hs[MAXM * 32 + MAXM + 64 + q] = expf(Ah * total);
        }
      }
      named_sync(bar_id, kGroupThreads);
    }

    // ---- heads: every warp of the group works on its rows.  Head jh is number
    //      2 p hc + (2 jh + (k & 1) | (k & 1) hc + jh) in the producer's issue
    //      order (p = k / 2; interleaved when both items of the pair fold).
    const int seq_base = (k >> 1) * 2 * hc;
    int s = seq_base % stages, use = seq_base / stages;
    bool inter = false;
    if (warp_all(wait_flag_at_least(&stage_use[s], use, abort, a.wait_limit))) {   // the pair's first head is issued
      __threadfence_block();
      inter = *reinterpret_cast<volatile int *>(&pair_inter[(k >> 1) % kPairSlots]) != 0;
    }
    // wait until the producer has requested use `use` of stage s, then for the data
    auto wait_stage = [&]() -> bool {
      if (!warp_all(wait_flag_at_least(&stage_use[s], use, abort, a.wait_limit))) return false;
      return warp_all(mbar_wait_bounded(&full[s], (uint32_t)(use & 1), abort, a.wait_limit));
    };
    constexpr int hstep = kMma ? 2 : 1;   // heads taken by this warp: sub, sub + hstep, ...
    {
      const int seq = seq_base + (inter ? 2 * sub + (k & 1) : (k & 1) * hc + sub);   // its first head
      s = seq % stages;
      use = seq / stages;
    }
    const int step = (inter ? 2 : 1) * hstep;
    // tensor-core path: the B fragments (C as f16, column 0) for the item, in
    // the permuted k order: thread (g, t) holds C[32 t + 4 ks .. + 3]
    uint32_t bfr[kMma ? 16 : 1];
    float cinv = 0.0f;
    if constexpr (kMma) {
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        uint2 v = make_uint2(0u, 0u);
        if ((lane >> 2) == 0 && !rp.refuse)
          v = *reinterpret_cast<const uint2 *>(sCh + 32 * (lane & 3) + 4 * ks);
        bfr[2 * ks] = v.x;
        bfr[2 * ks + 1] = v.y;
      }
      if (!rp.refuse) cinv = *sCinv;
    }
    for (int jh = sub; jh < hc; jh += hstep, s += step) {
      const int h = h0 + jh;
      while (s >= stages) {
        s -= stages;
        ++use;
      }
      if (rp.refuse) {
        if (!wait_stage()) break;
      } else {
        // checkpoint slots: read (src) and written by a fold (dst)
        const size_t sbh = (size_t)rp.src * a.H + h, dbh = (size_t)rp.dst * a.H + h;
        const float *hc_src = a.hc + sbh * P * N;
        float *hc_dst = a.hc + dbh * P * N;
        uint8_t *rc = (RF != RSSM_READ_FP32) ? a.rc_codes + dbh * TB : nullptr;
        const float *hs = ssc + jh * HS;
        const float *hcoef = hs, *hdec = hs + MAXM * 32, *hfw = hs + MAXM * 32 + MAXM;
        const float *hdecf = hfw + 64;
        {
          const bool got = wait_stage();
          // a tensor-core fold has group barriers inside: every warp must agree on doing it
          if (kUmma && (pre || post)) {
            if (named_sync_or(bar_id, kGroupThreads, !got)) break;
          } else if (!got) {
            break;
          }
        }
        const Stage stg{smem + s * stage_bytes, XOFF, XROW, n, L};
        bool done = false;
        if constexpr (kUmma) {
          // ---- tensor-core fold of the head by the whole group: h <- dec h +
          //      sum_i x_i (fw_i B_i)^T over the window [i0, i0 + nf), as D^T[n][p] =
          //      sum_i B_i[n] (fw_i x_i[p]), 16 entries per MMA block.  Operands:
          //      A = the B rows (bf16, exact), B = three bf16 parts of fw_i x_i[p],
          //      each warp writing its own 8 rows p.  The epilogue thread of state
          //      column n adds dec h[p][n] from the stage for 32 rows p and stores the
          //      result to the stage (to_stage: a pre-fold the outputs read) and/or
          //      to the checkpoint.  Returns false if the MMA never completed.
          auto fold_tc = [&](int i0, int nf, const float *fwv, float dec, bool to_stage, bool to_global) -> bool {
            constexpr int KG = 2, KE = 16;
            uint8_t *uA = reinterpret_cast<uint8_t *>(sB + umma_off);
            uint8_t *uB = uA + (N / 8) * KG * 128;
            constexpr int partB = (P / 8) * KG * 128;
            const uint32_t tm = tmem_base + (uint32_t)(gi * P);
            for (int blk = 0; blk < nf; blk += KE) {
              for (int idx = gt; idx < KE * (N / 8); idx += kGroupThreads) {
                const int i = idx / (N / 8), cc = idx - i * (N / 8);
                uint4 val = make_uint4(0u, 0u, 0u, 0u);
                if (blk + i < nf) {   // B row (bf16 values widened exactly in sB): back to bf16
                  const float *src = sB + (i0 + blk + i) * N + 8 * cc;
                  const float4 lo4 = *reinterpret_cast<const float4 *>(src);
                  const float4 hi4 = *reinterpret_cast<const float4 *>(src + 4);
                  const __nv_bfloat162 p0 = __floats2bfloat162_rn(lo4.x, lo4.y), p1 = __floats2bfloat162_rn(lo4.z, lo4.w);
                  const __nv_bfloat162 p2 = __floats2bfloat162_rn(hi4.x, hi4.y), p3 = __floats2bfloat162_rn(hi4.z, hi4.w);
                  val = make_uint4(*reinterpret_cast<const uint32_t *>(&p0), *reinterpret_cast<const uint32_t *>(&p1),
                                   *reinterpret_cast<const uint32_t *>(&p2), *reinterpret_cast<const uint32_t *>(&p3));
                }
                *reinterpret_cast<uint4 *>(uA + umma::mn_offset(8 * cc, i, KG)) = val;
              }
              for (int q = lane; q < KE * T::RPW; q += 32) {
                const int i = q >> 3, r8 = q & 7, p = gw * T::RPW + r8;
                const float x = blk + i < nf ? fwv[blk + i] * stg.x<Tin>(i0 + blk + i, p) : 0.0f;
                uint16_t xh, xm, xl;
                umma::split3_bf16(x, xh, xm, xl);
                const uint32_t off = umma::mn_offset(p, i, KG);
                *reinterpret_cast<uint16_t *>(uB + off) = xh;
                *reinterpret_cast<uint16_t *>(uB + partB + off) = xm;
                *reinterpret_cast<uint16_t *>(uB + 2 * partB + off) = xl;
              }
              fence_proxy_async();   // operands written by this thread -> visible to the tensor core
              umma::fence_before_sync();
              named_sync(bar_id, kGroupThreads);
              if (gt == 0) {
                umma::fence_after_sync();
                constexpr uint32_t idesc = umma::idesc_bf16_f32_mn(N, P);
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
                return false;
              }
            }
            const int q = gw & 3, c = 32 * q + lane, rh = (gw >> 2) * 32;
            float d[32];
            umma::ld_32x32b_x32(tm + ((uint32_t)(32 * q) << 16) + (uint32_t)rh, d);
            umma::fence_before_sync();
            float *tile = reinterpret_cast<float *>(stg.base);
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const int p = rh + j;
              const float val = fmaf(dec, tile[p * N + c], d[j]);
              if (to_stage) tile[p * N + c] = val;
              if (to_global) __stcs(hc_dst + (size_t)p * N + c, val);
            }
            return true;
          };
          bool okf = true;
          if (pre) {   // the new tokens do not fit: fold the committed window first, into the stage
            okf = fold_tc(0, n, hfw, hdecf[0], true, !post);
            if (named_sync_or(bar_id, kGroupThreads, !okf)) break;   // the folded tile is complete
          }
          const int row0 = gw * T::RPW + lane / T::LPR;
          float4 v[T::NLD];
#pragma unroll
          for (int l = 0; l < T::NLD; ++l)
            v[l] = *reinterpret_cast<const float4 *>(stg.base + ((size_t)(row0 + l * T::RPI) * N + c0) * 4);
          if (m > 0)
            outputs<P, N, kGroupWarps, Tin, MAXM>(v, a, sC, hcoef, hdec, stg, b, h, n, w0, row0, lane, c0);
          if (post) {  // the decode filled the window: fold all of it
            const bool okp = fold_tc(w0, n - w0 + 1, hfw + 32, hdecf[1], false, true);
            if (named_sync_or(bar_id, kGroupThreads, !okp)) break;
          }
          done = true;
        }
        if constexpr (kMma) {
          if (!pre && !post) {   // ---- tensor-core read: this warp's 16-row tile
            const int mt = gw & 3, g8 = lane >> 2, t4 = lane & 3;
            const int ra = mt * 16 + g8, rb = ra + 8;
            float d[4] = {0.0f, 0.0f, 0.0f, 0.0f};
            uint32_t af[4];
            if constexpr (RF == RSSM_READ_NVFP4) {
              // thread t4 holds bytes [16 t4, 16 t4 + 16) of its rows: k-step ks uses
              // bytes 2 ks (k pair t4) and 2 ks + 1 (k pair t4 + 4); scale block
              // 2 t4 + ks / 4
              const uint4 qa = *reinterpret_cast<const uint4 *>(stg.base + (size_t)ra * RB + 16 * t4);
              const uint4 qb = *reinterpret_cast<const uint4 *>(stg.base + (size_t)rb * RB + 16 * t4);
              const __half2 sa = __half2(__nv_cvt_fp8x2_to_halfraw2(
                  *reinterpret_cast<const uint16_t *>(stg.base + TB + ra * (N / 16) + 2 * t4), __NV_E4M3));
              const __half2 sbl = __half2(__nv_cvt_fp8x2_to_halfraw2(
                  *reinterpret_cast<const uint16_t *>(stg.base + TB + rb * (N / 16) + 2 * t4), __NV_E4M3));
              const uint32_t wa[4] = {qa.x, qa.y, qa.z, qa.w}, wb[4] = {qb.x, qb.y, qb.z, qb.w};
#pragma unroll
              for (int ks = 0; ks < 8; ++ks) {
                const __half2 sca = ks < 4 ? __low2half2(sa) : __high2half2(sa);
                const __half2 scb = ks < 4 ? __low2half2(sbl) : __high2half2(sbl);
                const int sh = (ks & 1) * 16;
                af[0] = e2m1x2_scaled(wa[ks >> 1] >> sh, sca);
                af[1] = e2m1x2_scaled(wb[ks >> 1] >> sh, scb);
                af[2] = e2m1x2_scaled(wa[ks >> 1] >> (sh + 8), sca);
                af[3] = e2m1x2_scaled(wb[ks >> 1] >> (sh + 8), scb);
                mma_16816(d, af, bfr[2 * ks], bfr[2 * ks + 1]);
              }
            } else {
              // thread t4 holds bytes [32 t4, 32 t4 + 32) of its rows: k-step ks uses the
              // 4 bytes 4 ks .. 4 ks + 3 (k pairs t4 and t4 + 4); row scale after
              const uint4 qa0 = *reinterpret_cast<const uint4 *>(stg.base + (size_t)ra * RB + 32 * t4);
              const uint4 qa1 = *reinterpret_cast<const uint4 *>(stg.base + (size_t)ra * RB + 32 * t4 + 16);
              const uint4 qb0 = *reinterpret_cast<const uint4 *>(stg.base + (size_t)rb * RB + 32 * t4);
              const uint4 qb1 = *reinterpret_cast<const uint4 *>(stg.base + (size_t)rb * RB + 32 * t4 + 16);
              const uint32_t wa[8] = {qa0.x, qa0.y, qa0.z, qa0.w, qa1.x, qa1.y, qa1.z, qa1.w};
              const uint32_t wb[8] = {qb0.x, qb0.y, qb0.z, qb0.w, qb1.x, qb1.y, qb1.z, qb1.w};
#pragma unroll
              for (int ks = 0; ks < 8; ++ks) {
                af[0] = e4m3x2_h2(wa[ks]);
                af[1] = e4m3x2_h2(wb[ks]);
                af[2] = e4m3x2_h2(wa[ks] >> 16);
                af[3] = e4m3x2_h2(wb[ks] >> 16);
                mma_16816(d, af, bfr[2 * ks], bfr[2 * ks + 1]);
              }
              const float *srow = reinterpret_cast<const float *>(stg.base + TB);
              d[0] *= srow[ra];
              d[2] *= srow[rb];
            }
            // Epilogue: lane (r16 = lane & 15, entry parity lane >> 4) sums the window
            // terms of row r16 over every other entry; the h C value of row r16 sits
            // in d[0] (r16 < 8) or d[2] of lane 4 (r16 & 7).
            const int r16 = lane & 15, row = mt * 16 + r16;
            float ws = 0.0f;
            for (int i = w0 + (lane >> 4); i <= n; i += 2) ws = fmaf(hcoef[i - w0], stg.x<Tin>(i, row), ws);
            ws += __shfl_xor_sync(kFull, ws, 16);
            const float va = __shfl_sync(kFull, d[0], 4 * (r16 & 7));
            const float vb = __shfl_sync(kFull, d[2], 4 * (r16 & 7));
            if (lane < 16) {
              const float hcv = (r16 < 8 ? va : vb) * cinv;
              a.out[((size_t)b * a.H + h) * P + row] =
                  fmaf(__ldg(a.D + h), stg.x<Tin>(n, row), fmaf(hdec[0], hcv, ws));
            }
            done = true;
          }
        }
        if (!done) {
          // ---- CUDA-core path, per group of 8 rows ("virtual warp"; two per warp
          //      when four warps share a head)
#pragma unroll 1
          for (int vw = 0; vw < (kMma ? 2 : 1); ++vw) {
            const int row0 = (kMma ? ((gw & 3) * 2 + vw) : gw) * T::RPW + lane / T::LPR;
            float4 f[T::NLD];   // fp32 checkpoint values for a fold (read-copy layers)
            if constexpr (RF != RSSM_READ_FP32) {
              if (pre || post) {
#pragma unroll
                for (int l = 0; l < T::NLD; ++l) f[l] = ld_stream(hc_src + (size_t)(row0 + l * T::RPI) * N + c0);
              }
            }
            float4 v[T::NLD];
            if (pre) {   // the new tokens do not fit: fold the committed window first
              if constexpr (RF == RSSM_READ_FP32) {
#pragma unroll
                for (int l = 0; l < T::NLD; ++l)
                  f[l] = *reinterpret_cast<const float4 *>(stg.base + ((size_t)(row0 + l * T::RPI) * N + c0) * 4);
              }
              fold_tile<P, N, kGroupWarps, Tin>(f, hfw, hdecf[0], 0, n, stg, sB, row0, c0);
#pragma unroll
              for (int l = 0; l < T::NLD; ++l) {
                const int row = row0 + l * T::RPI;
                if (!post) st_stream(hc_dst + (size_t)row * N + c0, f[l]);
                if constexpr (RF == RSSM_READ_FP32)
                  v[l] = f[l];
                else
                  v[l] = quantize4<RF, T::LPR>(f[l], rc + (size_t)row * RB, a.rc_scales, dbh * P + row, N, c0, lane);
              }
            } else {
#pragma unroll
              for (int l = 0; l < T::NLD; ++l) {
                const int row = row0 + l * T::RPI;
                if constexpr (RF == RSSM_READ_FP32) {
                  v[l] = *reinterpret_cast<const float4 *>(stg.base + ((size_t)row * N + c0) * 4);
                } else if constexpr (RF == RSSM_READ_FP8_E4M3_ROW) {
                  const uint32_t w = *reinterpret_cast<const uint32_t *>(stg.base + (size_t)row * RB + c0);
                  dec_e4m3x4(w, reinterpret_cast<const float *>(stg.base + TB)[row], v[l]);
                } else {
                  const uint32_t w = *reinterpret_cast<const uint16_t *>(stg.base + (size_t)row * RB + c0 / 2);
                  const float sc = dec_e4m3(stg.base[TB + row * (N / 16) + c0 / 16]);
                  dec_e2m1x4(w, sc, v[l]);
                }
              }
            }
            if (m > 0)
              outputs<P, N, kGroupWarps, Tin, MAXM>(v, a, sC, hcoef, hdec, stg, b, h, n, w0, row0, lane, c0);
            if (post) {  // the decode filled the window: fold all of it
              if constexpr (RF == RSSM_READ_FP32) {
#pragma unroll
                for (int l = 0; l < T::NLD; ++l) f[l] = v[l];
              }
              fold_tile<P, N, kGroupWarps, Tin>(f, hfw + 32, hdecf[1], w0, n + 1, stg, sB, row0, c0);
#pragma unroll
              for (int l = 0; l < T::NLD; ++l) {
                const int row = row0 + l * T::RPI;
                st_stream(hc_dst + (size_t)row * N + c0, f[l]);
                if constexpr (RF != RSSM_READ_FP32)
                  quantize4<RF, T::LPR>(f[l], rc + (size_t)row * RB, a.rc_scales, dbh * P + row, N, c0, lane);
              }
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);   // this warp is done with stage s
    }

    // ---- item end: the group's warps are done; the last CTA of sequence b
    //      moves its pointers.  An abort stops the group here.
    const bool any_abort = named_sync_or(bar_id, kGroupThreads, *abort != 0);
    if (any_abort) {
      if (gt == 0) atomicOr(a.status, (unsigned)RSSM_STATUS_TIMEOUT);
      break;   // every consumer thread still meets the others at the TMEM release below
    }
    if (!rp.refuse && gt == 0) {
      __threadfence();
      if (atomicAdd(a.arrivals + b, 1) == a.G * nchunk - 1) {
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

// Conventional update: h <- e^{dt A} h + dt x B^T ; y = h C + D x ; h written back.
// SF (state format): fp32, or a state kept in low precision (FP8 row / NVFP4,
// read-copy layout) that is decoded, updated in fp32 and rounded again every
// token; y comes from the updated fp32 values before that rounding.
template <int P, int N, typename Tin, int SF>
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
  constexpr int RB = rc_row_bytes<SF, N>();
  float4 t[T::NLD];
#pragma unroll
  for (int l = 0; l < T::NLD; ++l) {
    const size_t row = bh * P + row0 + l * T::RPI;
    if constexpr (SF == RSSM_READ_FP32)
      t[l] = ld_stream(a.state_in + row * N + c0);
    else
      t[l] = load_read_copy4<SF>(a.codes_in + row * RB, a.scales_in, row, N, c0);
  }
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
    if constexpr (SF == RSSM_READ_FP32)
      st_stream(a.state_out + bh * P * N + (size_t)row * N + c0, t[l]);
    else
      quantize4<SF, T::LPR>(t[l], a.codes_out + (bh * P + row) * RB, a.scales_out, bh * P + row, N, c0, lane);
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

int heads_per_cta(int hpg) {
  int hc = hpg < 16 ? hpg : 16;
  while (hpg % hc) --hc;
  return hc;
}

template <int P, int N, typename Tin, int RF, int MAXM>
cudaError_t launch_step(const StepArgs &a, cudaStream_t s) {
  auto kern = m2_replay_kernel<P, N, Tin, RF, MAXM>;
  const int hc = heads_per_cta(a.hpg);
  const size_t xrow = (size_t)P * sizeof(Tin);
  const size_t stage = ((size_t)tile_bytes<RF, P, N>() + scale_bytes<RF, P, N>() + (a.L + MAXM) * xrow + 127) & ~(size_t)127;
  const size_t mma_off = (size_t)group_mma_off<P, N, Tin, RF, MAXM>(a.L, hc);
  const size_t umma_off = (mma_off + mma_floats<P, N, Tin, RF, MAXM>() + 31) & ~(size_t)31;
  const size_t group_floats = (umma_off + umma_floats<P, N, Tin, RF>() + 31) & ~(size_t)31;
  const size_t fixed = kGroups * sizeof(float) * group_floats;
  // One CTA per SM (its 544 threads use the register file); as many stages as
  // fit in its shared memory, at most 5 for fp32 tiles (32 KiB each) and
  // kMaxStages for the smaller read-copy tiles.
  int dev = 0, sms = 0, max_smem = 0;
  cudaError_t e;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&max_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev)) != cudaSuccess) return e;
  const size_t budget = (size_t)max_smem - 2048;
  if (fixed + 2 * stage > budget) return cudaErrorInvalidConfiguration;
  int stages = (int)((budget - fixed) / stage);
  if (stages > kMaxStages) stages = kMaxStages;
  if (RF == RSSM_READ_FP32 && stages > 5) stages = 5;
  const size_t smem = fixed + (size_t)stages * stage;
  if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) != cudaSuccess) return e;
  int per_sm = 0;
  if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kReplayThreads, smem)) != cudaSuccess) return e;
  if (per_sm < 1) return cudaErrorInvalidConfiguration;
  const long long items = (long long)a.B * a.G * (a.hpg / hc);
  const long long slots = (long long)sms * per_sm;
  const unsigned grid = (unsigned)(items < slots ? items : slots);
  kern<<<dim3(grid), dim3(kReplayThreads), smem, s>>>(a, hc, stages);
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

template <int P, int N, int SF>
cudaError_t launch_conv_fmt(const ConvArgs &a, int in_dtype, cudaStream_t s) {
  if (in_dtype == RSSM_BF16)
    m2_conv_kernel<P, N, __nv_bfloat16, SF><<<dim3((unsigned)(a.B * a.H)), dim3(kThreads), 0, s>>>(a);
  else
    m2_conv_kernel<P, N, float, SF><<<dim3((unsigned)(a.B * a.H)), dim3(kThreads), 0, s>>>(a);
  return cudaGetLastError();
}

template <int P, int N>
cudaError_t launch_conv(const ConvArgs &a, int in_dtype, int state_fmt, cudaStream_t s) {
  switch (state_fmt) {
    case RSSM_READ_FP32: return launch_conv_fmt<P, N, RSSM_READ_FP32>(a, in_dtype, s);
    case RSSM_READ_FP8_E4M3_ROW: return launch_conv_fmt<P, N, RSSM_READ_FP8_E4M3_ROW>(a, in_dtype, s);
    default: return launch_conv_fmt<P, N, RSSM_READ_NVFP4>(a, in_dtype, s);
  }
}

}  // namespace

bool mamba2_supported(int R, int C) { return R == 64 && (C == 64 || C == 128); }

cudaError_t mamba2_step(const StepArgs &a, int in_dtype, int read_fmt, cudaStream_t s) {
  if (m2_rc_decode_path(a, in_dtype, read_fmt)) return m2_rc_decode_step(a, read_fmt, s);
  if (a.R == 64 && a.C == 64) return dispatch_dtype<64, 64>(a, in_dtype, read_fmt, s);
  return dispatch_dtype<64, 128>(a, in_dtype, read_fmt, s);
}

cudaError_t mamba2_conventional(const ConvArgs &a, int in_dtype, int state_fmt, cudaStream_t s) {
  if (a.R == 64 && a.C == 64) return launch_conv<64, 64>(a, in_dtype, state_fmt, s);
  return launch_conv<64, 128>(a, in_dtype, state_fmt, s);
}

}  // namespace rssm
