// Gated DeltaNet replay decode, the serving path: one token per sequence, the
// fp32 checkpoint read directly, bf16 inputs, d_k = d_v = 128.  Verify, flush,
// read copies and fp32 inputs keep the general kernel of gdn.cu.
//
// Replay form ("ReplaySSM: Rethinking State Storage for Faster Hybrid-Model
// Decoding", deskofai.com summary, paragraphs 2-3: outputs from the checkpoint
// and the buffered inputs, the full state written once per window), gated
// delta rule S_t = a_t S_{t-1} (I - b_t k_t k_t^T) + b_t v_t k_t^T, o = S q,
// with g = ln a and seg(i,e) the g summed over the window entries after i up
// to e:
//   z = e^{G} S_c k_e + sum_{i<e} e^{seg(i,e)} (k_i . k_e) w_i
//   w_e = b_e (v_e - z),   o_e = e^{G} S_c q_e + sum_{i<=e} e^{seg(i,e)} (k_i . q_e) w_i
//   fold (window full): S_c <- e^{G} S_c + sum_{i<=e} e^{seg(i,e)} w_i k_i^T
// The w_i of committed entries are kept in the ring (solved when their token
// was decoded, against the same checkpoint).
//
// Roles of the 768 threads of a persistent CTA (one per SM):
//  * one producer warp: streams each unit -- half a head, 64 state rows (32 KiB
//    fp32) and the committed w rows of those rows -- into a ring of
//    shared-memory stages with 1-D TMA bulk copies, in the consumers' order;
//  * seven prologue warps: for each item (a sequence and a chunk of heads), up
//    to two items ahead of the consumers, they append the new token to the
//    rings and compute every head's window scalars (dots of the window k rows
//    with q and k_e, segment decays as warp suffix sums, fold weights) into one
//    of three item slots, so the consumers never wait on global memory for
//    them; a head is one task, and the tasks go to the warps in turn;
//  * sixteen consumer warps: per unit, warp w owns rows 4w .. 4w+3, a row spread
//    over 8 lanes (4 chunks of 4 columns); both matrix-vector products, the
//    window sums, w_e and o_e; a fold runs on the tensor cores (tcgen05): the
//    rank-l update D^T[c][r] = sum_i k_i[c] (fw_i w_i[r]) as one M = 128 x N = 64
//    MMA chain with an fp32 accumulator in TMEM (k rows exact in bf16, the
//    weighted w split into three bf16 parts), and the epilogue adds e^{G} S.
#include "rssm_device.cuh"
#include "umma.cuh"

namespace rssm {
namespace {

constexpr int DK = 128, DV = 128, HALF = 64;
constexpr int kCons = 16;                       // consumer warps
constexpr int kPro = 7;                         // prologue warps (24 warps in all keep 80 registers)
constexpr int kConsThreads = kCons * 32;
constexpr int kThreads = (kCons + kPro + 1) * 32;
constexpr int kProWarp0 = kCons, kProdWarp = kCons + kPro;
constexpr int kMaxStages = 8;
constexpr int kSlots = 3;
constexpr int kW = 32;                          // window positions a scalar array covers
constexpr uint32_t kTmemCols = DV;              // the fold accumulator: 128 fp32 columns (value rows)

// Per head in an item slot (floats): k_e, q_e, v_e (fp32, exact from bf16),
// Mk[32] and Mq[32] (window entries after the output window start, scaled by
// their decays), fold weights of the window-full fold fwd[32] and of a pre-fold
// fwp[32], then scalars.
struct HeadSlot {
  static constexpr int K = 0, Q = DK, V = 2 * DK, MK = 3 * DK, MQ = MK + kW, FWD = MQ + kW, FWP = FWD + kW;
  static constexpr int BETA = FWP + kW, MQE = BETA + 1, DEC = BETA + 2, DECP = BETA + 3;
  static constexpr int FLOATS = (DECP + 1 + 15) & ~15;
};
// Item slot: the row plan (ints), then hc heads.
struct SlotPlan {
  int b, chunk, st, n, src, dst, refuse, pre, post;
};
constexpr int kPlanFloats = 16;

struct Smem {   // byte offsets in the dynamic shared memory
  int stage_bytes, woff, stages_off, slot_off, slot_bytes, umma_off, total;
};
__host__ __device__ inline Smem smem_layout(int L, int hc, int stages) {
  Smem y;
  y.woff = HALF * DK * 4;
  y.stage_bytes = (y.woff + L * HALF * 4 + 127) & ~127;
  y.stages_off = 0;
  y.slot_off = stages * y.stage_bytes;
  y.slot_bytes = ((kPlanFloats + hc * HeadSlot::FLOATS) * 4 + 127) & ~127;
  y.umma_off = y.slot_off + kSlots * y.slot_bytes;
  const int KG = 2 * ((L + 15) / 16);            // fold operands: every window entry at once
  y.total = y.umma_off + (DK / 8 + 3 * DV / 8) * KG * 128;   // A: k rows; B: three parts, both halves
  return y;
}

__device__ __forceinline__ float4 bf4(uint2 raw) {
  const __nv_bfloat16 *e = reinterpret_cast<const __nv_bfloat16 *>(&raw);
  return make_float4(__bfloat162float(e[0]), __bfloat162float(e[1]), __bfloat162float(e[2]), __bfloat162float(e[3]));
}
__device__ __forceinline__ float dot4(const float4 a, const float4 b) {
  return a.x * b.x + a.y * b.y + a.z * b.z + a.w * b.w;
}

__global__ void __launch_bounds__(kThreads, 1) gdn_decode_kernel(const StepArgs a, const int hc, const int stages) {
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ uint64_t full[kMaxStages], empty[kMaxStages], slot_full[kSlots], slot_empty[kSlots];
  __shared__ uint64_t ops_bar, mma_bar, epi_bar;   // fold: operands written, MMAs done, folded tile written
  __shared__ uint32_t tmem_base;
  __shared__ int abort_flag, never_set;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int L = a.L, cap = a.cap;
  const Smem Y = smem_layout(L, hc, stages);
  const int nchunk = a.H / hc;
  const int nitems = a.B * nchunk;
  const int my_items = (int)blockIdx.x < nitems ? (nitems - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
  const int units = 2 * hc;
  volatile int *abort = &abort_flag;
  const __nv_bfloat16 *qin = reinterpret_cast<const __nv_bfloat16 *>(a.in[0]);
  const __nv_bfloat16 *kin = reinterpret_cast<const __nv_bfloat16 *>(a.in[1]);
  const __nv_bfloat16 *vin = reinterpret_cast<const __nv_bfloat16 *>(a.in[2]);
  const float *alin = reinterpret_cast<const float *>(a.in[3]);
  const float *bein = reinterpret_cast<const float *>(a.in[4]);
  __nv_bfloat16 *kring = reinterpret_cast<__nv_bfloat16 *>(a.buf0);
  __nv_bfloat16 *vring = reinterpret_cast<__nv_bfloat16 *>(a.buf1);
  float *gring = a.buf2, *bring = a.buf3, *wring = a.buf4;

  if (tid == 0) {
    for (int s = 0; s < stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kCons);
    }
    for (int s = 0; s < kSlots; ++s) {
      mbar_init(&slot_full[s], hc);   // one arrival per head of the item
      mbar_init(&slot_empty[s], kCons);
    }
    mbar_init(&ops_bar, kCons);
    mbar_init(&mma_bar, 1);
    mbar_init(&epi_bar, kCons);
    abort_flag = 0;
    never_set = 0;
    mbar_fence_init();
  }
  if (warp == 0) {   // one 128-column fp32 accumulator for the folds; freed by warp 0 at the end
    umma::alloc(&tmem_base, kTmemCols);
    umma::relinquish();
  }
  umma::fence_before_sync();
  __syncthreads();
  umma::fence_after_sync();

  auto item_of = [&](int k, int &b, int &chunk) {
    const int item = (int)blockIdx.x + k * (int)gridDim.x;
    b = item / nchunk;
    chunk = item - b * nchunk;
  };

  if (warp == kProdWarp) {
    // ------------------------------------------------------------ producer
    if (lane != 0) return;
    int issued = 0;
    RowPlan rp{};
    RowRaw nxt{};   // pointers of the next item, requested one item ahead
    int b = 0, chunk = 0;
    const uint64_t stream_once = l2_evict_first_policy();
    if (my_items > 0) {
      item_of(0, b, chunk);
      nxt = load_row(a, b);
    }
    for (int seq = 0; seq < my_items * units; ++seq) {
      const int k = seq / units, unit = seq - k * units, s = seq % stages, u = seq / stages;
      if (u > 0 && !mbar_wait_bounded(&empty[s], (uint32_t)((u - 1) & 1), abort, a.wait_limit)) {
        atomicOr(a.status, (unsigned)RSSM_STATUS_TIMEOUT);
        break;
      }
      if (unit == 0) {
        item_of(k, b, chunk);
        rp = plan_from(a, nxt);
        if (k + 1 < my_items) {
          int bn, cn;
          item_of(k + 1, bn, cn);
          nxt = load_row(a, bn);
        }
      }
      issued = seq + 1;
      if (rp.refuse) {
        mbar_arrive(&full[s]);
        continue;
      }
      const int jh = unit >> 1, hf = unit & 1, h = chunk * hc + jh;
      const size_t bh = (size_t)b * a.H + h, sbh = (size_t)rp.src * a.H + h;
      uint8_t *dst = smem + Y.stages_off + s * Y.stage_bytes;
      mbar_arrive_expect_tx(&full[s], (uint32_t)(HALF * DK * 4 + rp.n * HALF * 4));
      bulk_g2s_hint(dst, a.hc + (sbh * DV + hf * HALF) * DK, HALF * DK * 4, &full[s], stream_once);
      if (rp.n > 0) {   // committed w rows of this half, oldest first (the ring may wrap)
        const float *src = wring + (bh * 2 + hf) * cap * HALF;
        const int c1 = rp.n < cap - rp.st ? rp.n : cap - rp.st;
        bulk_g2s(dst + Y.woff, src + (size_t)rp.st * HALF, c1 * HALF * 4, &full[s]);
        if (rp.n > c1) bulk_g2s(dst + Y.woff + c1 * HALF * 4, src, (rp.n - c1) * HALF * 4, &full[s]);
      }
    }
    if (*abort) {   // let the requested copies land (bounded) before the CTA can retire
      for (int q = issued - stages > 0 ? issued - stages : 0; q < issued; ++q)
        mbar_wait_bounded(&full[q % stages], (uint32_t)((q / stages) & 1), nullptr, 200000000LL);
    }
    return;
  }

  if (warp >= kProWarp0) {
    // ------------------------------------------------------------ prologue
    const int pw = warp - kProWarp0;
    const int c0 = lane * 4;   // this lane's 4 columns of a row
    // When the consumers hand back the slot of item k (they are done with it), the
    // last CTA of its sequence to be done moves the sequence's pointers: prologue
    // warp 0 counts this CTA in.  The pointers were read (by this warp and the
    // producer) before the item was handed to the consumers, so they are stable.
    auto arrive_item = [&](const SlotPlan &p) {
      if (p.refuse) return;
      __threadfence();
      if (atomicAdd(a.arrivals + p.b, 1) == nchunk - 1) {
        a.arrivals[p.b] = 0;
        int st2 = p.st, n2 = p.n, fl = a.flushes[p.b];
        if (p.pre) {
          st2 = (p.st + p.n) % cap;
          n2 = 0;
          ++fl;
        }
        n2 += 1;
        if (p.post) {
          st2 = (st2 + n2) % cap;
          n2 = 0;
          ++fl;
        }
        a.start[p.b] = st2;
        a.len[p.b] = n2;
        a.flushes[p.b] = fl;
      }
    };
    // The item's heads are tasks t = k hc + jh, dealt to the prologue warps in
    // turn (warp pw: tasks pw, pw + kPro, ...); a slot is full once every head
    // of its item has arrived.  The task of head 0 also writes the item's plan
    // and reports the slot's previous item done.
    bool pro_failed = false;
    const int ntasks = my_items * hc;
    RowRaw nxt{};   // pointers of this warp's next task's sequence, requested one task ahead
    if (pw < ntasks) {
      int b0, c0_;
      item_of(pw / hc, b0, c0_);
      nxt = load_row(a, b0);
    }
    for (int t = pw; t < ntasks; t += kPro) {
      const int k = t / hc, jh = t - k * hc;
      const int sl = k % kSlots, use = k / kSlots;
      if (use > 0 && !warp_all(mbar_wait_bounded(&slot_empty[sl], (uint32_t)((use - 1) & 1), abort, a.wait_limit))) {
        atomicOr(a.status, (unsigned)RSSM_STATUS_TIMEOUT);
        pro_failed = true;
        break;
      }
      float *slot = reinterpret_cast<float *>(smem + Y.slot_off + sl * Y.slot_bytes);
      SlotPlan *plan = reinterpret_cast<SlotPlan *>(slot);
      if (use > 0 && jh == 0 && lane == 0) arrive_item(*plan);   // the slot's previous item is done
      int b, chunk;
      item_of(k, b, chunk);
      const RowPlan rp = plan_from(a, nxt);
      if (t + kPro < ntasks) {
        int bn, cn;
        item_of((t + kPro) / hc, bn, cn);
        nxt = load_row(a, bn);
      }
      __syncwarp();
      if (jh == 0 && lane == 0) {
        plan->b = b; plan->chunk = chunk; plan->st = rp.st; plan->n = rp.n; plan->src = rp.src;
        plan->dst = rp.dst; plan->refuse = rp.refuse; plan->pre = rp.pre; plan->post = rp.post;
        if (rp.refuse && rp.bit && chunk == 0) atomicOr(a.status, rp.bit);
      }
      if (!rp.refuse) {
        const int n = rp.n, st = rp.st, w0 = rp.pre ? n : 0;
        const int slot_n = (st + n) % cap;   // ring slot of the new entry
        {
          const int h = chunk * hc + jh;
          const size_t bh = (size_t)b * a.H + h, tok = bh;   // one token per sequence
          float *hsl = slot + kPlanFloats + jh * HeadSlot::FLOATS;
          // the new token's rows (this lane's 4 columns) and scalars, the gates of the
          // committed entries (lane i: entry i) and the first 8 committed k rows of
          // the output window: all requested before any is used (one round trip)
          const uint2 qr = __ldg(reinterpret_cast<const uint2 *>(qin + tok * DK + c0));
          const uint2 kr = __ldg(reinterpret_cast<const uint2 *>(kin + tok * DK + c0));
          const uint2 vr = __ldg(reinterpret_cast<const uint2 *>(vin + tok * DV + c0));
          const float alpha = __ldg(alin + tok), beta = __ldg(bein + tok);
          const float gi = lane < n ? gring[bh * cap + (st + lane) % cap] : 0.0f;
          auto krow = [&](int i) -> uint2 {
            return __ldg(reinterpret_cast<const uint2 *>(kring + (bh * cap + (st + i) % cap) * DK + c0));
          };
          uint2 kw[8];
#pragma unroll
          for (int c = 0; c < 8; ++c) kw[c] = w0 + c < n ? krow(w0 + c) : make_uint2(0u, 0u);
          const float4 q4 = bf4(qr), k4 = bf4(kr), v4 = bf4(vr);
          // raw dots k_i . q and k_i . k_e over the committed entries of the output
          // window [w0, n), 8 entries per transposed reduction
          auto dots8 = [&](int i0, const uint2 *kw8) {
            float part[16];
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              const float4 ki = bf4(kw8[c]);
              part[2 * c] = dot4(ki, q4);
              part[2 * c + 1] = dot4(ki, k4);
            }
            tr_sum<16, 16>(part, lane);
            if ((lane & 1) == 0) {
              const int idx = tr_base<16, 16>(lane), c = idx >> 1, i = i0 + c;
              if (i < n) hsl[((idx & 1) ? HeadSlot::MK : HeadSlot::MQ) + (i - w0)] = part[0];
            }
          };
          if (w0 < n) dots8(w0, kw);
          for (int i0 = w0 + 8; i0 < n; i0 += 8) {   // windows longer than 8
            uint2 kx[8];
#pragma unroll
            for (int c = 0; c < 8; ++c) kx[c] = i0 + c < n ? krow(i0 + c) : make_uint2(0u, 0u);
            dots8(i0, kx);
          }
          // ring appends (after every read of the ring): k row, v row (half-major),
          // ln alpha, beta
          *reinterpret_cast<uint2 *>(kring + (bh * cap + slot_n) * DK + c0) = kr;
          {
            const int hf = c0 / HALF;
            *reinterpret_cast<uint2 *>(vring + ((bh * 2 + hf) * cap + slot_n) * HALF + (c0 - hf * HALF)) = vr;
          }
          const float ge = logf(alpha);
          if (lane == 0) {
            gring[bh * cap + slot_n] = ge;
            bring[bh * cap + slot_n] = beta;
          }
          *reinterpret_cast<float4 *>(hsl + HeadSlot::K + c0) = k4;
          *reinterpret_cast<float4 *>(hsl + HeadSlot::Q + c0) = q4;
          *reinterpret_cast<float4 *>(hsl + HeadSlot::V + c0) = v4;
          const float mqe = warp_sum(dot4(k4, q4));
          __syncwarp();
          // decays over the output window [w0, n]: lane l holds entry w0 + l
          {
            const int len = n - w0 + 1;
            const float gl = __shfl_sync(kFull, gi, (w0 + lane) & 31);   // entry w0 + lane's gate, all lanes
            const float v = lane < len ? (w0 + lane < n ? gl : ge) : 0.0f;
            float after, total;
            suffix_scan(v, lane, after, total);
            const float ex = expf(after);
            if (lane < len - 1) {
              hsl[HeadSlot::MQ + lane] *= ex;
              hsl[HeadSlot::MK + lane] *= ex;
            }
            if (lane < len) hsl[HeadSlot::FWD + lane] = ex;   // window-full fold weights (same window)
            if (lane == 0) {
              hsl[HeadSlot::DEC] = expf(total);
              hsl[HeadSlot::MQE] = mqe;
              hsl[HeadSlot::BETA] = beta;
            }
          }
          if (rp.pre) {   // a pre-fold of the committed entries [0, n)
            const float v = lane < n ? gi : 0.0f;
            float after, total;
            suffix_scan(v, lane, after, total);
            if (lane < n) hsl[HeadSlot::FWP + lane] = expf(after);
            if (lane == 0) hsl[HeadSlot::DECP] = expf(total);
          }
        }
      }
      __threadfence();   // ring appends visible before the item's pointers can move
      __syncwarp();
      if (lane == 0) mbar_arrive(&slot_full[sl]);
    }
    if (pw == 0 && !pro_failed) {   // the last items: wait until the consumers are done with them
      for (int k = my_items - kSlots > 0 ? my_items - kSlots : 0; k < my_items; ++k) {
        const int sl = k % kSlots, use = k / kSlots;
        if (!warp_all(mbar_wait_bounded(&slot_empty[sl], (uint32_t)(use & 1), abort, a.wait_limit))) break;
        if (lane == 0) arrive_item(*reinterpret_cast<const SlotPlan *>(smem + Y.slot_off + sl * Y.slot_bytes));
      }
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  // Per head the consumers take both of its units (the two halves of the state,
  // two consecutive stages) together: warp w owns rows 4w .. 4w+3 of each half,
  // a row spread over 8 lanes, so every lane works on two independent rows.
  // The consumer warps synchronise only through mbarriers with bounded waits
  // (stage full / empty, item slot full / empty, fold operands ready, fold
  // done, folded tile written), never through a named barrier until the TMEM
  // release at the end: a warp that gives up (an abort) stops arriving, the
  // others' waits then run out as well, and every warp still reaches the end.
  const int cw = warp, g4 = lane >> 3, j8 = lane & 7;
  const int row = 4 * cw + g4;     // this lane's row inside each half
  uint8_t *uA = smem + Y.umma_off;
  const int KG = 2 * ((L + 15) / 16);
  uint8_t *uB = uA + (DK / 8) * KG * 128;
  const int partB = (DV / 8) * KG * 128;
  const uint32_t tm = tmem_base;
  int folds = 0, epis = 0;   // completed folds (ops_bar, mma_bar phases) and folded-tile writes (epi_bar)
  bool failed = false;
  if (a.stall_test && blockIdx.x == 0) {   // the timeout self-test: this CTA's waits run out
    stall_on_unset_flag(&never_set, abort, a.wait_limit);
    if (tid == 0) atomicOr(a.status, (unsigned)RSSM_STATUS_TIMEOUT);
  }
  for (int k = 0; k < my_items && !failed; ++k) {
    const int sl = k % kSlots;
    if (!warp_all(mbar_wait_bounded(&slot_full[sl], (uint32_t)((k / kSlots) & 1), abort, a.wait_limit))) {
      failed = true;
      break;
    }
    const float *slot = reinterpret_cast<const float *>(smem + Y.slot_off + sl * Y.slot_bytes);
    const SlotPlan plan = *reinterpret_cast<const SlotPlan *>(slot);
    const int b = plan.b, n = plan.n, st = plan.st, w0 = plan.pre ? n : 0;
    const int slot_n = (st + n) % cap;
    for (int jh = 0; jh < hc; ++jh) {
      const int seq0 = k * units + 2 * jh, s0 = seq0 % stages, s1 = (seq0 + 1) % stages;
      if (!warp_all(mbar_wait_bounded(&full[s0], (uint32_t)((seq0 / stages) & 1), abort, a.wait_limit) &&
                    mbar_wait_bounded(&full[s1], (uint32_t)(((seq0 + 1) / stages) & 1), abort, a.wait_limit))) {
        failed = true;
        break;
      }
      auto release = [&]() {
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&empty[s0]);
          mbar_arrive(&empty[s1]);
        }
      };
      if (plan.refuse) {
        release();
        continue;
      }
      const int h = plan.chunk * hc + jh;
      const size_t bh = (size_t)b * a.H + h;
      const float *hsl = slot + kPlanFloats + jh * HeadSlot::FLOATS;
      float *tile[2] = {reinterpret_cast<float *>(smem + Y.stages_off + s0 * Y.stage_bytes),
                        reinterpret_cast<float *>(smem + Y.stages_off + s1 * Y.stage_bytes)};
      const float *wst[2] = {tile[0] + Y.woff / 4, tile[1] + Y.woff / 4};
      float *hc_rows = a.hc + ((size_t)plan.dst * a.H + h) * DV * DK;   // the head's 128 rows

      // The A operand of a fold over the window [i0, i0 + nf): the window's k rows
      // (bf16, exact; committed rows straight from the ring, the new token's from
      // the slot), zero beyond.  Copies in flight until the fold waits for them.
      auto build_a = [&](int i0, int nf) {
        const int KE = KG * 8;
        for (int idx = tid; idx < KE * (DK / 8); idx += kConsThreads) {
          const int i = idx / (DK / 8), cc = idx - i * (DK / 8);
          uint8_t *dst = uA + umma::mn_offset(8 * cc, i, KG);
          if (i < nf && i0 + i < n) {
            cp_async16(dst, kring + (bh * cap + (st + i0 + i) % cap) * DK + 8 * cc);
          } else {
            uint4 val = make_uint4(0u, 0u, 0u, 0u);
            if (i < nf) {   // the new token's k (fp32 copy of bf16 values): back to bf16
              const float4 lo = *reinterpret_cast<const float4 *>(hsl + HeadSlot::K + 8 * cc);
              const float4 hi = *reinterpret_cast<const float4 *>(hsl + HeadSlot::K + 8 * cc + 4);
              const __nv_bfloat162 p0 = __floats2bfloat162_rn(lo.x, lo.y), p1 = __floats2bfloat162_rn(lo.z, lo.w);
              const __nv_bfloat162 p2 = __floats2bfloat162_rn(hi.x, hi.y), p3 = __floats2bfloat162_rn(hi.z, hi.w);
              val = make_uint4(*reinterpret_cast<const uint32_t *>(&p0), *reinterpret_cast<const uint32_t *>(&p1),
                               *reinterpret_cast<const uint32_t *>(&p2), *reinterpret_cast<const uint32_t *>(&p3));
            }
            *reinterpret_cast<uint4 *>(dst) = val;
          }
        }
      };
      // Tensor-core fold of the head (both halves, 128 rows) over the window
      // [i0, i0 + nf) with weights fw; the new entry n's w of this lane's two
      // rows is wn[hf].  D^T[c][r] = sum_i k_i[c] (fw_i w_i[r]) is one M = 128 x
      // N = 128 MMA chain.  with_a: build the A operand here (else it was built,
      // and may still be in flight, earlier).  Each warp writes the B operand of
      // its rows and counts in on ops_bar; thread 0 issues the MMAs once all
      // have, and commits them to mma_bar.  The result goes to the stage tiles (a
      // pre-fold the outputs read; the warps then meet on epi_bar) and/or to the
      // checkpoint.  Returns false if a wait gave up.
      auto fold_tc = [&](int i0, int nf, const float *fw, float dF, const float (&wn)[2], bool with_a,
                         bool to_stage, bool to_global) -> bool {
        const int KE = KG * 8;
        if (with_a) build_a(i0, nf);
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          for (int i = j8; i < KE; i += 8) {   // B: three parts of fw_i w_i[r], this lane's rows
            float x = 0.0f;
            if (i < nf) x = fw[i] * (i0 + i < n ? wst[hf][(i0 + i) * HALF + row] : wn[hf]);
            uint16_t xh, xm, xl;
            umma::split3_bf16(x, xh, xm, xl);
            const uint32_t off = umma::mn_offset(hf * HALF + row, i, KG);
            *reinterpret_cast<uint16_t *>(uB + off) = xh;
            *reinterpret_cast<uint16_t *>(uB + partB + off) = xm;
            *reinterpret_cast<uint16_t *>(uB + 2 * partB + off) = xl;
          }
        }
        cp_async_wait_all();
        fence_proxy_async();   // this thread's operand writes -> visible to the tensor core
        umma::fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(&ops_bar);
        if (tid == 0) {
          if (mbar_wait_bounded(&ops_bar, (uint32_t)(folds & 1), abort, a.wait_limit)) {
            umma::fence_after_sync();
            constexpr uint32_t idesc = umma::idesc_bf16_f32_mn(DK, DV);
            for (int part = 0; part < 3; ++part)
              for (int ks = 0; ks < KG / 2; ++ks)
                umma::mma_bf16(tm, umma::smem_desc_mn(smem_u32(uA) + 256 * ks, 128, KG * 128),
                               umma::smem_desc_mn(smem_u32(uB + part * partB) + 256 * ks, 128, KG * 128), idesc,
                               part > 0 || ks > 0);
          } else {
            *abort = 1;   // no MMA issued: the commit below completes at once, the others see the abort
          }
          umma::commit(&mma_bar);
        }
        // the MMAs always complete: wait without the abort flag (bounded), so that
        // TMEM and the operands are never reused or released under a running MMA
        const bool done = warp_all(mbar_wait_bounded(&mma_bar, (uint32_t)(folds & 1), nullptr, kDefaultWaitLimit));
        ++folds;
        umma::fence_after_sync();
        if (!done || *abort) return false;
        // epilogue: lane = key column c; warp quarter of the head's rows cw >> 2
        const int q = cw & 3, c = 32 * q + lane, rh = (cw >> 2) * 32;
        float d[32];
        umma::ld_32x32b_x32(tm + ((uint32_t)(32 * q) << 16) + (uint32_t)rh, d);   // rows rh .. rh + 31
        umma::fence_before_sync();
        float *t = tile[rh / HALF];
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const int r = rh + j, rr = r % HALF;
          const float val = fmaf(dF, t[rr * DK + c], d[j]);
          if (to_stage) t[rr * DK + c] = val;
          if (to_global) __stcs(hc_rows + (size_t)r * DK + c, val);
        }
        if (to_stage) {   // the folded tiles are read row-wise by other warps: all must have written
          __syncwarp();
          if (lane == 0) mbar_arrive(&epi_bar);
          const bool ok = warp_all(mbar_wait_bounded(&epi_bar, (uint32_t)(epis & 1), abort, a.wait_limit));
          ++epis;
          if (!ok) return false;
        }
        return true;
      };

      // a window-full fold without a pre-fold: its A operand is requested now, to
      // land while the outputs are made
      const bool a_early = plan.post && !plan.pre;
      if (a_early) build_a(w0, n - w0 + 1);
      if (plan.pre) {   // the window was full: fold it into the stages first
        const float none[2] = {0.0f, 0.0f};
        if (!fold_tc(0, n, hsl + HeadSlot::FWP, hsl[HeadSlot::DECP], none, true, true, !plan.post)) {
          failed = true;
          break;
        }
      }
      // ---- outputs of both rows.  This lane: columns 32 c + 4 j8 .. + 3 (c = 0..3);
      //      a head without a fold reads the stages once into registers (tile
      //      chunks and the w of its window entries i = w0 + j8 + 8 t) and hands
      //      them back before computing, so the next copies start sooner
      float4 f[2][4];
      float wv[2][kW / 8];
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
#pragma unroll
        for (int c = 0; c < 4; ++c) f[hf][c] = *reinterpret_cast<const float4 *>(tile[hf] + row * DK + 32 * c + 4 * j8);
#pragma unroll
        for (int t = 0; t < kW / 8; ++t) {
          const int i = w0 + j8 + 8 * t;
          wv[hf][t] = i < n ? wst[hf][i * HALF + row] : 0.0f;
        }
      }
      const bool held = plan.post;   // a fold still reads the stages
      if (!held) release();
      const float dec = hsl[HeadSlot::DEC];
      float pz[2] = {0.0f, 0.0f}, pa[2] = {0.0f, 0.0f};
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int col = 32 * c + 4 * j8;
        const float4 k4 = *reinterpret_cast<const float4 *>(hsl + HeadSlot::K + col);
        const float4 q4 = *reinterpret_cast<const float4 *>(hsl + HeadSlot::Q + col);
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          pz[hf] += dot4(f[hf][c], k4);
          pa[hf] += dot4(f[hf][c], q4);
        }
      }
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        pz[hf] *= dec;
        pa[hf] *= dec;
      }
#pragma unroll
      for (int t = 0; t < kW / 8; ++t) {   // committed window entries, 8 lanes of the row
        const int i = w0 + j8 + 8 * t;
        if (i < n) {
          const float mk = hsl[HeadSlot::MK + (i - w0)], mq = hsl[HeadSlot::MQ + (i - w0)];
#pragma unroll
          for (int hf = 0; hf < 2; ++hf) {
            pz[hf] = fmaf(mk, wv[hf][t], pz[hf]);
            pa[hf] = fmaf(mq, wv[hf][t], pa[hf]);
          }
        }
      }
#pragma unroll
      for (int o = 4; o >= 1; o >>= 1) {
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          pz[hf] += __shfl_xor_sync(kFull, pz[hf], o);
          pa[hf] += __shfl_xor_sync(kFull, pa[hf], o);
        }
      }
      float wn[2];
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        const int vrow = hf * HALF + row;
        wn[hf] = hsl[HeadSlot::BETA] * (hsl[HeadSlot::V + vrow] - pz[hf]);
        if (j8 == 0) {
          a.out[bh * DV + vrow] = a.out_scale * fmaf(hsl[HeadSlot::MQE], wn[hf], pa[hf]);
          wring[((bh * 2 + hf) * cap + slot_n) * HALF + row] = wn[hf];
        }
      }
      if (plan.post) {   // the decode filled the window: fold all of it
        if (!fold_tc(w0, n - w0 + 1, hsl + HeadSlot::FWD, dec, wn, !a_early, false, true)) {
          failed = true;
          break;
        }
      }
      if (held) release();
    }
    if (failed) break;
    // ---- item end: this warp is done with the item; when all are, the slot goes
    //      back to the prologue warps, which count the item in for its sequence
    __syncwarp();
    if (lane == 0) mbar_arrive(&slot_empty[sl]);
  }
  if (failed) {
    *abort = 1;
    if (lane == 0) atomicOr(a.status, (unsigned)RSSM_STATUS_TIMEOUT);
  }
  // every consumer thread meets here (also after an abort) before TMEM is released
  umma::fence_before_sync();
  named_sync(3, kConsThreads);
  if (warp == 0) {
    umma::fence_after_sync();
    umma::dealloc(tm, kTmemCols);
  }
}

}  // namespace

bool gdn_decode_fast_path(const StepArgs &a, int in_dtype, int read_fmt) {
  return a.mode == kDecode && a.m == 1 && in_dtype == RSSM_BF16 && read_fmt == RSSM_READ_FP32 && a.R == DV &&
         a.C == DK && a.L <= kW;
}

cudaError_t gdn_decode_step(const StepArgs &a, cudaStream_t s) {
  int dev = 0, sms = 0, max_smem = 0;
  cudaError_t e;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&max_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev)) != cudaSuccess) return e;
  const int budget = max_smem - 2048;   // the static shared variables
  int hc = 4;
  while (a.H % hc) --hc;
  int stages = kMaxStages;
  while (stages > 2 && smem_layout(a.L, hc, stages).total > budget) --stages;
  const Smem y = smem_layout(a.L, hc, stages);
  if (y.total > budget) return cudaErrorInvalidConfiguration;
  if ((e = cudaFuncSetAttribute(gdn_decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, y.total)) != cudaSuccess)
    return e;
  const long long items = (long long)a.B * (a.H / hc);
  const unsigned grid = (unsigned)(items < sms ? items : sms);
  gdn_decode_kernel<<<dim3(grid), dim3(kThreads), y.total, s>>>(a, hc, stages);
  return cudaGetLastError();
}

}  // namespace rssm
