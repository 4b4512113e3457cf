// Kimi Delta Attention replay decode, the serving path: one token per
// sequence, the fp32 checkpoint read directly, bf16 inputs, d_k = d_v = 128.
// Flush, fp32 inputs and the other launches keep the kernel of kda.cu.
//
// KDA is read as the gated delta rule with one gate per key channel
// ("ReplaySSM: Rethinking State Storage for Faster Hybrid-Model Decoding",
// babnews.org teaser, names the layer).  With g = ln alpha per channel,
// seg(s,e)[c] the g of the window entries after s up to e summed per channel
// and G[c] the g of the whole window summed (the ring keeps alpha, and every
// e^{seg} is formed as the running product of the alphas):
//   z = S_c (e^{G} . k_e) + sum_{s<e} ((k_s . e^{seg(s,e)}) . k_e) w_s
//   w_e = b_e (v_e - z),
//   o_e = out_scale (S_c (e^{G} . q_e) + sum_{s<=e} ((k_s . e^{seg(s,e)}) . q_e) w_s)
//   fold (window full): S_c <- S_c Diag(e^{G}) + sum_{s<=e} w_s (k_s . e^{seg(s,e)})^T
// (. between vectors: elementwise).  The w_s of committed entries are kept in
// the ring, solved when their token was decoded.
//
// Roles of the 672 threads of a persistent CTA (one per SM), as in the Gated
// DeltaNet serving kernel (dr_decode.cu):
//  * one producer lane streams half-head units -- 64 state rows (32 KiB fp32)
//    and the committed w rows of those rows -- into shared-memory stages with
//    1-D TMA bulk copies;
//  * four prologue warps, one item (a sequence and a chunk of heads) ahead of
//    the consumers, append the token to the rings and compute per head the
//    vectors e^{G}.k_e and e^{G}.q_e and the window dots above: lane l owns key
//    channels 4l .. 4l+3, walks the window from the newest entry down keeping
//    the per-channel products, and reduces 8 entries' dots at a time.  For an
//    item whose window fills, they also write the fold's A operand
//    (k_s . e^{seg(s,e)}, in its MMA layout) and e^{G} to a per-CTA scratch
//    region of the ring buffer, from which the consumers copy it;
//  * sixteen consumer warps make both matrix-vector products, w_e and o_e (warp
//    w owns rows 4w .. 4w+3 of each half, a row over 8 lanes).  A fold is one
//    tcgen05 MMA chain D^T[c][r] = sum_s (k_s . e^{seg(s,e)})[c] w_s[r],
//    M = 128 x N = 128, accumulator in TMEM.  Both operands are fp32 values,
//    each split exactly into three bf16 parts (hi, mid, lo, every part at most
//    2^-8 of the one before); the MMA accumulates the six part products
//    hi.hi, hi.mid, mid.hi, hi.lo, lo.hi, mid.mid and leaves out mid.lo, lo.mid
//    and lo.lo, each at most 2^-24 of |a b|.  The epilogue adds e^{G}[c] S[r][c].
#include "rssm_device.cuh"
#include "rssm_kda.h"
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
constexpr int kScratchCtas = 256;               // CTAs the fold scratch is sized for

// Bytes of one head's fold operands in the scratch: A in three parts, then e^{G}.
__host__ __device__ constexpr int fold_part_bytes(int KG) { return (DK / 8) * KG * 128; }
__host__ __device__ constexpr int fold_head_bytes(int KG) { return 3 * fold_part_bytes(KG) + DK * 4; }

// Per head in an item slot (floats): e^{G}.k_e and e^{G}.q_e (fp32 [DK]), v_e
// (bf16 [DV]), the window dots Mk[32] and Mq[32] (entries after the output
// window start), beta_e and k_e . q_e.
struct HeadSlot {
  static constexpr int GK = 0, GQ = DK, VB = 2 * DK, MK = VB + DV / 2, MQ = MK + kW;
  static constexpr int BETA = MQ + kW, MQE = BETA + 1;
  static constexpr int FLOATS = (MQE + 1 + 15) & ~15;
};
struct SlotPlan {
  int b, chunk, st, n, src, dst, refuse, pre, post;
};
constexpr int kPlanFloats = 16;

struct Smem {   // byte offsets in the dynamic shared memory
  int stage_bytes, woff, slot_off, slot_bytes, eg_off, umma_off, total;
};
__host__ __device__ inline Smem smem_layout(int L, int hc, int stages) {
  Smem y;
  y.woff = HALF * DK * 4;
  y.stage_bytes = (y.woff + L * HALF * 4 + 127) & ~127;
  y.slot_off = stages * y.stage_bytes;
  y.slot_bytes = ((kPlanFloats + hc * HeadSlot::FLOATS) * 4 + 127) & ~127;
  y.eg_off = y.slot_off + kSlots * y.slot_bytes;   // e^{G} of a fold's window, per key channel
  y.umma_off = y.eg_off + DK * 4;
  const int KG = 2 * ((L + 15) / 16);
  y.total = y.umma_off + 3 * (DK / 8 + DV / 8) * KG * 128;   // A and B, three parts each
  return y;
}

__device__ __forceinline__ float4 bf4(uint2 raw) {
  const __nv_bfloat16 *e = reinterpret_cast<const __nv_bfloat16 *>(&raw);
  return make_float4(__bfloat162float(e[0]), __bfloat162float(e[1]), __bfloat162float(e[2]), __bfloat162float(e[3]));
}
__device__ __forceinline__ float dot4(const float4 a, const float4 b) {
  return a.x * b.x + a.y * b.y + a.z * b.z + a.w * b.w;
}
__device__ __forceinline__ float4 mul4(const float4 a, const float4 b) {
  return make_float4(a.x * b.x, a.y * b.y, a.z * b.z, a.w * b.w);
}

__device__ __forceinline__ uint32_t pack_bf16x2(uint16_t lo, uint16_t hi) { return (uint32_t)lo | ((uint32_t)hi << 16); }

// KG: K-groups of 8 window entries in the fold operands (2 for L <= 16, 4 for L <= 32).
template <int KG>
__global__ void __launch_bounds__(kThreads, 1) kda_decode_kernel(const StepArgs a, const int hc, const int stages) {
  constexpr int KE = KG * 8;   // window entries a fold contracts over (zero-padded)
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
  __nv_bfloat16 *kring = reinterpret_cast<__nv_bfloat16 *>(a.buf0);   // [B,H,cap,dk]
  __nv_bfloat16 *vring = reinterpret_cast<__nv_bfloat16 *>(a.buf1);   // [B,H,cap,dv]
  float *aring = a.buf2;                                               // [B,H,cap,dk] alpha
  float *bring = a.buf3;                                               // [B,H,cap]
  float *wring = a.buf4;                                               // [B,H,2,cap,dv/2]

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
      uint8_t *dst = smem + s * Y.stage_bytes;
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
    const int c0 = lane * 4;   // this lane's 4 key channels / value rows
    // When the consumers hand back the slot of item k, the last CTA of its
    // sequence to be done moves the sequence's pointers: prologue warp 0 counts
    // this CTA in.
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
      int b0, ch0;
      item_of(pw / hc, b0, ch0);
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
          // the new token's rows (this lane's 4 channels) and the newest 8 committed
          // entries of the output window: requested before any is used
          const uint2 qr = __ldg(reinterpret_cast<const uint2 *>(qin + tok * DK + c0));
          const uint2 kr = __ldg(reinterpret_cast<const uint2 *>(kin + tok * DK + c0));
          const uint2 vr = __ldg(reinterpret_cast<const uint2 *>(vin + tok * DV + c0));
          const float4 al = __ldg(reinterpret_cast<const float4 *>(alin + tok * DK + c0));
          const float beta = __ldg(bein + tok);
          auto ring_at = [&](int i) -> size_t { return bh * cap + (st + i) % cap; };
          uint2 kw[8];
          float4 aw[8];
          auto load8 = [&](int top) {   // entries top, top - 1, ..., top - 7 (those >= w0)
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              const int i = top - c;
              kw[c] = make_uint2(0u, 0u);
              aw[c] = make_float4(1.0f, 1.0f, 1.0f, 1.0f);
              if (i >= w0) {
                kw[c] = __ldg(reinterpret_cast<const uint2 *>(kring + ring_at(i) * DK + c0));
                aw[c] = *reinterpret_cast<const float4 *>(aring + ring_at(i) * DK + c0);
              }
            }
          };
          load8(n - 1);
          // the token's v row to the slot; ring appends (no read of the ring touches
          // slot_n): k row, v row, alpha, beta
          reinterpret_cast<uint2 *>(hsl + HeadSlot::VB)[lane] = vr;
          *reinterpret_cast<uint2 *>(kring + (bh * cap + slot_n) * DK + c0) = kr;
          *reinterpret_cast<uint2 *>(vring + (bh * cap + slot_n) * DV + c0) = vr;
          *reinterpret_cast<float4 *>(aring + (bh * cap + slot_n) * DK + c0) = al;
          if (lane == 0) {
            bring[bh * cap + slot_n] = beta;
            hsl[HeadSlot::BETA] = beta;
          }
          const float4 q4 = bf4(qr), k4 = bf4(kr);
          // walk the output window [w0, n) from the newest entry down: acc holds
          // e^{seg(i, n)} = prod_{i < r <= n} alpha_r for the current entry i; the
          // dots of two entries at a time go through one transposed reduction
          // (lanes 8 j .. 8 j + 7 end with value j: (entry, q or k))
          float4 acc = al;
          for (int top = n - 1; top >= w0; top -= 8) {
            if (top != n - 1) load8(top);   // windows longer than 8
#pragma unroll
            for (int c = 0; c < 8; c += 2) {
              float part[4];
#pragma unroll
              for (int e2 = 0; e2 < 2; ++e2) {
                const float4 kd = mul4(bf4(kw[c + e2]), acc);   // k_i . e^{seg(i, n)}
                part[2 * e2] = dot4(kd, q4);
                part[2 * e2 + 1] = dot4(kd, k4);
                if (top - c - e2 >= w0) acc = mul4(acc, aw[c + e2]);
              }
              tr_sum<4, 16>(part, lane);
              if ((lane & 7) == 0) {
                const int idx = tr_base<4, 16>(lane), i = top - c - (idx >> 1);
                if (i >= w0) hsl[((idx & 1) ? HeadSlot::MK : HeadSlot::MQ) + (i - w0)] = part[0];
              }
            }
          }
          // acc is now e^{G} over [w0, n] per channel
          *reinterpret_cast<float4 *>(hsl + HeadSlot::GK + c0) = mul4(acc, k4);
          *reinterpret_cast<float4 *>(hsl + HeadSlot::GQ + c0) = mul4(acc, q4);
          const float mqe = warp_sum(dot4(k4, q4));
          if (lane == 0) hsl[HeadSlot::MQE] = mqe;
          if (rp.post && !rp.pre) {
            // the window fills: the fold's A operand, column i = k_i . e^{seg(i, n)}
            // of this lane's 4 channels in three bf16 parts (8-byte stores), zero
            // columns beyond the new entry, and e^{G}, to this head's scratch
            uint8_t *sa = a.fold_scratch + (((size_t)blockIdx.x * kSlots + sl) * hc + jh) * fold_head_bytes(KG);
            auto put_a = [&](int i, const float4 x) {
              uint16_t h0, m0, l0, h1, m1, l1, h2, m2, l2, h3, m3, l3;
              umma::split3_bf16(x.x, h0, m0, l0);
              umma::split3_bf16(x.y, h1, m1, l1);
              umma::split3_bf16(x.z, h2, m2, l2);
              umma::split3_bf16(x.w, h3, m3, l3);
              uint8_t *dst = sa + umma::mn_offset(c0, i, KG);
              *reinterpret_cast<uint2 *>(dst) = make_uint2(pack_bf16x2(h0, h1), pack_bf16x2(h2, h3));
              *reinterpret_cast<uint2 *>(dst + fold_part_bytes(KG)) = make_uint2(pack_bf16x2(m0, m1), pack_bf16x2(m2, m3));
              *reinterpret_cast<uint2 *>(dst + 2 * fold_part_bytes(KG)) =
                  make_uint2(pack_bf16x2(l0, l1), pack_bf16x2(l2, l3));
            };
            *reinterpret_cast<float4 *>(sa + 3 * fold_part_bytes(KG) + c0 * 4) = acc;
            put_a(n, k4);
            for (int i = n + 1; i < KE; ++i) put_a(i, make_float4(0.0f, 0.0f, 0.0f, 0.0f));
            float4 dec = al;   // the same walk again (w0 = 0 here), rows re-read from L2
            for (int top = n - 1; top >= 0; top -= 8) {
              load8(top);
#pragma unroll
              for (int c = 0; c < 8; ++c) {
                if (top - c >= 0) {
                  put_a(top - c, mul4(bf4(kw[c]), dec));
                  dec = mul4(dec, aw[c]);
                }
              }
            }
          }
        }
      }
      __threadfence();   // ring appends and fold operands visible to the consumers and the next launch
      __syncwarp();
      if (lane == 0) mbar_arrive(&slot_full[sl]);
    }
    if (pw == 0 && !pro_failed) {   // the last items: wait until the consumers are done with them (bounded)
      for (int k = my_items - kSlots > 0 ? my_items - kSlots : 0; k < my_items; ++k) {
        const int sl = k % kSlots, use = k / kSlots;
        if (!warp_all(mbar_wait_bounded(&slot_empty[sl], (uint32_t)(use & 1), abort, a.wait_limit))) break;
        if (lane == 0) arrive_item(*reinterpret_cast<const SlotPlan *>(smem + Y.slot_off + sl * Y.slot_bytes));
      }
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  // Per head the consumers take both of its units (two consecutive stages):
  // warp w owns rows 4w .. 4w+3 of each half, a row spread over 8 lanes.  They
  // synchronise only through mbarriers with bounded waits until the TMEM
  // release at the end.
  const int cw = warp, g4 = lane >> 3, j8 = lane & 7;
  const int row = 4 * cw + g4;     // this lane's row inside each half
  uint8_t *uA = smem + Y.umma_off;                  // three parts of A [DK x KE]
  constexpr int partA = (DK / 8) * KG * 128;
  uint8_t *uB = uA + 3 * partA;                      // three parts of B [DV x KE]
  constexpr int partB = (DV / 8) * KG * 128;
  float *eg_s = reinterpret_cast<float *>(smem + Y.eg_off);
  const uint32_t tm = tmem_base;
  int folds = 0, epis = 0;
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
      float *tile[2] = {reinterpret_cast<float *>(smem + s0 * Y.stage_bytes),
                        reinterpret_cast<float *>(smem + s1 * Y.stage_bytes)};
      const float *wst[2] = {tile[0] + Y.woff / 4, tile[1] + Y.woff / 4};
      float *hc_rows = a.hc + ((size_t)plan.dst * a.H + h) * DV * DK;   // the head's 128 rows

      // The A operand of a fold over the window [i0, i0 + nf): column i holds
      // k_{i0+i} . e^{seg(i0+i, i0+nf-1)} in three bf16 parts, zero beyond;
      // e^{G} of that window goes to eg_s.  A window-full fold without a
      // pre-fold copies both from the scratch the prologue wrote; otherwise
      // thread c < DK walks channel c from the newest entry down (the rings
      // hold the new token's rows by now).
      auto build_a = [&](int i0, int nf) {
        if (plan.post && !plan.pre) {
          const uint8_t *sa = a.fold_scratch + (((size_t)blockIdx.x * kSlots + sl) * hc + jh) * fold_head_bytes(KG);
          for (int idx = tid; idx < 3 * partA / 16; idx += kConsThreads) cp_async16(uA + 16 * idx, sa + 16 * idx);
          for (int idx = tid; idx < DK * 4 / 16; idx += kConsThreads)
            cp_async16(reinterpret_cast<uint8_t *>(eg_s) + 16 * idx, sa + 3 * partA + 16 * idx);
          return;
        }
        if (tid < DK) {
          const int c = tid;
          float kv[KE], av[KE];
#pragma unroll
          for (int i = 0; i < KE; ++i) {
            kv[i] = 0.0f;
            av[i] = 1.0f;
            if (i < nf) {
              const size_t r = bh * cap + (st + i0 + i) % cap;
              kv[i] = __bfloat162float(__ldcg(kring + r * DK + c));
              av[i] = __ldcg(aring + r * DK + c);
            }
          }
          float acc = 1.0f;
#pragma unroll
          for (int i = KE - 1; i >= 0; --i) {
            float x = 0.0f;
            if (i < nf) {
              x = kv[i] * acc;
              acc *= av[i];
            }
            uint16_t xh, xm, xl;
            umma::split3_bf16(x, xh, xm, xl);
            const uint32_t off = umma::mn_offset(c, i, KG);
            *reinterpret_cast<uint16_t *>(uA + off) = xh;
            *reinterpret_cast<uint16_t *>(uA + partA + off) = xm;
            *reinterpret_cast<uint16_t *>(uA + 2 * partA + off) = xl;
          }
          eg_s[c] = acc;
        }
      };
      // Tensor-core fold of the head (both halves, 128 rows) over the window
      // [i0, i0 + nf); the new entry n's w of this lane's two rows is wn[hf].
      // with_a: build the A operand here (else it was built earlier).  The
      // result goes to the stage tiles (a pre-fold the outputs read; the warps
      // then meet on epi_bar) and/or to the checkpoint.  Returns false if a wait
      // gave up.
      auto fold_tc = [&](int i0, int nf, const float (&wn)[2], bool with_a, bool to_stage, bool to_global) -> bool {
        if (with_a) build_a(i0, nf);
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          for (int i = j8; i < KE; i += 8) {   // B: three parts of w_i[r], this lane's rows
            float x = 0.0f;
            if (i < nf) x = i0 + i < n ? wst[hf][(i0 + i) * HALF + row] : wn[hf];
            uint16_t xh, xm, xl;
            umma::split3_bf16(x, xh, xm, xl);
            const uint32_t off = umma::mn_offset(hf * HALF + row, i, KG);
            *reinterpret_cast<uint16_t *>(uB + off) = xh;
            *reinterpret_cast<uint16_t *>(uB + partB + off) = xm;
            *reinterpret_cast<uint16_t *>(uB + 2 * partB + off) = xl;
          }
        }
        cp_async_wait_all();   // this thread's copies of the A operand
        fence_proxy_async();   // this thread's operand writes -> visible to the tensor core
        umma::fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(&ops_bar);
        // every warp waits for the operands too: e^{G} in eg_s, written by the
        // A builders, is read in the epilogue
        if (!warp_all(mbar_wait_bounded(&ops_bar, (uint32_t)(folds & 1), abort, a.wait_limit))) *abort = 1;
        if (tid == 0) {
          if (!*abort) {
            umma::fence_after_sync();
            constexpr uint32_t idesc = umma::idesc_bf16_f32_mn(DK, DV);
            constexpr int pa[6] = {0, 0, 1, 0, 2, 1}, pb[6] = {0, 1, 0, 2, 0, 1};
#pragma unroll
            for (int t = 0; t < 6; ++t)
              for (int ks = 0; ks < KG / 2; ++ks)
                umma::mma_bf16(tm, umma::smem_desc_mn(smem_u32(uA + pa[t] * partA) + 256 * ks, 128, KG * 128),
                               umma::smem_desc_mn(smem_u32(uB + pb[t] * partB) + 256 * ks, 128, KG * 128), idesc,
                               t > 0 || ks > 0);
          }
          umma::commit(&mma_bar);   // with no MMA issued it completes at once
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
        const float dF = eg_s[c];
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

      // a window-full fold without a pre-fold: its A operand is built now, while
      // the stages' reads are in flight
      const bool a_early = plan.post && !plan.pre;
      if (a_early) build_a(w0, n - w0 + 1);
      if (plan.pre) {   // the window was full: fold it into the stages first
        const float none[2] = {0.0f, 0.0f};
        if (!fold_tc(0, n, none, true, true, !plan.post)) {
          failed = true;
          break;
        }
      }
      // ---- outputs of both rows.  This lane: columns 32 c + 4 j8 .. + 3 (c = 0..3)
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
      float pz[2] = {0.0f, 0.0f}, pa[2] = {0.0f, 0.0f};
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int col = 32 * c + 4 * j8;
        const float4 gk = *reinterpret_cast<const float4 *>(hsl + HeadSlot::GK + col);
        const float4 gq = *reinterpret_cast<const float4 *>(hsl + HeadSlot::GQ + col);
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          pz[hf] += dot4(f[hf][c], gk);
          pa[hf] += dot4(f[hf][c], gq);
        }
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
        const float vv = __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(hsl + HeadSlot::VB)[vrow]);
        wn[hf] = hsl[HeadSlot::BETA] * (vv - pz[hf]);
        if (j8 == 0) {
          a.out[bh * DV + vrow] = a.out_scale * fmaf(hsl[HeadSlot::MQE], wn[hf], pa[hf]);
          wring[((bh * 2 + hf) * cap + slot_n) * HALF + row] = wn[hf];
        }
      }
      if (plan.post) {   // the decode filled the window: fold all of it
        if (!fold_tc(w0, n - w0 + 1, wn, !a_early, false, true)) {
          failed = true;
          break;
        }
      }
      if (held) release();
    }
    if (failed) break;
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

bool kda_decode_fast_path(const StepArgs &a, int in_dtype) {
  return a.mode == kDecode && a.m == 1 && in_dtype == RSSM_BF16 && a.R == DV && a.C == DK && a.L <= kW &&
         a.fold_scratch != nullptr && a.rc_codes == nullptr;
}

static int heads_per_item(int H) {
  int hc = 4;
  while (H % hc) --hc;
  return hc;
}

size_t kda_fold_scratch_bytes(const rssm_layer_desc &d) {
  if (d.in_dtype != RSSM_BF16 || d.read_fmt != RSSM_READ_FP32 || d.headdim != DV || d.dstate != DK || d.window > kW)
    return 0;
  const int hc = heads_per_item(d.nheads);
  const size_t items = (size_t)d.batch * (d.nheads / hc);
  const size_t ctas = items < (size_t)kScratchCtas ? items : (size_t)kScratchCtas;
  const int KG = d.window <= 16 ? 2 : 4;
  return ctas * kSlots * hc * fold_head_bytes(KG);
}

cudaError_t kda_decode_step(const StepArgs &a, cudaStream_t s) {
  int dev = 0, sms = 0, max_smem = 0;
  cudaError_t e;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&max_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev)) != cudaSuccess) return e;
  const int budget = max_smem - 2048;   // the static shared variables
  const int hc = heads_per_item(a.H);
  int stages = kMaxStages;
  while (stages > 2 && smem_layout(a.L, hc, stages).total > budget) --stages;
  const Smem y = smem_layout(a.L, hc, stages);
  if (y.total > budget) return cudaErrorInvalidConfiguration;
  auto kern = a.L <= 16 ? kda_decode_kernel<2> : kda_decode_kernel<4>;
  if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, y.total)) != cudaSuccess) return e;
  const long long items = (long long)a.B * (a.H / hc);
  long long grid = items < sms ? items : sms;
  if (grid > kScratchCtas) grid = kScratchCtas;   // the fold scratch holds this many CTAs
  kern<<<dim3((unsigned)grid), dim3(kThreads), y.total, s>>>(a, hc, stages);
  return cudaGetLastError();
}

}  // namespace rssm
