// Host side of the librssm C ABI: argument checks, buffer layout, launches.
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <new>
#include <string>

#include <nvtx3/nvToolsExt.h>

#include "rssm_internal.h"
#include "rssm_kda.h"

struct rssm_handle {
  rssm_layer_desc d;
  rssm_layout lay;
  size_t ckpt_bytes, buf_bytes, rc_bytes, meta_bytes;
  float *ckpt;
  uint8_t *buf, *rc, *meta;
  const float *A, *D;
  long long wait_limit;
  int stall_next;   // rssm_arm_timeout_test: the next replay launch takes the timeout path
};

namespace {

// An NVTX range named after the rssm_* call it covers, open for the call's
// duration (a no-op unless a profiler that collects NVTX ranges is attached).
struct CallRange {
  explicit CallRange(const char *name) { nvtxRangePushA(name); }
  ~CallRange() { nvtxRangePop(); }
  CallRange(const CallRange &) = delete;
  CallRange &operator=(const CallRange &) = delete;
};

thread_local std::string g_err;
std::atomic<uint64_t> g_launches{0};

int fail(int code, const char *fmt, ...) __attribute__((format(printf, 2, 3)));
int fail(int code, const char *fmt, ...) {
  char msg[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(msg, sizeof msg, fmt, ap);
  va_end(ap);
  g_err = msg;
  return code;
}

int ok() {
  g_err.clear();
  return RSSM_OK;
}

int cuda_fail(cudaError_t e, const char *what) {
  return fail(RSSM_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

bool aligned(const void *p, size_t a) { return ((uintptr_t)p % a) == 0; }

int validate_desc(const rssm_layer_desc *d) {
  if (!d) return fail(RSSM_ERR_INVALID_ARG, "desc is NULL");
  if (d->kind != RSSM_MAMBA2 && d->kind != RSSM_GDN && d->kind != RSSM_KDA)
    return fail(RSSM_ERR_INVALID_ARG, "kind must be RSSM_MAMBA2, RSSM_GDN or RSSM_KDA");
  if (d->batch < 1 || d->nheads < 1 || d->headdim < 1 || d->dstate < 1)
    return fail(RSSM_ERR_INVALID_ARG, "batch, nheads, headdim and dstate must be positive");
  if ((long long)d->batch * d->nheads > (1LL << 31) - 1)
    return fail(RSSM_ERR_INVALID_ARG, "batch * nheads too large");
  if (d->kind == RSSM_MAMBA2 && (d->ngroups < 1 || d->nheads % d->ngroups))
    return fail(RSSM_ERR_INVALID_ARG, "nheads must be a positive multiple of ngroups");
  if (d->window < 1 || d->window > rssm::kMaxWindow)
    return fail(RSSM_ERR_INVALID_ARG, "window must be in [1, %d]", rssm::kMaxWindow);
  if (d->max_draft < 0 || d->max_draft > rssm::kMaxDraft || d->max_draft > d->window)
    return fail(RSSM_ERR_INVALID_ARG, "max_draft must be in [0, min(window, %d)]", rssm::kMaxDraft);
  if (d->in_dtype != RSSM_F32 && d->in_dtype != RSSM_BF16)
    return fail(RSSM_ERR_INVALID_ARG, "in_dtype must be RSSM_F32 or RSSM_BF16");
  if (d->read_fmt != RSSM_READ_FP32 && d->read_fmt != RSSM_READ_FP8_E4M3_ROW &&
      d->read_fmt != RSSM_READ_NVFP4)
    return fail(RSSM_ERR_INVALID_ARG, "unknown read_fmt");
  const bool sup = d->kind == RSSM_MAMBA2 ? rssm::mamba2_supported(d->headdim, d->dstate)
                    : d->kind == RSSM_GDN  ? rssm::gdn_supported(d->headdim, d->dstate)
                                           : rssm::kda_supported(d->headdim, d->dstate);
  if (!sup)
    return fail(RSSM_ERR_UNSUPPORTED, "no kernel for %s headdim=%d dstate=%d in this build",
                d->kind == RSSM_MAMBA2 ? "Mamba-2" : d->kind == RSSM_GDN ? "GDN" : "KDA", d->headdim, d->dstate);
  return RSSM_OK;
}

void compute_layout(const rssm_layer_desc *d, rssm_layout *L, size_t *ckpt, size_t *buf,
                    size_t *rc, size_t *meta) {
  std::memset(L, 0, sizeof *L);
  const size_t B = d->batch, H = d->nheads, R = d->headdim, C = d->dstate;
  const size_t cap = d->window + (d->max_draft > 1 ? d->max_draft : 1);
  const size_t esz = d->in_dtype == RSSM_BF16 ? 2 : 4;
  const size_t nslots = d->branching ? 2 * B : B;   // checkpoint slots
  L->cap = cap;
  *ckpt = nslots * H * R * C * sizeof(float);
  size_t off = 0;
  if (d->kind == RSSM_MAMBA2) {
    const size_t G = d->ngroups;
    L->buf_off[0] = off; off = align256(off + B * H * cap * R * esz);      // x_buf
    L->buf_off[1] = off; off = align256(off + B * G * cap * C * esz);      // B_buf
    L->buf_off[2] = off; off = align256(off + B * H * cap * sizeof(float)); // dt_buf
  } else if (d->kind == RSSM_KDA) {
    L->buf_off[0] = off; off = align256(off + B * H * cap * C * esz);      // k_buf [B,H,cap,dk]
    L->buf_off[1] = off; off = align256(off + B * H * cap * R * esz);      // v_buf [B,H,cap,dv]
    L->buf_off[2] = off; off = align256(off + B * H * cap * C * sizeof(float)); // g_buf [B,H,cap,dk]
    L->buf_off[3] = off; off = align256(off + B * H * cap * sizeof(float)); // beta_buf [B,H,cap]
    L->buf_off[4] = off; off = align256(off + B * H * cap * R * sizeof(float)); // w_buf [B,H,2,cap,dv/2]
  } else {
    L->buf_off[0] = off; off = align256(off + B * H * cap * C * esz);      // k_buf [B,H,cap,dk]
    L->buf_off[1] = off; off = align256(off + B * H * cap * R * esz);      // v_buf [B,H,2,cap,dv/2]
    L->buf_off[2] = off; off = align256(off + B * H * cap * sizeof(float)); // g_buf [B,H,cap]
    L->buf_off[3] = off; off = align256(off + B * H * cap * sizeof(float)); // beta_buf [B,H,cap]
    L->buf_off[4] = off; off = align256(off + B * H * cap * R * sizeof(float)); // w_buf [B,H,2,cap,dv/2]
  }
  if (d->branching) {   // a copy of the ring regions for rssm_branch
    L->branch_scratch_off = off;
    off = align256(off + off);
  }
  if (d->kind == RSSM_KDA) {   // operands of the decode kernel's folds, per CTA
    const size_t fs = rssm::kda_fold_scratch_bytes(*d);
    if (fs) {
      L->fold_scratch_off = off;
      off = align256(off + fs);
    }
  }
  *buf = off;
  if (d->read_fmt == RSSM_READ_FP32) {
    *rc = 0;
  } else if (d->read_fmt == RSSM_READ_FP8_E4M3_ROW) {
    L->rc_codes_off = 0;
    L->rc_scales_off = align256(nslots * H * R * C);
    *rc = align256(L->rc_scales_off + nslots * H * R * sizeof(float));
  } else {
    L->rc_codes_off = 0;
    L->rc_scales_off = align256(nslots * H * R * C / 2);
    *rc = align256(L->rc_scales_off + nslots * H * R * (C / 16));
  }
  off = 0;
  L->meta_start_off = off; off = align256(off + B * 4);
  L->meta_len_off = off; off = align256(off + B * 4);
  L->meta_pending_off = off; off = align256(off + B * 4);
  L->meta_flushes_off = off; off = align256(off + B * 4);
  L->meta_arrivals_off = off; off = align256(off + B * 4);
  L->meta_status_off = off; off = align256(off + 4);
  if (d->branching) {
    L->meta_slot_off = off; off = align256(off + B * 4);
    L->meta_dst_off = off; off = align256(off + B * 4);
    L->meta_seen_off = off; off = align256(off + B * 4);
    L->meta_work_off = off; off = align256(off + 5 * B * 4);
  }
  *meta = off;
}

rssm::StepArgs step_args(const rssm_handle *h, int mode, int m) {
  rssm::StepArgs a;
  std::memset(&a, 0, sizeof a);
  const rssm_layer_desc &d = h->d;
  a.B = d.batch; a.H = d.nheads;
  a.G = d.kind == RSSM_MAMBA2 ? d.ngroups : 1;
  a.hpg = d.nheads / a.G;
  a.R = d.headdim; a.C = d.dstate;
  a.L = d.window; a.cap = (int)h->lay.cap;
  a.m = m; a.mode = mode; a.auto_flush = d.auto_flush != 0;
  a.out_scale = d.out_scale;
  a.wait_limit = h->wait_limit;
  a.A = h->A; a.D = h->D;
  a.hc = h->ckpt;
  if (d.branching) {
    a.slot = reinterpret_cast<const int32_t *>(h->meta + h->lay.meta_slot_off);
    a.dst = reinterpret_cast<const int32_t *>(h->meta + h->lay.meta_dst_off);
  }
  a.rc_codes = h->rc ? h->rc + h->lay.rc_codes_off : nullptr;
  a.rc_scales = h->rc ? h->rc + h->lay.rc_scales_off : nullptr;
  a.buf0 = h->buf + h->lay.buf_off[0];
  a.buf1 = h->buf + h->lay.buf_off[1];
  a.buf2 = reinterpret_cast<float *>(h->buf + h->lay.buf_off[2]);
  if (d.kind != RSSM_MAMBA2) {
    a.buf3 = reinterpret_cast<float *>(h->buf + h->lay.buf_off[3]);
    a.buf4 = reinterpret_cast<float *>(h->buf + h->lay.buf_off[4]);
  }
  if (h->lay.fold_scratch_off) a.fold_scratch = h->buf + h->lay.fold_scratch_off;
  a.start = reinterpret_cast<int32_t *>(h->meta + h->lay.meta_start_off);
  a.len = reinterpret_cast<int32_t *>(h->meta + h->lay.meta_len_off);
  a.pending = reinterpret_cast<int32_t *>(h->meta + h->lay.meta_pending_off);
  a.flushes = reinterpret_cast<int32_t *>(h->meta + h->lay.meta_flushes_off);
  a.arrivals = reinterpret_cast<int32_t *>(h->meta + h->lay.meta_arrivals_off);
  a.status = reinterpret_cast<uint32_t *>(h->meta + h->lay.meta_status_off);
  return a;
}

int n_inputs(const rssm_handle *h) { return h->d.kind == RSSM_MAMBA2 ? 4 : 5; }

int check_inputs(const rssm_handle *h, const void *const *in, const void *out) {
  if (!in) return fail(RSSM_ERR_INVALID_ARG, "in is NULL");
  for (int i = 0; i < n_inputs(h); ++i) {
    if (!in[i]) return fail(RSSM_ERR_INVALID_ARG, "in[%d] is NULL", i);
    if (!aligned(in[i], 16)) return fail(RSSM_ERR_INVALID_ARG, "in[%d] is not 16-byte aligned", i);
  }
  if (!out) return fail(RSSM_ERR_INVALID_ARG, "out is NULL");
  if (!aligned(out, 16)) return fail(RSSM_ERR_INVALID_ARG, "out is not 16-byte aligned");
  if (h->d.kind == RSSM_MAMBA2 && (!h->A || !h->D))
    return fail(RSSM_ERR_STATE, "Mamba-2 parameters not set (rssm_set_params)");
  return RSSM_OK;
}

int32_t *meta_i32(const rssm_handle *h, size_t off) { return reinterpret_cast<int32_t *>(h->meta + off); }

// Layers that branch: before each replay launch, give the rows that fold in it
// a free checkpoint slot (no-op otherwise).
int plan_slots_for(rssm_handle *h, const rssm::StepArgs &a, cudaStream_t s) {
  if (!h->d.branching) return RSSM_OK;
  cudaError_t e = rssm::plan_slots(a, meta_i32(h, h->lay.meta_slot_off), meta_i32(h, h->lay.meta_dst_off),
                                   meta_i32(h, h->lay.meta_seen_off), meta_i32(h, h->lay.meta_work_off), s);
  g_launches.fetch_add(1, std::memory_order_relaxed);
  if (e != cudaSuccess) return cuda_fail(e, "slot planner launch");
  return RSSM_OK;
}

cudaError_t replay_launch(const rssm_handle *h, const rssm::StepArgs &a, cudaStream_t s) {
  switch (h->d.kind) {
    case RSSM_MAMBA2: return rssm::mamba2_step(a, h->d.in_dtype, h->d.read_fmt, s);
    case RSSM_GDN: return rssm::gdn_step(a, h->d.in_dtype, h->d.read_fmt, s);
    default: return rssm::kda_step(a, h->d.in_dtype, h->d.read_fmt, s);
  }
}

int launch_step(rssm_handle *h, int mode, int m, const void *const *in, void *out,
                const int32_t *mask, cudaStream_t s) {
  rssm::StepArgs a = step_args(h, mode, m);
  if (in)
    for (int i = 0; i < n_inputs(h); ++i) a.in[i] = in[i];
  a.out = static_cast<float *>(out);
  a.mask = mask;
  int rc = plan_slots_for(h, a, s);
  if (rc) return rc;
  a.stall_test = h->stall_next;   // armed self-test: this launch takes the timeout path
  h->stall_next = 0;
  cudaError_t e = replay_launch(h, a, s);
  g_launches.fetch_add(1, std::memory_order_relaxed);
  if (e != cudaSuccess) return cuda_fail(e, "replay kernel launch");
  return ok();
}

}  // namespace

extern "C" {

int rssm_workspace_size(const rssm_layer_desc *desc, size_t *ckpt_bytes, size_t *buf_bytes,
                        size_t *read_copy_bytes, size_t *meta_bytes, rssm_layout *layout) {
  const CallRange call_range(__func__);
  int rc = validate_desc(desc);
  if (rc) return rc;
  if (!ckpt_bytes || !buf_bytes || !read_copy_bytes || !meta_bytes)
    return fail(RSSM_ERR_INVALID_ARG, "size outputs must not be NULL");
  rssm_layout tmp;
  compute_layout(desc, layout ? layout : &tmp, ckpt_bytes, buf_bytes, read_copy_bytes, meta_bytes);
  return ok();
}

int rssm_create(const rssm_layer_desc *desc, void *ckpt_dev, void *buf_dev, void *read_copy_dev,
                void *meta_dev, rssm_handle **out) {
  const CallRange call_range(__func__);
  int rc = validate_desc(desc);
  if (rc) return rc;
  if (!out) return fail(RSSM_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  if (!ckpt_dev || !buf_dev || !meta_dev)
    return fail(RSSM_ERR_INVALID_ARG, "ckpt, buf and meta must not be NULL");
  if (!aligned(ckpt_dev, 256) || !aligned(buf_dev, 256) || !aligned(meta_dev, 256))
    return fail(RSSM_ERR_INVALID_ARG, "device buffers must be 256-byte aligned");
  if (desc->read_fmt != RSSM_READ_FP32) {
    if (!read_copy_dev) return fail(RSSM_ERR_INVALID_ARG, "read_fmt needs a read_copy buffer");
    if (!aligned(read_copy_dev, 256)) return fail(RSSM_ERR_INVALID_ARG, "read_copy must be 256-byte aligned");
  }
  rssm_handle *h = new (std::nothrow) rssm_handle;
  if (!h) return fail(RSSM_ERR_INVALID_ARG, "out of host memory");
  std::memset(h, 0, sizeof *h);
  h->d = *desc;
  compute_layout(desc, &h->lay, &h->ckpt_bytes, &h->buf_bytes, &h->rc_bytes, &h->meta_bytes);
  h->ckpt = static_cast<float *>(ckpt_dev);
  h->buf = static_cast<uint8_t *>(buf_dev);
  h->rc = desc->read_fmt == RSSM_READ_FP32 ? nullptr : static_cast<uint8_t *>(read_copy_dev);
  h->meta = static_cast<uint8_t *>(meta_dev);
  h->wait_limit = rssm::kDefaultWaitLimit;
  *out = h;
  return ok();
}

int rssm_destroy(rssm_handle *h) {
  const CallRange call_range(__func__);
  delete h;
  return ok();
}

int rssm_reset(rssm_handle *h, rssm_stream_t stream) {
  const CallRange call_range(__func__);
  if (!h) return fail(RSSM_ERR_INVALID_ARG, "handle is NULL");
  cudaError_t e = cudaMemsetAsync(h->meta, 0, h->meta_bytes, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(meta)");
  if (h->d.branching) {
    e = rssm::init_slots(h->d.batch, meta_i32(h, h->lay.meta_slot_off), meta_i32(h, h->lay.meta_dst_off),
                         (cudaStream_t)stream);
    g_launches.fetch_add(1, std::memory_order_relaxed);
    if (e != cudaSuccess) return cuda_fail(e, "slot init launch");
  }
  return ok();
}

int rssm_set_params(rssm_handle *h, const float *A_dev, const float *D_dev) {
  const CallRange call_range(__func__);
  if (!h) return fail(RSSM_ERR_INVALID_ARG, "handle is NULL");
  if (h->d.kind == RSSM_MAMBA2 && (!A_dev || !D_dev))
    return fail(RSSM_ERR_INVALID_ARG, "A and D must not be NULL");
  h->A = A_dev;
  h->D = D_dev;
  return ok();
}

int rssm_set_wait_limit(rssm_handle *h, long long cycles) {
  const CallRange call_range(__func__);
  if (!h) return fail(RSSM_ERR_INVALID_ARG, "handle is NULL");
  if (cycles < 0) return fail(RSSM_ERR_INVALID_ARG, "wait limit must be >= 0 (0 = default)");
  h->wait_limit = cycles == 0 ? rssm::kDefaultWaitLimit : cycles;
  return ok();
}

int rssm_arm_timeout_test(rssm_handle *h) {
  const CallRange call_range(__func__);
  if (!h) return fail(RSSM_ERR_INVALID_ARG, "handle is NULL");
  if (h->d.kind == RSSM_KDA && rssm::kda_fold_scratch_bytes(h->d) == 0)
    return fail(RSSM_ERR_UNSUPPORTED, "only the KDA decode serving kernel (bf16 inputs) has waits to run out");
  h->stall_next = 1;
  return ok();
}

int rssm_decode_step(rssm_handle *h, const void *const *in, void *out_dev, rssm_stream_t stream) {
  const CallRange call_range(__func__);
  if (!h) return fail(RSSM_ERR_INVALID_ARG, "handle is NULL");
  int rc = check_inputs(h, in, out_dev);
  if (rc) return rc;
  return launch_step(h, rssm::kDecode, 1, in, out_dev, nullptr, (cudaStream_t)stream);
}

int rssm_verify(rssm_handle *h, int k, const void *const *in, void *out_dev, rssm_stream_t stream) {
  const CallRange call_range(__func__);
  if (!h) return fail(RSSM_ERR_INVALID_ARG, "handle is NULL");
  if (h->d.max_draft < 1) return fail(RSSM_ERR_STATE, "handle was created with max_draft = 0");
  if (k < 1 || k > h->d.max_draft)
    return fail(RSSM_ERR_CAPACITY, "k = %d outside [1, max_draft = %d]", k, h->d.max_draft);
  int rc = check_inputs(h, in, out_dev);
  if (rc) return rc;
  return launch_step(h, rssm::kVerify, k, in, out_dev, nullptr, (cudaStream_t)stream);
}

int rssm_rollback(rssm_handle *h, const int32_t *n_reject_dev, rssm_stream_t stream) {
  const CallRange call_range(__func__);
  if (!h) return fail(RSSM_ERR_INVALID_ARG, "handle is NULL");
  if (!n_reject_dev) return fail(RSSM_ERR_INVALID_ARG, "n_reject is NULL");
  rssm::StepArgs a = step_args(h, rssm::kVerify, 0);
  cudaError_t e = rssm::rollback(a.B, n_reject_dev, a.len, a.pending, a.status, (cudaStream_t)stream);
  g_launches.fetch_add(1, std::memory_order_relaxed);
  if (e != cudaSuccess) return cuda_fail(e, "rollback launch");
  return ok();
}

int rssm_flush(rssm_handle *h, const int32_t *row_mask_dev, rssm_stream_t stream) {
  const CallRange call_range(__func__);
  if (!h) return fail(RSSM_ERR_INVALID_ARG, "handle is NULL");
  if (h->d.kind == RSSM_MAMBA2 && (!h->A || !h->D))
    return fail(RSSM_ERR_STATE, "Mamba-2 parameters not set (rssm_set_params)");
  return launch_step(h, rssm::kFlush, 0, nullptr, nullptr, row_mask_dev, (cudaStream_t)stream);
}

int rssm_quantize_read_copy(rssm_handle *h, rssm_stream_t stream) {
  const CallRange call_range(__func__);
  if (!h) return fail(RSSM_ERR_INVALID_ARG, "handle is NULL");
  if (!h->rc) return fail(RSSM_ERR_STATE, "handle has no read copy (read_fmt = RSSM_READ_FP32)");
  rssm::QuantArgs q;
  q.rows = (size_t)h->d.batch * (h->d.branching ? 2 : 1) * h->d.nheads * h->d.headdim;
  q.C = h->d.dstate;
  q.hc = h->ckpt;
  q.codes = h->rc + h->lay.rc_codes_off;
  q.scales = h->rc + h->lay.rc_scales_off;
  cudaError_t e = rssm::quantize_read_copy(q, h->d.read_fmt, (cudaStream_t)stream);
  g_launches.fetch_add(1, std::memory_order_relaxed);
  if (e != cudaSuccess) return cuda_fail(e, "quantize launch");
  return ok();
}

int rssm_conventional_step(rssm_handle *h, const float *state_in_dev, float *state_out_dev,
                           const void *const *in, void *out_dev, rssm_stream_t stream) {
  const CallRange call_range(__func__);
  if (!h) return fail(RSSM_ERR_INVALID_ARG, "handle is NULL");
  if (!state_in_dev || !state_out_dev) return fail(RSSM_ERR_INVALID_ARG, "state pointers must not be NULL");
  if (!aligned(state_in_dev, 16) || !aligned(state_out_dev, 16))
    return fail(RSSM_ERR_INVALID_ARG, "state pointers must be 16-byte aligned");
  int rc = check_inputs(h, in, out_dev);
  if (rc) return rc;
  rssm::ConvArgs a;
  std::memset(&a, 0, sizeof a);
  a.B = h->d.batch; a.H = h->d.nheads;
  a.G = h->d.kind == RSSM_MAMBA2 ? h->d.ngroups : 1;
  a.hpg = a.H / a.G;
  a.R = h->d.headdim; a.C = h->d.dstate;
  a.out_scale = h->d.out_scale;
  a.A = h->A; a.D = h->D;
  a.state_in = state_in_dev; a.state_out = state_out_dev;
  for (int i = 0; i < n_inputs(h); ++i) a.in[i] = in[i];
  a.out = static_cast<float *>(out_dev);
  cudaError_t e = h->d.kind == RSSM_MAMBA2
                      ? rssm::mamba2_conventional(a, h->d.in_dtype, RSSM_READ_FP32, (cudaStream_t)stream)
                  : h->d.kind == RSSM_GDN
                      ? rssm::gdn_conventional(a, h->d.in_dtype, RSSM_READ_FP32, (cudaStream_t)stream)
                      : rssm::kda_conventional(a, h->d.in_dtype, (cudaStream_t)stream);
  g_launches.fetch_add(1, std::memory_order_relaxed);
  if (e != cudaSuccess) return cuda_fail(e, "conventional kernel launch");
  return ok();
}

int rssm_conventional_step_quantized(rssm_handle *h, const void *codes_in_dev, const void *scales_in_dev,
                                     void *codes_out_dev, void *scales_out_dev, const void *const *in,
                                     void *out_dev, rssm_stream_t stream) {
  const CallRange call_range(__func__);
  if (!h) return fail(RSSM_ERR_INVALID_ARG, "handle is NULL");
  if (h->d.read_fmt == RSSM_READ_FP32)
    return fail(RSSM_ERR_STATE, "the layer has no low-precision format (read_fmt is RSSM_READ_FP32)");
  if (h->d.kind == RSSM_KDA)
    return fail(RSSM_ERR_UNSUPPORTED, "no stored low-precision state baseline for KDA layers");
  if (!codes_in_dev || !scales_in_dev || !codes_out_dev || !scales_out_dev)
    return fail(RSSM_ERR_INVALID_ARG, "state code and scale pointers must not be NULL");
  if (!aligned(codes_in_dev, 16) || !aligned(codes_out_dev, 16))
    return fail(RSSM_ERR_INVALID_ARG, "state code pointers must be 16-byte aligned");
  if (h->d.read_fmt == RSSM_READ_FP8_E4M3_ROW && (!aligned(scales_in_dev, 4) || !aligned(scales_out_dev, 4)))
    return fail(RSSM_ERR_INVALID_ARG, "FP8 row scales must be 4-byte aligned");
  int rc = check_inputs(h, in, out_dev);
  if (rc) return rc;
  rssm::ConvArgs a;
  std::memset(&a, 0, sizeof a);
  a.B = h->d.batch; a.H = h->d.nheads;
  a.G = h->d.kind == RSSM_MAMBA2 ? h->d.ngroups : 1;
  a.hpg = a.H / a.G;
  a.R = h->d.headdim; a.C = h->d.dstate;
  a.out_scale = h->d.out_scale;
  a.A = h->A; a.D = h->D;
  a.codes_in = static_cast<const uint8_t *>(codes_in_dev);
  a.scales_in = scales_in_dev;
  a.codes_out = static_cast<uint8_t *>(codes_out_dev);
  a.scales_out = scales_out_dev;
  for (int i = 0; i < n_inputs(h); ++i) a.in[i] = in[i];
  a.out = static_cast<float *>(out_dev);
  cudaError_t e = h->d.kind == RSSM_MAMBA2
                      ? rssm::mamba2_conventional(a, h->d.in_dtype, h->d.read_fmt, (cudaStream_t)stream)
                      : rssm::gdn_conventional(a, h->d.in_dtype, h->d.read_fmt, (cudaStream_t)stream);
  g_launches.fetch_add(1, std::memory_order_relaxed);
  if (e != cudaSuccess) return cuda_fail(e, "quantized-state conventional kernel launch");
  return ok();
}

int rssm_branch(rssm_handle *h, const int32_t *parent_dev, rssm_stream_t stream) {
  const CallRange call_range(__func__);
  if (!h) return fail(RSSM_ERR_INVALID_ARG, "handle is NULL");
  if (!parent_dev) return fail(RSSM_ERR_INVALID_ARG, "parent is NULL");
  if (!h->d.branching) return fail(RSSM_ERR_STATE, "handle was created with branching = 0");
  rssm::BranchArgs b;
  std::memset(&b, 0, sizeof b);
  const rssm_layer_desc &d = h->d;
  b.B = d.batch;
  b.slot = meta_i32(h, h->lay.meta_slot_off);
  b.dst = meta_i32(h, h->lay.meta_dst_off);
  b.seen = meta_i32(h, h->lay.meta_seen_off);
  int32_t *work = meta_i32(h, h->lay.meta_work_off);
  b.freelist = work;
  b.eff = work + 4 * (size_t)d.batch;
  b.start = meta_i32(h, h->lay.meta_start_off);
  b.len = meta_i32(h, h->lay.meta_len_off);
  b.pending = meta_i32(h, h->lay.meta_pending_off);
  b.flushes = meta_i32(h, h->lay.meta_flushes_off);
  b.status = reinterpret_cast<uint32_t *>(h->meta + h->lay.meta_status_off);
  // each ring region is [B][outer][cap][entry]
  const int H = d.nheads;
  const int esz = d.in_dtype == RSSM_BF16 ? 2 : 4;
  if (d.kind == RSSM_MAMBA2) {
    const int outer[3] = {H, d.ngroups, H}, entry[3] = {d.headdim * esz, d.dstate * esz, 4};
    b.nreg = 3;
    for (int r = 0; r < 3; ++r) b.outer[r] = outer[r], b.entry_bytes[r] = entry[r];
  } else if (d.kind == RSSM_KDA) {   // k [H][cap][dk] | v [H][cap][dv] | g [H][cap][dk] fp32 | beta | w [2H][cap][dv/2]
    const int outer[5] = {H, H, H, H, 2 * H};
    const int entry[5] = {d.dstate * esz, d.headdim * esz, d.dstate * 4, 4, d.headdim / 2 * 4};
    b.nreg = 5;
    for (int r = 0; r < 5; ++r) b.outer[r] = outer[r], b.entry_bytes[r] = entry[r];
  } else {   // k [H][cap][dk] | v [2H][cap][dv/2] | g, beta [H][cap] | w [2H][cap][dv/2] fp32
    const int outer[5] = {H, 2 * H, H, H, 2 * H};
    const int entry[5] = {d.dstate * esz, d.headdim / 2 * esz, 4, 4, d.headdim / 2 * 4};
    b.nreg = 5;
    for (int r = 0; r < 5; ++r) b.outer[r] = outer[r], b.entry_bytes[r] = entry[r];
  }
  b.cap = (int)h->lay.cap;
  for (int r = 0; r < b.nreg; ++r) {
    b.ring[r] = h->buf + h->lay.buf_off[r];
    b.scratch[r] = h->buf + h->lay.branch_scratch_off + h->lay.buf_off[r];
  }
  cudaError_t e = rssm::branch_rows(b, parent_dev, work, (cudaStream_t)stream);
  g_launches.fetch_add(2, std::memory_order_relaxed);
  if (e != cudaSuccess) return cuda_fail(e, "branch launches");
  return ok();
}

int rssm_restore(rssm_handle *h, const int32_t *keep_dev, rssm_stream_t stream) {
  const CallRange call_range(__func__);
  if (!h) return fail(RSSM_ERR_INVALID_ARG, "handle is NULL");
  if (!keep_dev) return fail(RSSM_ERR_INVALID_ARG, "keep is NULL");
  rssm::StepArgs a = step_args(h, rssm::kDecode, 0);
  cudaError_t e = rssm::restore_rows(a.B, keep_dev, a.len, a.pending, a.status, (cudaStream_t)stream);
  g_launches.fetch_add(1, std::memory_order_relaxed);
  if (e != cudaSuccess) return cuda_fail(e, "restore launch");
  return ok();
}

int rssm_get_slots(rssm_handle *h, int32_t *out_dev, rssm_stream_t stream) {
  const CallRange call_range(__func__);
  if (!h) return fail(RSSM_ERR_INVALID_ARG, "handle is NULL");
  if (!out_dev) return fail(RSSM_ERR_INVALID_ARG, "out is NULL");
  if (!h->d.branching) return fail(RSSM_ERR_STATE, "handle was created with branching = 0");
  cudaError_t e = rssm::effective_slots(h->d.batch, meta_i32(h, h->lay.meta_slot_off),
                                        meta_i32(h, h->lay.meta_dst_off), meta_i32(h, h->lay.meta_seen_off),
                                        meta_i32(h, h->lay.meta_flushes_off), out_dev, (cudaStream_t)stream);
  g_launches.fetch_add(1, std::memory_order_relaxed);
  if (e != cudaSuccess) return cuda_fail(e, "slot lookup launch");
  return ok();
}

// A layer's whole replay state as one host blob: checkpoint (all slots) | read
// copy | ring regions (not the branch scratch) | meta.
namespace {
struct Piece {
  uint8_t *dev;
  size_t bytes;
};
int state_pieces(const rssm_handle *h, Piece (&p)[4]) {
  p[0] = {reinterpret_cast<uint8_t *>(h->ckpt), h->ckpt_bytes};
  p[1] = {h->rc, h->rc ? h->rc_bytes : 0};
  p[2] = {h->buf, h->d.branching ? h->lay.branch_scratch_off
                  : h->lay.fold_scratch_off ? h->lay.fold_scratch_off : h->buf_bytes};
  p[3] = {h->meta, h->meta_bytes};
  return 4;
}
}  // namespace

int rssm_state_bytes(rssm_handle *h, size_t *bytes) {
  const CallRange call_range(__func__);
  if (!h) return fail(RSSM_ERR_INVALID_ARG, "handle is NULL");
  if (!bytes) return fail(RSSM_ERR_INVALID_ARG, "bytes is NULL");
  Piece p[4];
  size_t total = 0;
  for (int i = 0; i < state_pieces(h, p); ++i) total += p[i].bytes;
  *bytes = total;
  return ok();
}

static int copy_state(rssm_handle *h, uint8_t *host, size_t bytes, bool to_host, cudaStream_t s) {
  if (!h) return fail(RSSM_ERR_INVALID_ARG, "handle is NULL");
  if (!host) return fail(RSSM_ERR_INVALID_ARG, "host buffer is NULL");
  Piece p[4];
  const int n = state_pieces(h, p);
  size_t total = 0;
  for (int i = 0; i < n; ++i) total += p[i].bytes;
  if (bytes != total) return fail(RSSM_ERR_INVALID_ARG, "host buffer has %zu bytes, the state has %zu", bytes, total);
  size_t off = 0;
  for (int i = 0; i < n; ++i) {
    if (p[i].bytes == 0) continue;
    cudaError_t e = to_host ? cudaMemcpyAsync(host + off, p[i].dev, p[i].bytes, cudaMemcpyDeviceToHost, s)
                            : cudaMemcpyAsync(p[i].dev, host + off, p[i].bytes, cudaMemcpyHostToDevice, s);
    if (e != cudaSuccess) return cuda_fail(e, to_host ? "state export copy" : "state import copy");
    off += p[i].bytes;
  }
  return ok();
}

int rssm_export_state(rssm_handle *h, void *host_dst, size_t bytes, rssm_stream_t stream) {
  const CallRange call_range(__func__);
  return copy_state(h, static_cast<uint8_t *>(host_dst), bytes, true, (cudaStream_t)stream);
}

int rssm_import_state(rssm_handle *h, const void *host_src, size_t bytes, rssm_stream_t stream) {
  const CallRange call_range(__func__);
  return copy_state(h, static_cast<uint8_t *>(const_cast<void *>(host_src)), bytes, false, (cudaStream_t)stream);
}

int rssm_get_bookkeeping(rssm_handle *h, int32_t *out_dev, rssm_stream_t stream) {
  const CallRange call_range(__func__);
  if (!h) return fail(RSSM_ERR_INVALID_ARG, "handle is NULL");
  if (!out_dev) return fail(RSSM_ERR_INVALID_ARG, "out is NULL");
  rssm::StepArgs a = step_args(h, rssm::kDecode, 0);
  cudaError_t e = rssm::gather_bookkeeping(a.B, a.start, a.len, a.pending, a.flushes, out_dev,
                                           (cudaStream_t)stream);
  g_launches.fetch_add(1, std::memory_order_relaxed);
  if (e != cudaSuccess) return cuda_fail(e, "bookkeeping gather launch");
  return ok();
}

int rssm_get_lengths(rssm_handle *h, int32_t *len_dev, int32_t *pending_dev, rssm_stream_t stream) {
  const CallRange call_range(__func__);
  if (!h) return fail(RSSM_ERR_INVALID_ARG, "handle is NULL");
  if (!len_dev || !pending_dev) return fail(RSSM_ERR_INVALID_ARG, "len or pending is NULL");
  const size_t n = sizeof(int32_t) * (size_t)h->d.batch;
  cudaError_t e = cudaMemcpyAsync(len_dev, h->meta + h->lay.meta_len_off, n, cudaMemcpyDeviceToDevice,
                                  (cudaStream_t)stream);
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(pending_dev, h->meta + h->lay.meta_pending_off, n, cudaMemcpyDeviceToDevice,
                        (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "copying the window lengths");
  return ok();
}

int rssm_get_status(rssm_handle *h, uint32_t *bits, int clear, rssm_stream_t stream) {
  const CallRange call_range(__func__);
  if (!h) return fail(RSSM_ERR_INVALID_ARG, "handle is NULL");
  if (!bits) return fail(RSSM_ERR_INVALID_ARG, "bits is NULL");
  uint32_t *dev = reinterpret_cast<uint32_t *>(h->meta + h->lay.meta_status_off);
  cudaError_t e = cudaMemcpyAsync(bits, dev, sizeof(uint32_t), cudaMemcpyDeviceToHost, (cudaStream_t)stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e == cudaSuccess && clear) e = cudaMemsetAsync(dev, 0, sizeof(uint32_t), (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "reading the status word");
  return ok();
}

const char *rssm_last_error_string(void) { return g_err.c_str(); }

uint64_t rssm_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

}  // extern "C"

// ---------------------------------------------------------------------------
// Decode step with library-owned scratch (rssm_decode_step_static_scratch).
//
// The replay kernel needs one int32 arrival counter per sequence: the CTAs of a
// sequence count themselves in, and the last one moves the ring pointers.
// rssm_decode_step keeps those counters in the caller's meta buffer.  Some
// callers cannot hand the library any memory beyond the layer's own buffers
// at call time: code that records decode steps into a CUDA graph (no
// allocation may happen inside the capture), serving engines that reserve all
// device memory up front and forbid later cudaMalloc, and latency-critical
// loops that must avoid cudaMalloc's implicit device synchronisation.  For
// them the counters below live in a fixed array in the library's own device
// image, so the call allocates nothing.
namespace {

static __device__ __align__(256) int32_t g_static_arrivals[RSSM_STATIC_SCRATCH_MAX_BATCH];

constexpr int kMaxDevices = 64;
std::atomic<int32_t *> g_static_arrivals_dev[kMaxDevices];

// Device address of g_static_arrivals for the current device (host code may
// not use the symbol itself as an address).  Looked up once per device.
int static_arrivals_for_current_device(int32_t **out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(RSSM_ERR_UNSUPPORTED, "device index %d too large", dev);
  int32_t *p = g_static_arrivals_dev[dev].load(std::memory_order_acquire);
  if (!p) {
    e = cudaGetSymbolAddress(reinterpret_cast<void **>(&p), g_static_arrivals);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(g_static_arrivals)");
    g_static_arrivals_dev[dev].store(p, std::memory_order_release);
  }
  *out = p;
  return RSSM_OK;
}

}  // namespace

extern "C" int rssm_decode_step_static_scratch(rssm_handle *h, const void *const *in, void *out_dev,
                                               rssm_stream_t stream) {
  const CallRange call_range(__func__);
  if (!h) return fail(RSSM_ERR_INVALID_ARG, "handle is NULL");
  if (h->d.batch > RSSM_STATIC_SCRATCH_MAX_BATCH)
    return fail(RSSM_ERR_INVALID_ARG,
                "batch %d exceeds the %d sequences the library's static scratch holds; "
                "use rssm_decode_step",
                h->d.batch, RSSM_STATIC_SCRATCH_MAX_BATCH);
  int rc = check_inputs(h, in, out_dev);
  if (rc) return rc;
  int32_t *arrivals = nullptr;
  rc = static_arrivals_for_current_device(&arrivals);
  if (rc) return rc;
  // The counters must start at zero; a previous call leaves them at zero unless
  // it was cut short, so clear the ones this call uses.
  cudaError_t e = cudaMemsetAsync(arrivals, 0, sizeof(int32_t) * (size_t)h->d.batch, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(static scratch)");
  rssm::StepArgs a = step_args(h, rssm::kDecode, 1);
  for (int i = 0; i < n_inputs(h); ++i) a.in[i] = in[i];
  a.out = static_cast<float *>(out_dev);
  a.arrivals = arrivals;
  rc = plan_slots_for(h, a, (cudaStream_t)stream);
  if (rc) return rc;
  a.stall_test = h->stall_next;
  h->stall_next = 0;
  e = replay_launch(h, a, (cudaStream_t)stream);
  g_launches.fetch_add(1, std::memory_order_relaxed);
  if (e != cudaSuccess) return cuda_fail(e, "replay kernel launch");
  return ok();
}
