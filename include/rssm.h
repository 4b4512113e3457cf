/*
 * rssm.h -- C ABI of librssm, the ReplaySSM decode hot path for one GPU
 * (NVIDIA B200, sm_100a).
 *
 * Source of the method.  The three web pages titled "ReplaySSM: Rethinking
 * State Storage for Faster Hybrid-Model Decoding" (deskofai.com news summary,
 * cited below as [summary ¶n]; nexus-ai-blog.com guide, [guide "section"];
 * babnews.org teaser, [teaser]) describe it:
 *   - a layer's state is stored as a checkpoint plus a buffer of recent inputs;
 *     output computation is separated from state updates [summary ¶2];
 *   - instead of rewriting the full state every token, inputs are cached and
 *     folded in ("flushed") when the buffer fills; draft inputs are appended,
 *     and rejected drafts are dropped by moving a pointer, with no per-token
 *     state snapshots [summary ¶3];
 *   - the checkpoint stays high precision for the recurrence while a
 *     low-precision (NVFP4) copy serves the reads [summary ¶4];
 *   - window L = 16 is the default [summary ¶6];
 *   - Mamba-2, Gated DeltaNet and KDA are the SSM layers [teaser].
 * The pages print no formula.  The library implements the Mamba-2 and gated
 * delta-rule recurrences (Mamba-2 SSD; gated delta rule) in replay form:
 *   Mamba-2 (a_r = dt_r * A_h, seg(s,t) = sum_{s<r<=t} a_r, G_t = seg(0,t)):
 *     y_t = e^{G_t} h_c C_t + sum_{s<=t} e^{seg(s,t)} dt_s (B_s . C_t) x_s + D_h x_t
 *     flush: h_c <- e^{G_l} h_c + sum_{s<=l} e^{seg(s,l)} dt_s x_s B_s^T
 *   Gated DeltaNet (a_r = ln alpha_r), WY/UT form with u_t = h_c k_t:
 *     w_t = beta_t (v_t - e^{G_t} u_t - sum_{s<t} e^{seg(s,t)} (k_s . k_t) w_s)
 *     o_t = out_scale (e^{G_t} h_c q_t + sum_{s<=t} e^{seg(s,t)} (k_s . q_t) w_s)
 *     flush: h_c <- e^{G_l} h_c + sum_{s<=l} e^{seg(s,l)} w_s k_s^T
 *   KDA (one gate per key channel, a_r = ln alpha_r elementwise, e^{.} and
 *   (.) elementwise): as GDN with e^{G_t} u_t -> h_c (e^{G_t} (.) k_t),
 *   (k_s . k_t) e^{seg} -> (k_s (.) e^{seg(s,t)}) . k_t, likewise for q_t, and
 *     flush: h_c <- h_c Diag(e^{G_l}) + sum_{s<=l} w_s (k_s (.) e^{seg(s,l)})^T
 * which equal the token-by-token recurrences exactly (up to rounding).
 *
 * Conventions for every call
 *   - Return value: RSSM_OK or an RSSM_ERR_* code.  On an argument error the
 *     call returns at once and enqueues nothing.  rssm_last_error_string()
 *     returns a thread-local message for the last failing call on the thread.
 *   - Memory: the caller owns every buffer; the library keeps raw pointers.
 *     Pointers named *_dev are device pointers; others are host pointers.
 *     Device buffers must be 256-byte aligned (cudaMalloc / torch allocations
 *     are).  The handle itself is a small host object.
 *   - Asynchrony: all device work is enqueued on the given stream (NULL = the
 *     legacy default stream) and nothing waits for it, except
 *     rssm_get_status, which synchronises that stream.
 *   - Per-sequence device errors (a row whose window would overflow, a
 *     rollback larger than its pending drafts, a decode while drafts are
 *     pending) leave that row untouched -- no output written, no state or
 *     pointer moved -- and set a sticky bit in the device status word.
 *   - Row-major layouts; the last index is contiguous.
 *   - Tracing: every call that returns an int is an NVTX range named after
 *     the call (a no-op unless a profiler collecting NVTX ranges is attached).
 */
#ifndef RSSM_H
#define RSSM_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *rssm_stream_t; /* a cudaStream_t */

/* Status codes returned by every call. */
enum {
  RSSM_OK = 0,
  RSSM_ERR_INVALID_ARG = 1, /* null pointer, bad size, misaligned buffer   */
  RSSM_ERR_UNSUPPORTED = 2, /* shape/format this build has no kernel for   */
  RSSM_ERR_CAPACITY = 3,    /* more drafts than the window can hold        */
  RSSM_ERR_STATE = 4,       /* call not valid in the handle's state        */
  RSSM_ERR_CUDA = 5,        /* a CUDA runtime call or launch failed        */
  RSSM_ERR_TIMEOUT = 6      /* reserved for host-side waits                */
};

/* Sticky device status bits (rssm_get_status). */
enum {
  RSSM_STATUS_CAPACITY = 1u << 0, /* row could not append: window full, auto_flush off */
  RSSM_STATUS_STATE = 1u << 1,    /* row refused: drafts pending / bad rollback count  */
  RSSM_STATUS_TIMEOUT = 1u << 2   /* a bounded wait for an asynchronous copy gave up   */
};
/* After RSSM_STATUS_TIMEOUT the launch that set it was cut short: its outputs,
 * the rows' pointers and any fold it was making are unspecified, and the
 * per-sequence arrival counters in meta may be left nonzero.  Call rssm_reset
 * (and re-initialise the checkpoint) before using the handle again. */

enum { RSSM_MAMBA2 = 1, RSSM_GDN = 2, RSSM_KDA = 3 };
enum { RSSM_F32 = 0, RSSM_BF16 = 1 };
enum {
  RSSM_READ_FP32 = 0,        /* reads come from the fp32 checkpoint itself      */
  RSSM_READ_FP8_E4M3_ROW = 1, /* OCP E4M3 codes, one fp32 scale per state row   */
  RSSM_READ_NVFP4 = 2        /* E2M1 codes, one E4M3 scale per 16 row elements  */
};

/*
 * Layer descriptor.  Shapes are fixed for the life of a handle.
 *   Mamba-2: state h [batch, nheads, headdim P, dstate N] fp32; head h reads
 *            input group h / (nheads / ngroups).
 *   GDN:     state S [batch, nheads, headdim (= d_v), dstate (= d_k)] fp32,
 *            mapping keys to values; ngroups is ignored.
 *   KDA:     as GDN, with one gate per key channel (Kimi Delta Attention,
 *            named by [teaser]; read as S <- S Diag(alpha) (I - beta k k^T)
 *            + beta v k^T, o = out_scale S q): replay decode, verify and flush;
 *            with a read copy the reads see the copy and every fold solves
 *            the window again from the fp32 checkpoint (as GDN).
 * A "row" of the state is its last dimension: the contraction vector of one
 * output element (h[b,h,p,:] or S[b,h,i,:]).
 * Supported by this build: Mamba-2 headdim 64 with dstate 64 or 128;
 * GDN and KDA headdim = dstate = 128; 1 <= window <= 32; 0 <= max_draft <= 8 and
 * max_draft <= window.
 */
typedef struct {
  int kind;        /* RSSM_MAMBA2 | RSSM_GDN | RSSM_KDA                       */
  int batch;       /* sequences B                                             */
  int nheads;      /* H                                                       */
  int ngroups;     /* Mamba-2 G (nheads % ngroups == 0); GDN: ignored         */
  int headdim;     /* Mamba-2 P; GDN d_v                                      */
  int dstate;      /* Mamba-2 N; GDN d_k                                      */
  int window;      /* L: committed entries that trigger a flush (default 16) */
  int max_draft;   /* largest k accepted by rssm_verify (0: verify disabled)  */
  int in_dtype;    /* RSSM_F32 | RSSM_BF16 for x/B/C/dt (Mamba-2), q/k/v (GDN) */
  int read_fmt;    /* RSSM_READ_*                                             */
  int auto_flush;  /* nonzero: fold the window when it fills / must make room */
  float out_scale; /* GDN output scale (1.0 = none); ignored for Mamba-2      */
  int branching;   /* nonzero: rows may share checkpoints (rssm_branch)       */
} rssm_layer_desc;

/*
 * Byte offsets of the regions inside the caller's buffers (all 256-aligned).
 * cap = window + max(max_draft, 1) is the ring capacity per sequence.
 *   buf, Mamba-2: x_buf [B,H,cap,P] in_dtype | B_buf [B,G,cap,N] in_dtype |
 *                 dt_buf [B,H,cap] fp32
 *   buf, GDN:     k_buf [B,H,cap,dk] in_dtype | v_buf [B,H,2,cap,dv/2] in_dtype
 *                 (value rows split in two halves, half-major) |
 *                 g_buf [B,H,cap] fp32 (ln alpha) | beta_buf [B,H,cap] fp32 |
 *                 w_buf [B,H,2,cap,dv/2] fp32 (solved w_s, half-major; a cache
 *                 for reads, never used by a fold)
 *   buf, KDA:     k_buf [B,H,cap,dk] in_dtype | v_buf [B,H,cap,dv] in_dtype |
 *                 a_buf [B,H,cap,dk] fp32 (alpha per channel; decays are
 *                 running products of it) |
 *                 beta_buf [B,H,cap] fp32 | w_buf [B,H,2,cap,dv/2] fp32 (solved
 *                 w_s, half-major as for GDN)
 *   read copy, FP8 row: codes [B,H,R,C] uint8 | scales [B,H,R] fp32
 *   read copy, NVFP4:   codes [B,H,R,C/2] uint8 (element 2i in the low
 *                       nibble) | scales [B,H,R,C/16] uint8 (E4M3)
 *     (R, C = headdim, dstate)
 *   meta: int32 start[B] | int32 len[B] | int32 pending[B] | int32 flushes[B]
 *         | int32 arrivals[B] (internal) | uint32 status
 * Ring entry i (0-based, oldest first) of sequence b lives in slot
 * (start[b] + i) % cap.  len = committed entries, pending = unverified
 * drafts after them, flushes = number of folds so far.
 *
 * Branching layers (desc.branching != 0) [guide "The State-Storage
 * Bottleneck in Branching Workloads": beam search, best-of-n and tree search
 * spawn several continuations of one prefix]: several sequences may read one
 * checkpoint.  The checkpoint then holds 2B slots of [H,R,C] fp32 (ckpt
 * [2B,H,R,C]; the read copy likewise 2B slots); sequence b reads slot slot[b]
 * (int32 meta array, slot[b] = b after rssm_reset, so the caller initialises
 * slots 0..B-1 as the sequences' checkpoints).  A fold never writes a slot
 * that any sequence reads: before each replay launch a planner kernel gives
 * every sequence that folds in it a free slot (2B slots, at most B of them
 * read, so one always exists), and the sequence moves to that slot.  meta
 * also holds int32 dst[B], seen[B] and a work area of 5B int32 (internal),
 * and buf a scratch copy of the ring regions (branch_scratch_off).
 */
typedef struct {
  size_t cap;
  size_t buf_off[5];   /* region offsets in buf (unused entries 0)        */
  size_t rc_codes_off, rc_scales_off;
  size_t meta_start_off, meta_len_off, meta_pending_off, meta_flushes_off,
      meta_arrivals_off, meta_status_off;
  /* branching layers only (0 otherwise) */
  size_t meta_slot_off, meta_dst_off, meta_seen_off, meta_work_off;
  size_t branch_scratch_off;   /* in buf: a copy of the ring regions above */
  size_t fold_scratch_off;     /* in buf, KDA with bf16 inputs: the decode
                                  kernel's fold operands (0 if none) */
} rssm_layout;

typedef struct rssm_handle rssm_handle;

/* (No passage: plumbing.)  Sizes (bytes) of the four caller-owned device
 * buffers for a descriptor, and the layout inside them (layout may be NULL).  ckpt = the fp32 checkpoint;
 * read_copy is 0 for RSSM_READ_FP32.  desc.branching doubles the checkpoint
 * and read copy (2B slots) and adds the branch scratch and meta arrays. */
int rssm_workspace_size(const rssm_layer_desc *desc, size_t *ckpt_bytes,
                        size_t *buf_bytes, size_t *read_copy_bytes,
                        size_t *meta_bytes, rssm_layout *layout);

/* The layer storage [summary ¶2: a checkpoint plus a buffer of recent
 * inputs].  Validate the descriptor and bind the caller's device buffers to a
 * new handle (*out).  ckpt_dev holds the caller-initialised fp32 checkpoint.
 * Nothing is enqueued: the meta region must start zeroed (rssm_reset does it)
 * and the read copy must be built with rssm_quantize_read_copy before the
 * first decode when read_fmt != RSSM_READ_FP32. */
int rssm_create(const rssm_layer_desc *desc, void *ckpt_dev, void *buf_dev,
                void *read_copy_dev, void *meta_dev, rssm_handle **out);
/* (No passage: plumbing.)  Free the host handle; the caller's buffers are
 * untouched.  NULL is accepted and does nothing. */
int rssm_destroy(rssm_handle *h);

/* (No passage: plumbing.)  Zero the meta region (empty windows, no drafts,
 * status clear, arrival counters zero); branching layers: every sequence back
 * to slot b.  Enqueued on `stream`. */
int rssm_reset(rssm_handle *h, rssm_stream_t stream);

/* (No passage: plumbing; the parameters of the Mamba-2 recurrence above.)
 * Mamba-2 per-head parameters A[H] (< 0) and D[H], fp32 device arrays kept
 * by pointer (they must outlive the handle).  Required before any Mamba-2
 * compute call; ignored for GDN. */
int rssm_set_params(rssm_handle *h, const float *A_dev, const float *D_dev);

/* (No passage: plumbing.)  Give-up limit, in SM clock cycles, of the replay
 * kernels' bounded waits (for a stage's asynchronous copies, for the other
 * warps to release a stage).  A wait that runs out sets RSSM_STATUS_TIMEOUT
 * and the launch stops early, with the device context intact (see above).
 * 0 restores the default (2e9 cycles, about a second); negative values:
 * RSSM_ERR_INVALID_ARG.  Applies to the calls enqueued after it. */
int rssm_set_wait_limit(rssm_handle *h, long long cycles);

/* (No passage: a self-test of the timeout path.)  The next replay launch of
 * this Mamba-2 or GDN handle (decode, verify, flush) has the consumer warps of
 * its first CTA wait for a shared flag that nothing sets; the wait gives up
 * after the handle's wait limit, sets RSSM_STATUS_TIMEOUT and the CTA ends
 * early, exactly as a copy that never lands would make it.  Nothing faults or
 * hangs; the launch's results are unspecified (call rssm_reset afterwards).
 * Decodes of Mamba-2 read-copy layers with bf16 inputs (headdim 64, dstate
 * 128) run a kernel without waits: such a launch just clears the armed test.
 * KDA: only the decode serving kernel (bf16 inputs) waits, so only a decode of
 * such a handle takes the path (a verify or flush launch just clears the armed
 * test); a KDA handle with fp32 inputs gives RSSM_ERR_UNSUPPORTED. */
int rssm_arm_timeout_test(rssm_handle *h);

/*
 * Decode one token per sequence [summary ¶2-3]: append its inputs to the
 * window and write its output, reading the checkpoint (or its read copy)
 * without writing it.  in[] is a host array of device pointers:
 *   Mamba-2: in[0] x [B,H,P], in[1] B [B,G,N], in[2] C [B,G,N], in[3] dt [B,H]
 *            (in_dtype; dt already softplus'd);
 *   GDN:     in[0] q [B,H,dk], in[1] k [B,H,dk], in[2] v [B,H,dv] (in_dtype),
 *            in[3] alpha [B,H], in[4] beta [B,H] (fp32).
 *   KDA:     as GDN with in[3] alpha [B,H,dk] (fp32, one gate per key channel).
 * out_dev: fp32 y [B,H,P] / o [B,H,dv].
 * With auto_flush: a row whose window is already full is folded first, and a
 * row whose window becomes full (len == L) is folded after its output is
 * computed; a fold rewrites that row's checkpoint and read copy.  Without it
 * a full row sets RSSM_STATUS_CAPACITY and is skipped.  Rows with pending
 * drafts set RSSM_STATUS_STATE and are skipped.
 */
int rssm_decode_step(rssm_handle *h, const void *const *in, void *out_dev,
                     rssm_stream_t stream);

/*
 * Speculative verify [summary ¶3; guide "Example 3: Speculative decoding and
 * rollback"]: append k draft tokens per sequence as pending entries and write
 * all k outputs in one pass over the checkpoint.  Inputs as rssm_decode_step
 * with a draft axis after the batch axis ([B,k,...]); out_dev is [B,k,H,P] /
 * [B,k,H,dv].  Output j is the output after drafts 0..j.  1 <= k <= max_draft.
 * A row with len + k > L is folded first (auto_flush; else CAPACITY, skipped).
 */
int rssm_verify(rssm_handle *h, int k, const void *const *in, void *out_dev,
                rssm_stream_t stream);

/*
 * Accept / roll back [summary ¶3]: n_reject_dev (device int32 [B]) gives, per
 * sequence, how many of its pending drafts to drop (the rest are committed).
 * Only the pointers move: len += pending - n_reject, pending = 0.  A row with
 * n_reject outside [0, pending] sets RSSM_STATUS_STATE and is left as is.
 */
int rssm_rollback(rssm_handle *h, const int32_t *n_reject_dev,
                  rssm_stream_t stream);

/*
 * Flush [summary ¶3]: fold the committed window of every selected sequence
 * into its fp32 checkpoint (and refresh its read copy), then empty the window.
 * row_mask_dev: device int32 [B], nonzero = flush that row; NULL = all rows.
 * Rows with pending drafts set RSSM_STATUS_STATE and are skipped.
 */
int rssm_flush(rssm_handle *h, const int32_t *row_mask_dev,
               rssm_stream_t stream);

/*
 * Rebuild the whole low-precision read copy from the fp32 checkpoint
 * [summary ¶4] (all 2B slots of a branching layer).  Call after creating
 * the handle or writing the checkpoint.
 * RSSM_ERR_STATE if the handle has no read copy.
 */
int rssm_quantize_read_copy(rssm_handle *h, rssm_stream_t stream);

/*
 * The conventional per-token update, used as the in-run baseline [summary
 * ¶3: "rewriting the full state every token"]: reads the fp32 state
 * state_in_dev [B,H,P,N] (GDN [B,H,dv,dk]), applies one token (inputs as
 * rssm_decode_step), writes the new state to state_out_dev (may equal
 * state_in_dev for an in-place update) and the output to out_dev.  Uses only
 * the handle's shape and parameters; its window and checkpoint are untouched.
 */
int rssm_conventional_step(rssm_handle *h, const float *state_in_dev,
                           float *state_out_dev, const void *const *in,
                           void *out_dev, rssm_stream_t stream);

/*
 * The conventional per-token update with the state itself kept in low
 * precision -- the design a read copy replaces [summary ¶4: rounding a stored
 * state again at every token compounds the error, while a read copy beside an
 * fp32 recurrence does not].  A baseline for that comparison.
 *
 * The state is stored in the handle's read_fmt (RSSM_READ_FP8_E4M3_ROW or
 * RSSM_READ_NVFP4), in the read-copy layout above: codes_in_dev/scales_in_dev
 * hold it before the token, codes_out_dev/scales_out_dev receive it after (the
 * same buffers may be passed for an in-place update).  Per token: decode the
 * codes, apply the conventional update in fp32 (inputs as rssm_decode_step),
 * write the output from the updated fp32 values, then quantise the updated
 * state exactly as rssm_quantize_read_copy does and store it.  Uses only the
 * handle's shape, formats and parameters; its checkpoint, read copy and
 * window are untouched.
 * Errors: RSSM_ERR_STATE if read_fmt is RSSM_READ_FP32; RSSM_ERR_INVALID_ARG
 * for NULL or misaligned pointers (codes 16-byte, FP8 scales 4-byte aligned);
 * RSSM_ERR_UNSUPPORTED for KDA layers (Mamba-2 and GDN only).
 */
int rssm_conventional_step_quantized(rssm_handle *h, const void *codes_in_dev,
                                     const void *scales_in_dev,
                                     void *codes_out_dev, void *scales_out_dev,
                                     const void *const *in, void *out_dev,
                                     rssm_stream_t stream);

/*
 * rssm_decode_step without any caller-provided scratch.  (This entry point has
 * no counterpart on the pages; it serves integration needs only.)
 *
 * Identical inputs, outputs and results to rssm_decode_step.  The replay
 * kernel's only scratch -- one int32 arrival counter per sequence -- comes
 * from a fixed array inside the library (RSSM_STATIC_SCRATCH_MAX_BATCH
 * entries, 256 KiB on every GPU that loads the library, kept until the
 * process exits) instead of the caller's meta buffer, so the call performs
 * no allocation: for callers that record decode steps into a CUDA graph,
 * engines that reserve all device memory at start-up, and loops that cannot
 * afford cudaMalloc's implicit synchronisation.
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress); make that first call before any stream capture.
 *     The address is cached per device index for the life of the process,
 *     which assumes one CUDA context per device (no cudaDeviceReset between
 *     calls).
 *   - Each call clears the counters it uses (cudaMemsetAsync on `stream`).
 *   - All calls share the one array: calls that may run concurrently on the
 *     GPU (different streams, different handles) race and must not overlap.
 *   - batch > RSSM_STATIC_SCRATCH_MAX_BATCH: RSSM_ERR_INVALID_ARG.
 */
#define RSSM_STATIC_SCRATCH_MAX_BATCH 65536
int rssm_decode_step_static_scratch(rssm_handle *h, const void *const *in,
                                    void *out_dev, rssm_stream_t stream);

/*
 * Branch / fork [guide "The State-Storage Bottleneck in Branching
 * Workloads"]: every sequence b continues from the state sequence
 * parent_dev[b] had before the call (device int32 [B]; parent[b] == b keeps
 * b).  All sequences move at once, as a gather.  The child shares the
 * parent's checkpoint slot (no state is copied) and takes a copy of its
 * window (ring entries and pointers: start, len, flushes; pending is 0); its
 * own next fold writes a slot of its own.  A sequence whose parent is out of
 * range or has pending drafts sets RSSM_STATUS_STATE and keeps its own state.
 * Two kernel launches: the parents' pointers and live window entries are
 * gathered (into the scratch), then scattered into the children, so a
 * sequence that is both parent and child is read before it is overwritten.
 * RSSM_ERR_STATE if the handle was created with branching = 0.
 */
int rssm_branch(rssm_handle *h, const int32_t *parent_dev, rssm_stream_t stream);

/*
 * Restore to a position [guide "What a Replay-First Design Implies": the
 * decode loop can return a sequence to an earlier position]: sequence b returns to its
 * state after the first keep_dev[b] committed tokens of its current window
 * (the tokens since its last fold): len = keep.  Only the pointer moves.
 * keep outside [0, len] or pending drafts: RSSM_STATUS_STATE, row unchanged.
 * Any layer (branching or not).
 */
int rssm_restore(rssm_handle *h, const int32_t *keep_dev, rssm_stream_t stream);

/* [guide "The State-Storage Bottleneck in Branching Workloads"]  The
 * checkpoint slot each sequence reads, after the folds of the calls enqueued
 * so far (device int32 [B]); its checkpoint is ckpt slot out[b].
 * RSSM_ERR_STATE if the handle was created with branching = 0. */
int rssm_get_slots(rssm_handle *h, int32_t *out_dev, rssm_stream_t stream);

/*
 * (No passage: plumbing for serving.)  State export / import to host
 * (serving-side preemption, migration between processes or GPUs).  The blob is the layer's whole replay state in one host
 * buffer: checkpoint (every slot) | read copy | ring buffers | meta (pointers,
 * slots, status), in that order, raw bytes; rssm_state_bytes gives its size.
 * Import requires a handle created from the same descriptor.  Both are plain
 * cudaMemcpyAsync calls on `stream` (pinned host memory makes them
 * asynchronous; the caller synchronises before reading or reusing the blob).
 * No kernel runs and nothing is converted: export then import is bit-exact.
 * Errors: RSSM_ERR_INVALID_ARG for NULL pointers or a size that differs from
 * rssm_state_bytes.
 */
int rssm_state_bytes(rssm_handle *h, size_t *bytes);
int rssm_export_state(rssm_handle *h, void *host_dst, size_t bytes, rssm_stream_t stream);
int rssm_import_state(rssm_handle *h, const void *host_src, size_t bytes, rssm_stream_t stream);

/* The window pointers [summary ¶3: drafts are appended and dropped by moving
 * a pointer].  Copy the committed lengths into len_dev and the pending draft
 * counts into pending_dev (device int32 [B] each), enqueued on `stream`
 * (plain device-to-device copies).  NULL pointers: RSSM_ERR_INVALID_ARG. */
int rssm_get_lengths(rssm_handle *h, int32_t *len_dev, int32_t *pending_dev,
                     rssm_stream_t stream);

/* All per-sequence pointers [summary ¶3]: copy them into out_dev (device
 * int32 [4, B]: start, len, pending, flushes), one kernel launch. */
int rssm_get_bookkeeping(rssm_handle *h, int32_t *out_dev,
                         rssm_stream_t stream);

/* (No passage: plumbing.)  Synchronise `stream` and return the sticky device
 * status bits in *bits (host pointer).  clear != 0 resets them afterwards. */
int rssm_get_status(rssm_handle *h, uint32_t *bits, int clear,
                    rssm_stream_t stream);

/* (No passage: plumbing.)  Thread-local text describing the last error on
 * this thread ("" if none). */
const char *rssm_last_error_string(void);

/* (No passage: plumbing.)  Number of GPU kernels this library has launched
 * in this process.  Kernel launches only: the memsets and copies some calls
 * enqueue (rssm_reset, rssm_get_status, the static-scratch clear, state
 * export/import, rssm_get_lengths) are not counted. */
uint64_t rssm_launch_count(void);

#ifdef __cplusplus
}
#endif
#endif /* RSSM_H */
