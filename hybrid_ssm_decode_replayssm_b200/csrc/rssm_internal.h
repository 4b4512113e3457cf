// Internal interface between the C-ABI host code and the kernel launchers.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/rssm.h"

namespace rssm {

enum StepMode { kDecode = 0, kVerify = 1, kFlush = 2 };

constexpr int kMaxWindow = 32;
constexpr int kMaxDraft = 8;

// Everything a replay kernel needs about one call.  Pointers are device
// pointers into the caller's buffers.
struct StepArgs {
  // shape
  int B, H, G, hpg;      // hpg = heads per group (Mamba-2)
  int R, C;              // state rows / columns (P, N  or  dv, dk)
  int L, cap;            // window and ring capacity
  int m;                 // tokens appended by this call (1 decode, k verify, 0 flush)
  int mode;              // StepMode
  int auto_flush;
  float out_scale;       // GDN
  // parameters (Mamba-2)
  const float *A, *D;
  // checkpoint and read copy (with branching: 2B slots; row b reads slot[b]
  // and a fold of row b writes slot dst[b]; without: both NULL, slot b = row b)
  float *hc;
  const int32_t *slot, *dst;
  uint8_t *rc_codes;
  void *rc_scales;
  // ring buffers (layer specific, see rssm.h)
  void *buf0, *buf1;     // Mamba-2: x_buf, B_buf     GDN: k_buf, v_buf
  float *buf2, *buf3, *buf4;  // Mamba-2: dt_buf     GDN: g_buf, beta_buf, w_buf
  uint8_t *fold_scratch;      // KDA decode serving path: per-CTA fold operands (nullable)
  // per-call inputs / outputs
  const void *in[5];
  float *out;
  const int32_t *mask;   // flush row mask (nullable)
  // bookkeeping
  int32_t *start, *len, *pending, *flushes, *arrivals;
  uint32_t *status;
  // give-up limit (SM clock cycles) of the bounded waits on copies and on the
  // other warps; waits for the tensor cores and the final drain keep their own
  long long wait_limit;
  // nonzero: the consumer warps of CTA 0 first wait for a flag that nothing
  // sets, so that the wait runs out (rssm_arm_timeout_test)
  int stall_test;
};

constexpr long long kDefaultWaitLimit = 2000000000LL;   // about a second at B200 clocks

struct ConvArgs {
  int B, H, G, hpg, R, C;
  float out_scale;
  const float *A, *D;
  const float *state_in;       // fp32 state (state format RSSM_READ_FP32)
  float *state_out;
  const uint8_t *codes_in;     // low-precision state (FP8 row / NVFP4), read-copy layout
  const void *scales_in;
  uint8_t *codes_out;
  void *scales_out;
  const void *in[5];
  float *out;
};

struct QuantArgs {
  size_t rows;           // B*H*R
  int C;
  const float *hc;
  uint8_t *codes;
  void *scales;
};

// Launchers return cudaGetLastError() of their launch.
cudaError_t mamba2_step(const StepArgs &a, int in_dtype, int read_fmt, cudaStream_t s);
// Decode of read-copy layers (one token, bf16 inputs, headdim 64, dstate 128):
// its own kernel without a stage pipeline (m2_rc_decode.cu).
bool m2_rc_decode_path(const StepArgs &a, int in_dtype, int read_fmt);
cudaError_t m2_rc_decode_step(const StepArgs &a, int read_fmt, cudaStream_t s);
// state_fmt: RSSM_READ_FP32 (fp32 state), or the FP8 row / NVFP4 format of a
// state stored in low precision and rounded again after every token
cudaError_t mamba2_conventional(const ConvArgs &a, int in_dtype, int state_fmt, cudaStream_t s);
cudaError_t gdn_step(const StepArgs &a, int in_dtype, int read_fmt, cudaStream_t s);
// The GDN decode serving path (one token, bf16 inputs, fp32 reads): its own
// kernel with prologue warps and tensor-core folds (dr_decode.cu).
bool gdn_decode_fast_path(const StepArgs &a, int in_dtype, int read_fmt);
cudaError_t gdn_decode_step(const StepArgs &a, cudaStream_t s);
cudaError_t gdn_conventional(const ConvArgs &a, int in_dtype, int state_fmt, cudaStream_t s);
cudaError_t quantize_read_copy(const QuantArgs &a, int read_fmt, cudaStream_t s);
cudaError_t rollback(int B, const int32_t *n_reject, int32_t *len, int32_t *pending,
                     uint32_t *status, cudaStream_t s);
cudaError_t gather_bookkeeping(int B, const int32_t *start, const int32_t *len,
                               const int32_t *pending, const int32_t *flushes, int32_t *out,
                               cudaStream_t s);

// Branching (rows sharing checkpoint slots).  BranchArgs describes the meta
// arrays and the ring regions copied when a row takes another row's window.
struct BranchArgs {
  int B;
  int32_t *slot, *dst, *seen, *freelist, *eff;   // [B] [B] [B] [2B] [B]
  int32_t *start, *len, *pending, *flushes;
  uint32_t *status;
  int nreg;                   // ring regions in buf
  int cap;                    // ring capacity (entries)
  uint8_t *ring[5];           // region bases
  uint8_t *scratch[5];        // their copies in the branch scratch
  // A region is [B][outer][cap][entry bytes]: one sequence's row holds `outer`
  // rings (heads, groups or head halves) of cap entries each.
  int outer[5];
  int entry_bytes[5];
};
// Before a replay launch: adopt the slots written by the previous launch's
// folds, then give every row that folds in this launch a free slot.
cudaError_t plan_slots(const StepArgs &a, int32_t *slot, int32_t *dst, int32_t *seen, int32_t *freelist,
                       cudaStream_t s);
// rssm_branch: bookkeeping gather, then the window copy through the scratch.
// tmp: int32 [4B] scratch.
cudaError_t branch_rows(const BranchArgs &b, const int32_t *parent, int32_t *tmp, cudaStream_t s);
cudaError_t restore_rows(int B, const int32_t *keep, int32_t *len, const int32_t *pending,
                         uint32_t *status, cudaStream_t s);
cudaError_t init_slots(int B, int32_t *slot, int32_t *dst, cudaStream_t s);
cudaError_t effective_slots(int B, const int32_t *slot, const int32_t *dst, const int32_t *seen,
                            const int32_t *flushes, int32_t *out, cudaStream_t s);

bool mamba2_supported(int R, int C);
bool gdn_supported(int R, int C);

}  // namespace rssm
