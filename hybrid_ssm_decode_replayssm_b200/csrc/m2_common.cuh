// Device pieces shared by the Mamba-2 replay kernels (mamba2.cu, m2_rc_decode.cu):
// the register tile mapping, the stage view of a head's window rows, the
// rank-l fold of a tile, the outputs from a read view, and the f16 tensor-core
// read of a quantised copy.
#pragma once

#include "rssm_device.cuh"

namespace rssm {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

// Tile mapping: W warps cover the P rows of a [P, N] fp32 tile; a lane holds 4
// consecutive columns of a row (float4), LPR lanes cover one row, a warp
// instruction covers RPI rows.
template <int P, int N, int W = kWarps>
struct Tile {
  static constexpr int LPR = N / 4;     // lanes per state row
  static constexpr int RPI = 32 / LPR;  // rows covered by one warp instruction
  static constexpr int RPW = P / W;     // rows per warp
  static constexpr int NLD = RPW / RPI; // float4 per lane
  static_assert(N == 64 || N == 128, "dstate 64 or 128");
  static_assert(RPW % RPI == 0, "headdim must cover whole warp instructions");
};

template <int RF, int P, int N>
constexpr int tile_bytes() {
  return RF == RSSM_READ_FP32 ? P * N * 4 : RF == RSSM_READ_FP8_E4M3_ROW ? P * N : P * N / 2;
}
template <int RF, int P, int N>
constexpr int scale_bytes() {
  return RF == RSSM_READ_FP32 ? 0 : RF == RSSM_READ_FP8_E4M3_ROW ? P * 4 : P * (N / 16);
}
template <int RF, int N>
constexpr int rc_row_bytes() { return RF == RSSM_READ_NVFP4 ? N / 2 : N; }

// Stage layout for one head: [read tile | scales | committed x rows (L) | new x rows (MAXM)].
struct Stage {
  uint8_t *base;
  int xoff, xrow, n, L;
  template <typename Tin>
  __device__ __forceinline__ const Tin *row(int i) const {  // x row of window entry i
    const int r = i < n ? i : L + (i - n);
    return reinterpret_cast<const Tin *>(base + xoff + (size_t)r * xrow);
  }
  template <typename Tin>
  __device__ __forceinline__ float x(int i, int p) const { return to_f32<Tin>(row<Tin>(i)[p]); }
  // x_i at rows p0, p0 + step, ..., K values (one vector load when step == 1).
  template <typename Tin, int K>
  __device__ __forceinline__ void xs(int i, int p0, int step, float (&o)[K]) const {
    const Tin *r = row<Tin>(i) + p0;
    if (step == 1 && (K * sizeof(Tin)) % 16 == 0) {
#pragma unroll
      for (int c = 0; c < (int)(K * sizeof(Tin) / 16); ++c) {
        const uint4 raw = *reinterpret_cast<const uint4 *>(r + c * (16 / sizeof(Tin)));
        const Tin *e = reinterpret_cast<const Tin *>(&raw);
#pragma unroll
        for (int q = 0; q < (int)(16 / sizeof(Tin)); ++q) o[c * (16 / sizeof(Tin)) + q] = to_f32<Tin>(e[q]);
      }
    } else {
#pragma unroll
      for (int q = 0; q < K; ++q) o[q] = to_f32<Tin>(r[q * step]);
    }
  }
};

// t <- dec * t + sum_{i0 <= i < i1} x_i[row] (fw[i - i0] B_i[cols])   (rank-(i1-i0) fold)
template <int P, int N, int W, typename Tin>
__device__ __forceinline__ void fold_tile(float4 (&t)[Tile<P, N, W>::NLD], const float *s_fw, float dec,
                                          int i0, int i1, const Stage &stg, const float *s_B,
                                          int row0, int c0) {
  using T = Tile<P, N, W>;
#pragma unroll
  for (int l = 0; l < T::NLD; ++l) {
    t[l].x *= dec; t[l].y *= dec; t[l].z *= dec; t[l].w *= dec;
  }
  for (int i = i0; i < i1; ++i) {
    const float fw = s_fw[i - i0];
    float4 bv = *reinterpret_cast<const float4 *>(s_B + i * N + c0);
    bv.x *= fw; bv.y *= fw; bv.z *= fw; bv.w *= fw;
    float xr[T::NLD];
    stg.xs<Tin, T::NLD>(i, row0, T::RPI, xr);   // this lane's rows: one vector load when contiguous
#pragma unroll
    for (int l = 0; l < T::NLD; ++l) {
      t[l].x = fmaf(xr[l], bv.x, t[l].x);
      t[l].y = fmaf(xr[l], bv.y, t[l].y);
      t[l].z = fmaf(xr[l], bv.z, t[l].z);
      t[l].w = fmaf(xr[l], bv.w, t[l].w);
    }
  }
}

// Outputs of the m new tokens from the read view v (registers).  Lane l of a
// row's lane group adds the window terms of entries i = w0 + l (+ LPR, ...)
// to its partial sums, so that one transposed reduction over the row's lanes
// yields  dec_j (v . C_j) + sum_i coef_ji x_i[row]  for every row and output;
// the lanes left holding copies of a sum let one of them add D x_e and store.
template <int P, int N, int W, typename Tin, int MAXM>
__device__ __forceinline__ void outputs(const float4 (&v)[Tile<P, N, W>::NLD], const StepArgs &a,
                                        const float *s_C, const float *hcoef, const float *hdec,
                                        const Stage &stg, int b, int h, int n, int w0, int row0,
                                        int lane, int c0) {
  using T = Tile<P, N, W>;
  constexpr int NV = T::NLD * MAXM;
  constexpr int DUP = NV >= T::LPR ? 1 : T::LPR / NV;
  float part[NV];
#pragma unroll
  for (int j = 0; j < MAXM; ++j) {
    const float4 cv = *reinterpret_cast<const float4 *>(s_C + j * N + c0);
    const float dj = hdec[j];
#pragma unroll
    for (int l = 0; l < T::NLD; ++l)
      part[l * MAXM + j] = dj * (v[l].x * cv.x + v[l].y * cv.y + v[l].z * cv.z + v[l].w * cv.w);
  }
  const int emax = n + a.m - 1;   // last entry of the output window
  for (int i = w0 + lane % T::LPR; i <= emax; i += T::LPR) {
    float xr[T::NLD];
    stg.xs<Tin, T::NLD>(i, row0, T::RPI, xr);
#pragma unroll
    for (int j = 0; j < MAXM; ++j) {
      const float cj = hcoef[j * 32 + (i - w0)];   // 0 for entries after e_j
#pragma unroll
      for (int l = 0; l < T::NLD; ++l) part[l * MAXM + j] = fmaf(cj, xr[l], part[l * MAXM + j]);
    }
  }
  tr_sum<NV, T::LPR / 2>(part, lane);
  const int base = tr_base<NV, T::LPR / 2>(lane);
  constexpr int R = NV >= T::LPR ? NV / T::LPR : 1;
  const bool writer = (lane & (DUP - 1)) == 0;
  const float Dh = __ldg(a.D + h);
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const int idx = base + r, l = idx / MAXM, j = idx % MAXM;
    const int row = row0 + l * T::RPI;   // lanes keep their row group through the reduction
    if (writer && j < a.m) {
      const int e = n + j;
      a.out[(((size_t)b * a.m + j) * a.H + h) * P + row] = fmaf(Dh, stg.x<Tin>(e, row), part[r]);
    }
  }
}

__device__ __forceinline__ void mma_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t h2bits(__half2 v) { return *reinterpret_cast<uint32_t *>(&v); }
// two E2M1 codes (one byte, element 0 in the low nibble) -> f16x2, times a f16x2 scale
__device__ __forceinline__ uint32_t e2m1x2_scaled(uint32_t byte, __half2 sc) {
  const __half2_raw r = __nv_cvt_fp4x2_to_halfraw2((__nv_fp4x2_storage_t)(byte & 0xFFu), __NV_E2M1);
  return h2bits(__hmul2(__half2(r), sc));
}
// two E4M3 codes (16 bits, element 0 in the low byte) -> f16x2
__device__ __forceinline__ uint32_t e4m3x2_h2(uint32_t bits) {
  const __half2_raw r = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(bits & 0xFFFFu), __NV_E4M3);
  return h2bits(__half2(r));
}

}  // namespace
}  // namespace rssm
