// prep_row.cuh — the per-row arithmetic of "Exact Numerical Contract",
// "Preparation" steps 1-3, shared by the stand-alone prep kernel (prep.cu) and
// the fused prep + quantization kernels (prep_quant.cu), so both produce the same
// bits.  A head row of D dims is held by L = D/8 consecutive lanes of a warp,
// lane l holding dims 8l .. 8l+7 as one 16-byte chunk; 32/L rows share a warp
// (row `sub` = lane / L).  Every lane of the warp must call these together (they
// shuffle).
#pragma once

#include <cuda_bf16.h>

#include "qattn_device.cuh"

namespace qattn {
namespace prep {

// FP64 -> BF16 with one rounding: round |x| to the BF16 quantum of its binade
// (2^(e-7), e = floor(log2|x|), or 2^-133 below the normal range), ties to even.
__device__ __forceinline__ float bf16_round_f64(double x) {
  if (x == 0.0) return static_cast<float>(x);
  const double a = fabs(x);
  int e = ilogb(a);
  if (e < -126) e = -126;
  const double quantum = ldexp(1.0, e - 7);
  const double r = rint(a / quantum) * quantum;  // exact scaling by a power of two
  return static_cast<float>(copysign(r, x));     // <= 8 significant bits: exact
}

// The RoPE coefficients of position `pos` and pair i < R/2: cos and sin of
// pos * theta^(-2i/R), in FP64, each rounded once to BF16 (returned as FP32).
__device__ __forceinline__ double rope_freq(double theta, int i, int rotary_dim) {
  return pow(theta, -(2.0 * i) / static_cast<double>(rotary_dim));
}
__device__ __forceinline__ void rope_coef(int64_t pos, double freq, float* c, float* s) {
  const double ang = static_cast<double>(pos) * freq;
  double sv, cv;
  sincos(ang, &sv, &cv);
  *c = bf16_round_f64(cv);
  *s = bf16_round_f64(sv);
}

__device__ __forceinline__ float bf16_lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t u) { return __uint_as_float(u & 0xFFFF0000u); }
// Two FP32 values -> one BF16 pair (x in the low half), each rounded to nearest even.
__device__ __forceinline__ uint32_t bf16x2_rn(float2 v) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(v.x, v.y);
  return *reinterpret_cast<const uint32_t*>(&h);
}
__device__ __forceinline__ float2 unpack_bf16x2(uint32_t u) {
  return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xFFFF0000u));
}

// Sum of squares of the row (L lanes of 8 consecutive dims, left to right, then
// the XOR butterfly over the lanes): every lane of the row gets the same value.
template <int D>
__device__ __forceinline__ float sumsq8(const uint4 raw) {
  constexpr int L = D / 8;
  float x[8];
  x[0] = bf16_lo(raw.x); x[1] = bf16_hi(raw.x);
  x[2] = bf16_lo(raw.y); x[3] = bf16_hi(raw.y);
  x[4] = bf16_lo(raw.z); x[5] = bf16_hi(raw.z);
  x[6] = bf16_lo(raw.w); x[7] = bf16_hi(raw.w);
  float ss = __fmul_rn(x[0], x[0]);
#pragma unroll
  for (int e = 1; e < 8; ++e) ss = __fadd_rn(ss, __fmul_rn(x[e], x[e]));
#pragma unroll
  for (int off = L / 2; off >= 1; off >>= 1) ss = __fadd_rn(ss, __shfl_xor_sync(0xffffffffu, ss, off));
  return ss;
}

// r = 1/sqrt(ss/D + eps), IEEE square root and division.
template <int D>
__device__ __forceinline__ float rms_r(float ss, float eps) {
  return __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(__fmul_rn(ss, 1.0f / D), eps)));
}

// y = bf16(bf16(x * r) * w) for the lane's 8 values.
__device__ __forceinline__ void apply_norm8(const uint4 raw, const uint16_t* w, float r, int l,
                                            uint32_t (&yb)[4]) {
  const uint4 wr = *reinterpret_cast<const uint4*>(w + 8 * l);
  const uint32_t xv[4] = {raw.x, raw.y, raw.z, raw.w};
  const uint32_t wv[4] = {wr.x, wr.y, wr.z, wr.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t xr = bf16x2_rn(fmul2(unpack_bf16x2(xv[j]), make_float2(r, r)));
    yb[j] = bf16x2_rn(fmul2(unpack_bf16x2(xr), unpack_bf16x2(wv[j])));
  }
}

// The r of N chunks' rows at once.  A warp holds 32/L rows per chunk; lane i <
// N * (32/L) takes the sum of row (chunk i / (32/L), row i % (32/L)), computes its
// r, and the values go back to the rows' lanes: one square root and division for
// the warp's N * 32/L rows instead of one per chunk (the same bits).
template <int D, int N>
__device__ __forceinline__ void batch_rms_r(const float (&ss)[N], float eps, float (&r)[N]) {
  constexpr int L = D / 8, HPW = 32 / L;
  static_assert(N * HPW <= 32, "one lane per row");
  const int lane = threadIdx.x & 31;
  float mine = 0.0f;
#pragma unroll
  for (int c = 0; c < N; ++c) {
    const float t = __shfl_sync(0xffffffffu, ss[c], (lane % HPW) * L);
    if (lane / HPW == c) mine = t;
  }
  const float rm = rms_r<D>(mine, eps);
  const int sub = lane / L;
#pragma unroll
  for (int c = 0; c < N; ++c) r[c] = __shfl_sync(0xffffffffu, rm, c * HPW + sub);
}

// Step 1-2, RMSNorm: r = 1/sqrt(sum(x^2)/D + eps) with the sum taken as L lanes of
// 8 consecutive dims (left to right) then an XOR butterfly over the lanes;
// y = bf16(bf16(x * r) * w).  w == nullptr: no norm, y = x.  yb: the lane's 8
// values as 4 BF16 pairs.
template <int D>
__device__ __forceinline__ void rmsnorm8(const uint4 raw, const uint16_t* w, float eps, int l,
                                         uint32_t (&yb)[4]) {
  constexpr int L = D / 8;
  float x[8];
  x[0] = bf16_lo(raw.x); x[1] = bf16_hi(raw.x);
  x[2] = bf16_lo(raw.y); x[3] = bf16_hi(raw.y);
  x[4] = bf16_lo(raw.z); x[5] = bf16_hi(raw.z);
  x[6] = bf16_lo(raw.w); x[7] = bf16_hi(raw.w);
  float ss = __fmul_rn(x[0], x[0]);
#pragma unroll
  for (int e = 1; e < 8; ++e) ss = __fadd_rn(ss, __fmul_rn(x[e], x[e]));
#pragma unroll
  for (int off = L / 2; off >= 1; off >>= 1) ss = __fadd_rn(ss, __shfl_xor_sync(0xffffffffu, ss, off));
  // Packed FP32 pairs and BF16 pairs from here on: every element still sees
  // exactly the same roundings (RN products, RN sums, BF16 RN) as the scalar form.
  if (w != nullptr) {
    const float ms = __fmul_rn(ss, 1.0f / D);
    const float r = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(ms, eps)));
    const uint4 wr = *reinterpret_cast<const uint4*>(w + 8 * l);
    const uint32_t wv[4] = {wr.x, wr.y, wr.z, wr.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t xr = bf16x2_rn(fmul2(make_float2(x[2 * j], x[2 * j + 1]), make_float2(r, r)));
      yb[j] = bf16x2_rn(fmul2(unpack_bf16x2(xr), unpack_bf16x2(wv[j])));
    }
  } else {
    yb[0] = raw.x; yb[1] = raw.y; yb[2] = raw.z; yb[3] = raw.w;
  }
}

// Step 3, split-half RoPE on dims [0, R): lane l < R/16 pairs with lane l + R/16.
// Both halves as y*cos + o*sv with sv = -sin (first half) or +sin (second half),
// which is bit for bit y*cos - o*sin or y*cos + o*sin; other lanes pass through.
// cv / sn: cos and sin of the lane's 8 pairs (pair index 8l + e for l < R/16,
// 8l - R/2 + e for R/16 <= l < R/8); read only on rotating lanes.
__device__ __forceinline__ void rope8(uint32_t (&yb)[4], int sub, int l, int L, int half_lanes,
                                      int rot_lanes, const float (&cv)[8], const float (&sn)[8]) {
  const int pl = (l < half_lanes) ? l + half_lanes : (l < rot_lanes ? l - half_lanes : l);
  const int src_lane = sub * L + pl;
  uint32_t ob[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) ob[j] = __shfl_sync(0xffffffffu, yb[j], src_lane);
  if (l < rot_lanes) {
    const float sg = l < half_lanes ? -1.0f : 1.0f;       // exact sign flip
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 yc = fmul2(unpack_bf16x2(yb[j]), make_float2(cv[2 * j], cv[2 * j + 1]));
      const float2 os = fmul2(unpack_bf16x2(ob[j]), make_float2(sg * sn[2 * j], sg * sn[2 * j + 1]));
      yb[j] = bf16x2_rn(fadd2(yc, os));
    }
  }
}

}  // namespace prep
}  // namespace qattn
