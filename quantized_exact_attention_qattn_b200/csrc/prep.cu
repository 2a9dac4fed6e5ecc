// prep.cu — per-head Q/K RMSNorm + split-half RoPE, one CTA per (batch, token).
//
// "Exact Numerical Contract", section "Preparation", steps 1-3: normalize in
// FP32, round to BF16 RN, rotate dims [0, R) in split-half pairs (i, i+R/2)
// with BF16 coefficients and FP32 arithmetic, round to BF16 RN.  The sum of
// squares uses D/8 lanes of 8 consecutive dims and an XOR butterfly, which is
// exactly how a half-warp holding one 128-dim row in 16-byte chunks reduces it.
//
// HBM-bound: every (token, head) row is read once with 16-byte loads and
// written once with 16-byte stores; the RoPE coefficients of the token are
// computed once per CTA (FP64) into shared memory and reused by all heads,
// while the token's row loads are already in flight.
#include <cuda_bf16.h>

#include "qattn_device.cuh"
#include "qattn_internal.h"

#ifndef QATTN_PREP_TOKENS
#define QATTN_PREP_TOKENS 8
#endif
#ifndef QATTN_PREP_PASSES
#define QATTN_PREP_PASSES 2
#endif

namespace qattn {
namespace {

struct PrepArgs {
  BNHD q, k;
  const uint16_t* qw;
  const uint16_t* kw;
  uint16_t* q_out;
  uint16_t* k_out;
  int B, N, Hq, Hkv, rotary_dim;
  float eps;
  double theta;
  int64_t pos_offset;
};

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

template <int D>
__global__ void __launch_bounds__(256) prep_kernel(const PrepArgs a) {
  constexpr int L = D / 8;     // lanes holding one head row
  constexpr int HPW = 32 / L;  // head rows per warp
  __shared__ __align__(16) float s_cos[QATTN_PREP_TOKENS][D / 2];
  __shared__ __align__(16) float s_sin[QATTN_PREP_TOKENS][D / 2];
  __shared__ double s_freq[D / 2];   // theta^(-2i/R), the same for every token

  const int tiles = (a.N + QATTN_PREP_TOKENS - 1) / QATTN_PREP_TOKENS;
  const int b = blockIdx.x / tiles;
  const int n0 = (blockIdx.x - b * tiles) * QATTN_PREP_TOKENS;
  const int nt = min(QATTN_PREP_TOKENS, a.N - n0);    // tokens of this CTA
  const int half = a.rotary_dim / 2;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int sub = lane / L;        // which head row of this warp
  const int l = lane - sub * L;    // lane within the head row
  const int slots = (blockDim.x >> 5) * HPW;
  const int total = a.Hq + a.Hkv;
  const int rot_lanes = a.rotary_dim / 8;
  const int half_lanes = half / 8;

  auto row_src = [&](int n, int hh) {
    const bool isq = hh < a.Hq;
    const BNHD src = isq ? a.q : a.k;
    const int h = isq ? hh : hh - a.Hq;
    return src.ptr + b * src.sb + static_cast<int64_t>(n) * src.sn +
           static_cast<int64_t>(h) * src.sh + 8 * l;
  };
  constexpr int MAXP = QATTN_PREP_PASSES;   // head-row passes whose loads are issued together
  uint4 raw[MAXP];
  auto load_passes = [&](int n, int base0) {
#pragma unroll
    for (int pidx = 0; pidx < MAXP; ++pidx) {
      const int hh = base0 + pidx * slots + warp * HPW + sub;
      raw[pidx] = make_uint4(0, 0, 0, 0);
      if (hh < total) raw[pidx] = *reinterpret_cast<const uint4*>(row_src(n, hh));
    }
  };

  // The first loads go out before the FP64 RoPE tables of all the CTA's tokens
  // are computed (by all threads at once), so the table latency overlaps them.
  load_passes(n0, 0);
  for (int i = threadIdx.x; i < half; i += blockDim.x)
    s_freq[i] = pow(a.theta, -(2.0 * i) / static_cast<double>(a.rotary_dim));
  __syncthreads();
  for (int idx = threadIdx.x; idx < nt * half; idx += blockDim.x) {
    const int k = idx / half, i = idx - k * half;
    const double ang = static_cast<double>(a.pos_offset + n0 + k) * s_freq[i];
    double sv, cv;
    sincos(ang, &sv, &cv);
    s_cos[k][i] = bf16_round_f64(cv);
    s_sin[k][i] = bf16_round_f64(sv);
  }
  __syncthreads();

  for (int k = 0; k < nt; ++k) {
    const int n = n0 + k;
    for (int base0 = 0; base0 < total; base0 += MAXP * slots) {
      if (k > 0 || base0 > 0) load_passes(n, base0);
#pragma unroll
      for (int pidx = 0; pidx < MAXP; ++pidx) {
        const int base = base0 + pidx * slots;
        if (base >= total) break;                   // uniform over the CTA
        const int hh = base + warp * HPW + sub;
        const bool valid = hh < total;
        const bool isq = hh < a.Hq;
        const int h = isq ? hh : hh - a.Hq;
        const uint16_t* w = isq ? a.qw : a.kw;
        float x[8];
        x[0] = bf16_lo(raw[pidx].x); x[1] = bf16_hi(raw[pidx].x);
        x[2] = bf16_lo(raw[pidx].y); x[3] = bf16_hi(raw[pidx].y);
        x[4] = bf16_lo(raw[pidx].z); x[5] = bf16_hi(raw[pidx].z);
        x[6] = bf16_lo(raw[pidx].w); x[7] = bf16_hi(raw[pidx].w);

        // ---- RMSNorm (skipped when this tensor has no weight; uniform per warp
        //      only when Hq and Hkv rows do not share a warp, so every lane takes
        //      part in the shuffles regardless)
        float ss = __fmul_rn(x[0], x[0]);
#pragma unroll
        for (int e = 1; e < 8; ++e) ss = __fadd_rn(ss, __fmul_rn(x[e], x[e]));
#pragma unroll
        for (int off = L / 2; off >= 1; off >>= 1) ss = __fadd_rn(ss, __shfl_xor_sync(0xffffffffu, ss, off));
        // Packed FP32 pairs and BF16 pairs from here on: every element still sees
        // exactly the same roundings (RN products, RN sums, BF16 RN) as above.
        uint32_t yb[4];                                  // BF16 pairs, dims 8l + 2j, 8l + 2j + 1
        if (w != nullptr) {
          const float ms = __fmul_rn(ss, 1.0f / D);
          const float r = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(ms, a.eps)));
          const uint4 wr = *reinterpret_cast<const uint4*>(w + 8 * l);
          const uint32_t wv[4] = {wr.x, wr.y, wr.z, wr.w};
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint32_t xr = bf16x2_rn(fmul2(make_float2(x[2 * j], x[2 * j + 1]), make_float2(r, r)));
            yb[j] = bf16x2_rn(fmul2(unpack_bf16x2(xr), unpack_bf16x2(wv[j])));
          }
        } else {
          const uint32_t xv[4] = {raw[pidx].x, raw[pidx].y, raw[pidx].z, raw[pidx].w};
#pragma unroll
          for (int j = 0; j < 4; ++j) yb[j] = xv[j];
        }

        // ---- split-half RoPE: lane l < R/16 pairs with lane l + R/16.  Both halves
        //      as y*cos + o*sv, sv = -sin (first half) or +sin (second half), which
        //      is bit for bit y*cos - o*sin or y*cos + o*sin; other lanes pass through.
        if (rot_lanes > 0) {
          const int pl = (l < half_lanes) ? l + half_lanes : (l < rot_lanes ? l - half_lanes : l);
          const int src_lane = sub * L + pl;
          uint32_t ob[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) ob[j] = __shfl_sync(0xffffffffu, yb[j], src_lane);
          if (l < rot_lanes) {
            const bool first = l < half_lanes;
            const int i0 = first ? 8 * l : 8 * l - half;
            const float4 c0 = *reinterpret_cast<const float4*>(&s_cos[k][i0]);
            const float4 c1 = *reinterpret_cast<const float4*>(&s_cos[k][i0 + 4]);
            const float4 n0 = *reinterpret_cast<const float4*>(&s_sin[k][i0]);
            const float4 n1 = *reinterpret_cast<const float4*>(&s_sin[k][i0 + 4]);
            const float cv[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
            const float sn = first ? -1.0f : 1.0f;       // exact sign flip
            const float sv[8] = {sn * n0.x, sn * n0.y, sn * n0.z, sn * n0.w,
                                 sn * n1.x, sn * n1.y, sn * n1.z, sn * n1.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const float2 yc = fmul2(unpack_bf16x2(yb[j]), make_float2(cv[2 * j], cv[2 * j + 1]));
              const float2 os = fmul2(unpack_bf16x2(ob[j]), make_float2(sv[2 * j], sv[2 * j + 1]));
              yb[j] = bf16x2_rn(fadd2(yc, os));
            }
          }
        }

        if (valid) {
          const int H = isq ? a.Hq : a.Hkv;
          uint16_t* dst = (isq ? a.q_out : a.k_out) +
                          ((static_cast<int64_t>(b) * a.N + n) * H + h) * D + 8 * l;
          *reinterpret_cast<uint4*>(dst) = make_uint4(yb[0], yb[1], yb[2], yb[3]);
        }
      }
    }
  }
}

}  // namespace

cudaError_t launch_prep(int B, int N, int Hq, int Hkv, int D, BNHD q, BNHD k,
                        const uint16_t* qw, const uint16_t* kw, float eps, int rotary_dim,
                        double theta, int64_t pos_offset, uint16_t* q_out, uint16_t* k_out,
                        cudaStream_t st) {
  PrepArgs a{q, k, qw, kw, q_out, k_out, B, N, Hq, Hkv, rotary_dim, eps, theta, pos_offset};
  const dim3 grid(static_cast<unsigned>(B) *
                  static_cast<unsigned>((N + QATTN_PREP_TOKENS - 1) / QATTN_PREP_TOKENS));
  switch (D) {
    case 64: prep_kernel<64><<<grid, 256, 0, st>>>(a); break;
    case 128: prep_kernel<128><<<grid, 256, 0, st>>>(a); break;
    case 256: prep_kernel<256><<<grid, 256, 0, st>>>(a); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace qattn
