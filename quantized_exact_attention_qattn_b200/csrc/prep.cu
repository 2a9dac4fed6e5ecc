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

#include "prep_row.cuh"
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

using namespace prep;

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
  for (int i = threadIdx.x; i < half; i += blockDim.x) s_freq[i] = rope_freq(a.theta, i, a.rotary_dim);
  __syncthreads();
  for (int idx = threadIdx.x; idx < nt * half; idx += blockDim.x) {
    const int k = idx / half, i = idx - k * half;
    rope_coef(a.pos_offset + n0 + k, s_freq[i], &s_cos[k][i], &s_sin[k][i]);
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
        uint32_t yb[4];                                  // BF16 pairs, dims 8l + 2j, 8l + 2j + 1
        rmsnorm8<D>(raw[pidx], w, a.eps, l, yb);
        if (rot_lanes > 0) {
          float cv[8], sn[8];
          if (l < rot_lanes) {
            const int i0 = l < half_lanes ? 8 * l : 8 * l - half;
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              cv[e] = s_cos[k][i0 + e];
              sn[e] = s_sin[k][i0 + e];
            }
          }
          rope8(yb, sub, l, L, half_lanes, rot_lanes, cv, sn);
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
