// quant.cu — K mean / V maxima reductions and the INT8 / FP8 quantizers.
//
// "Exact Numerical Contract": "Preparation" step 4 (exact global K mean per
// head/dim, subtracted before K quantization), "Q And K Quantization" (INT8 Q
// per 32-row group inside 128-row tiles, INT8 K per 64-row block, amax/127
// scales, cvt.rni.sat.s8.f32) and "V And PV" (per-channel global V maximum,
// amax/2.25 scale, E4M3 RN satfinite).  The Hadamard variant follows the page
// "npu plan P7: int8 KV with per-head Hadamard rotation" (rotate Q and K by the
// same per-head H, int8 K with one scale per (head, token)).
//
// All kernels here are HBM-bound: 16-byte vector loads of BF16 rows, one pass
// over the data per kernel, FP64 column partials kept per 64-row block so the
// mean is a fixed-order (rows, then blocks, ascending) sum.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "prep_row.cuh"
#include "qattn_device.cuh"
#include "qattn_internal.h"

namespace qattn {
namespace {

constexpr int kKvRows = 64;   // K scale block / V tile rows
constexpr int kQRows = 32;    // Q scale group rows

__device__ __forceinline__ void unpack8(const uint4 r, float (&x)[8]) {
  x[0] = __uint_as_float(r.x << 16); x[1] = __uint_as_float(r.x & 0xFFFF0000u);
  x[2] = __uint_as_float(r.y << 16); x[3] = __uint_as_float(r.y & 0xFFFF0000u);
  x[4] = __uint_as_float(r.z << 16); x[5] = __uint_as_float(r.z & 0xFFFF0000u);
  x[6] = __uint_as_float(r.w << 16); x[7] = __uint_as_float(r.w & 0xFFFF0000u);
}

__device__ __forceinline__ const uint16_t* row_ptr(const BNHD& t, int b, int n, int h) {
  return t.ptr + b * t.sb + static_cast<int64_t>(n) * t.sn + static_cast<int64_t>(h) * t.sh;
}

// rni + saturate to s8 (the values here never leave [-127.x, 127.x]).
__device__ __forceinline__ int8_t q8_of(float v) {
  int i = __float2int_rn(v);
  i = i > 127 ? 127 : (i < -128 ? -128 : i);
  return static_cast<int8_t>(i);
}

__device__ __forceinline__ uint32_t pack4_s8(int8_t a, int8_t b, int8_t c, int8_t d) {
  return static_cast<uint32_t>(static_cast<uint8_t>(a)) |
         (static_cast<uint32_t>(static_cast<uint8_t>(b)) << 8) |
         (static_cast<uint32_t>(static_cast<uint8_t>(c)) << 16) |
         (static_cast<uint32_t>(static_cast<uint8_t>(d)) << 24);
}

// Max over the CTA (all threads call it); exact in any order.
template <int NT>
__device__ __forceinline__ float block_max(float v, float* red) {
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, off));
  const int warp = threadIdx.x >> 5;
  __syncthreads();
  if ((threadIdx.x & 31) == 0) red[warp] = v;
  __syncthreads();
  float m = red[0];
#pragma unroll
  for (int w = 1; w < NT / 32; ++w) m = fmaxf(m, red[w]);
  return m;
}

// ---------------------------------------------------------------- K / V stats
// One CTA per (64-row block j, batch b): FP64 column sums of K (rows ascending)
// and FP32 column maxima of |V| over the block's valid rows.
__global__ void __launch_bounds__(256) kv_reduce_kernel(int Nkv, int Hkv, int D, BNHD kp,
                                                        bool has_k, BNHD v, double* ksum,
                                                        float* vmax) {
  const int j = blockIdx.x, b = blockIdx.y, nK = gridDim.x;
  const int C = Hkv * D, CC = C / 8;
  const int r0 = j * kKvRows, r1 = min(Nkv, r0 + kKvRows);
  for (int cc = threadIdx.x; cc < CC; cc += blockDim.x) {
    const int h = (cc * 8) / D, d0 = (cc * 8) - h * D;
    double s[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    float m[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    int r = r0;
    for (; r + 4 <= r1; r += 4) {
      uint4 kr[4], vr[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        if (has_k) kr[u] = *reinterpret_cast<const uint4*>(row_ptr(kp, b, r + u, h) + d0);
        vr[u] = *reinterpret_cast<const uint4*>(row_ptr(v, b, r + u, h) + d0);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        float x[8];
        if (has_k) {
          unpack8(kr[u], x);
#pragma unroll
          for (int e = 0; e < 8; ++e) s[e] = __dadd_rn(s[e], static_cast<double>(x[e]));
        }
        unpack8(vr[u], x);
#pragma unroll
        for (int e = 0; e < 8; ++e) m[e] = fmaxf(m[e], fabsf(x[e]));
      }
    }
    for (; r < r1; ++r) {
      float x[8];
      if (has_k) {
        unpack8(*reinterpret_cast<const uint4*>(row_ptr(kp, b, r, h) + d0), x);
#pragma unroll
        for (int e = 0; e < 8; ++e) s[e] = __dadd_rn(s[e], static_cast<double>(x[e]));
      }
      unpack8(*reinterpret_cast<const uint4*>(row_ptr(v, b, r, h) + d0), x);
#pragma unroll
      for (int e = 0; e < 8; ++e) m[e] = fmaxf(m[e], fabsf(x[e]));
    }
    const size_t o = (static_cast<size_t>(b) * nK + j) * C + cc * 8;
    if (has_k) {
#pragma unroll
      for (int e = 0; e < 8; ++e) ksum[o + e] = s[e];
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) vmax[o + e] = m[e];
  }
}

// One thread per (batch, column): blocks summed in ascending order, mean rounded
// once to FP32; V maximum floored at 1e-7f, scale amax/2.25f and factor 2.25f/amax.
__global__ void kv_finalize_kernel(int B, int Nkv, int nK, int C, bool has_k,
                                   const double* ksum, const float* vmax, float* k_mean,
                                   float* v_scale, float* vfac, float vrange = 2.25f) {
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= static_cast<int64_t>(B) * C) return;
  const int b = static_cast<int>(idx / C), c = static_cast<int>(idx - static_cast<int64_t>(b) * C);
  const size_t base = static_cast<size_t>(b) * nK * C + c;
  // loads of K sums and V maxima are issued together, 16 blocks ahead of the
  // (strictly ascending) additions
  double s = 0.0;
  float a = 0.0f;
  int j = 0;
  for (; j + 16 <= nK; j += 16) {
    double ks[16];
    float vm[16];
#pragma unroll
    for (int u = 0; u < 16; ++u) {
      if (has_k) ks[u] = ksum[base + static_cast<size_t>(j + u) * C];
      vm[u] = vmax[base + static_cast<size_t>(j + u) * C];
    }
#pragma unroll
    for (int u = 0; u < 16; ++u) {
      if (has_k) s = __dadd_rn(s, ks[u]);
      a = fmaxf(a, vm[u]);
    }
  }
  for (; j < nK; ++j) {
    if (has_k) s = __dadd_rn(s, ksum[base + static_cast<size_t>(j) * C]);
    a = fmaxf(a, vmax[base + static_cast<size_t>(j) * C]);
  }
  if (has_k) k_mean[idx] = __double2float_rn(__ddiv_rn(s, static_cast<double>(Nkv)));
  a = fmaxf(1e-7f, a);
  v_scale[idx] = __fdiv_rn(a, vrange);      // 2.25 for E4M3 V, 127 for rotated INT8 V
  vfac[idx] = __fdiv_rn(vrange, a);
}

// ---------------------------------------------------------------- quantizer
struct QuantArgs {
  BNHD qp, kp, v;
  const float* k_mean;
  const float* vfac;
  int8_t* q8;
  float* q_scale;
  int8_t* k8;
  float* k_scale;
  uint8_t* v8t;
  int B, Nq, Nkv, Hq, Hkv, G, nK;
  int nq_blocks, nk_blocks, nv_blocks;
  int k_rows;              // rows per K scale: 64, or 32 (scales per 32-row group)
  int nK_scale;            // K scales per (batch, head): ceil(Nkv / k_rows)
  // kp holds RAW K rows to be prepared here (RMSNorm with kw, RoPE from the
  // coefficient tables) before the mean is subtracted; the fused path
  bool k_raw;
  const uint16_t* kw;
  float eps;
  int rotary_dim;
  const uint16_t* cos_t;   // BF16 [Nkv][rotary_dim/2]
  const uint16_t* sin_t;
};

// RoPE coefficients of the lane's 8 pairs at row n of BF16 tables [rows][R/2]
// (R a multiple of 16, so the lane's 8 entries are one 16-byte chunk); the tables
// may be in global or shared memory.
__device__ __forceinline__ void table_coefs(const uint16_t* cos_t, const uint16_t* sin_t, int n,
                                            int half, int l, int half_lanes, float (&cv)[8],
                                            float (&sn)[8]) {
  const int i0 = l < half_lanes ? 8 * l : 8 * l - half;
  unpack8(*reinterpret_cast<const uint4*>(cos_t + static_cast<int64_t>(n) * half + i0), cv);
  unpack8(*reinterpret_cast<const uint4*>(sin_t + static_cast<int64_t>(n) * half + i0), sn);
}

// Copy the RoPE coefficients of tokens n0 .. n0+63 (clamped to N-1) from the
// global tables [N][R/2] into shared memory [2][64][R/2] (all threads; the caller
// synchronizes before use).
__device__ __forceinline__ void stage_tables(const uint16_t* cos_t, const uint16_t* sin_t, int n0,
                                             int N, int half, uint16_t* s_tab) {
  const int per_tok = half / 8;                       // 16-byte chunks per token
  for (int idx = threadIdx.x; idx < kKvRows * per_tok; idx += blockDim.x) {
    const int tok = idx / per_tok, c = idx - tok * per_tok;
    const int64_t n = min(n0 + tok, N - 1);
    *reinterpret_cast<uint4*>(s_tab + tok * half + c * 8) =
        *reinterpret_cast<const uint4*>(cos_t + n * half + c * 8);
    *reinterpret_cast<uint4*>(s_tab + (kKvRows + tok) * half + c * 8) =
        *reinterpret_cast<const uint4*>(sin_t + n * half + c * 8);
  }
}

// RoPE of one normalized row chunk (BF16 pairs yb) in the row layout of
// prep_row.cuh; `n` indexes the row of the (global or staged) tables.
template <int D>
__device__ __forceinline__ uint4 rope_chunk(uint32_t (&yb)[4], int rotary_dim,
                                            const uint16_t* cos_t, const uint16_t* sin_t, int n) {
  constexpr int L = D / 8;
  const int lane = threadIdx.x & 31, sub = lane / L, l = lane - sub * L;
  const int rot_lanes = rotary_dim / 8, half = rotary_dim / 2, half_lanes = half / 8;
  if (rot_lanes > 0) {
    float cv[8], sn[8];
    if (l < rot_lanes) table_coefs(cos_t, sin_t, n, half, l, half_lanes, cv, sn);
    prep::rope8(yb, sub, l, L, half_lanes, rot_lanes, cv, sn);
  }
  return make_uint4(yb[0], yb[1], yb[2], yb[3]);
}

// RMSNorm + RoPE of N raw row chunks of a thread (chunk c: row `rows[c]` of the
// tables), with the rows' r computed together (batch_rms_r).  w == nullptr: no norm.
template <int D, int N>
__device__ __forceinline__ void prep_chunks(uint4 (&x)[N], const int (&rows)[N], const uint16_t* w,
                                            float eps, int rotary_dim, const uint16_t* cos_t,
                                            const uint16_t* sin_t) {
  constexpr int L = D / 8;
  const int l = (threadIdx.x & 31) % L;
  float r[N];
  if (w != nullptr) {
    float ss[N];
#pragma unroll
    for (int c = 0; c < N; ++c) ss[c] = prep::sumsq8<D>(x[c]);
    prep::batch_rms_r<D, N>(ss, eps, r);
  }
#pragma unroll
  for (int c = 0; c < N; ++c) {
    uint32_t yb[4];
    if (w != nullptr) {
      prep::apply_norm8(x[c], w, r[c], l, yb);
    } else {
      yb[0] = x[c].x; yb[1] = x[c].y; yb[2] = x[c].z; yb[3] = x[c].w;
    }
    x[c] = rope_chunk<D>(yb, rotary_dim, cos_t, sin_t, rows[c]);
  }
}

// RMSNorm + RoPE of one raw row chunk in the row layout of prep_row.cuh (L = D/8
// lanes per row); `n` indexes the row of the (global or staged) tables.
template <int D>
__device__ __forceinline__ uint4 prep_chunk(const uint4 raw, const uint16_t* w, float eps,
                                            int rotary_dim, const uint16_t* cos_t,
                                            const uint16_t* sin_t, int n) {
  constexpr int L = D / 8;
  const int lane = threadIdx.x & 31, sub = lane / L, l = lane - sub * L;
  uint32_t yb[4];
  prep::rmsnorm8<D>(raw, w, eps, l, yb);
  const int rot_lanes = rotary_dim / 8, half = rotary_dim / 2, half_lanes = half / 8;
  if (rot_lanes > 0) {
    float cv[8], sn[8];
    if (l < rot_lanes) table_coefs(cos_t, sin_t, n, half, l, half_lanes, cv, sn);
    prep::rope8(yb, sub, l, L, half_lanes, rot_lanes, cv, sn);
  }
  return make_uint4(yb[0], yb[1], yb[2], yb[3]);
}

// A group of ROWS rows x D dims of one (batch, head): amax over valid rows,
// one scale, int8 rows written head-major [B, H, N, D].
// With `pa` (the fused path) the rows are raw K and are first prepared here
// (RMSNorm + RoPE, the same arithmetic as qattn_prep); chunk c of thread t is
// row (t + 128c) / (D/8), which is the row layout of prep_row.cuh.
template <int D, int ROWS>
__device__ __forceinline__ void quant_group(const BNHD& src, const float* mean, int b, int h,
                                            int H, int N, int row0, int8_t* dst8, float* scale_out,
                                            float* red, const QuantArgs* pa = nullptr) {
  constexpr int CPR = D / 8;                 // 16-byte chunks per row
  constexpr int CH = ROWS * CPR / 128;       // chunks per thread
  // The raw BF16 chunks stay in registers (4 per chunk) and are unpacked twice,
  // for the maximum and for the codes, with the same arithmetic both times.
  uint4 raw[CH];
#pragma unroll
  for (int c = 0; c < CH; ++c) {
    const int id = threadIdx.x + c * 128;
    const int r = id / CPR, d0 = (id - r * CPR) * 8;
    const int n = row0 + r;
    raw[c] = (n < N) ? *reinterpret_cast<const uint4*>(row_ptr(src, b, n, h) + d0)
                     : make_uint4(0, 0, 0, 0);
  }
  if (pa != nullptr) {
    // the block's RoPE coefficients, staged once in shared memory (the row loads
    // above are already in flight)
    extern __shared__ __align__(16) uint16_t s_tab[];
    const int half = pa->rotary_dim / 2;
    if (half > 0) {
      stage_tables(pa->cos_t, pa->sin_t, row0, N, half, s_tab);
      __syncthreads();
    }
    int rows[CH];
#pragma unroll
    for (int c = 0; c < CH; ++c) rows[c] = (threadIdx.x + c * 128) / CPR;
    prep_chunks<D, CH>(raw, rows, pa->kw, pa->eps, pa->rotary_dim, s_tab, s_tab + kKvRows * half);
  }
  auto values = [&](int c, float (&x)[8]) {
    const int id = threadIdx.x + c * 128;
    const int d0 = (id % CPR) * 8;
    unpack8(raw[c], x);
    if (mean != nullptr) {
#pragma unroll
      for (int e = 0; e < 8; ++e) x[e] = __fsub_rn(x[e], mean[d0 + e]);
    }
  };
  float amax = 0.0f;
#pragma unroll
  for (int c = 0; c < CH; ++c) {
    const int id = threadIdx.x + c * 128;
    if (row0 + id / CPR < N) {               // rows past the end take no part
      float x[8];
      values(c, x);
#pragma unroll
      for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(x[e]));
    }
  }
  amax = fmaxf(1e-7f, block_max<128>(amax, red));
  const float f = __fdiv_rn(127.0f, amax);
  if (threadIdx.x == 0) *scale_out = __fdiv_rn(amax, 127.0f);
#pragma unroll
  for (int c = 0; c < CH; ++c) {
    const int id = threadIdx.x + c * 128;
    const int r = id / CPR, d0 = (id - r * CPR) * 8;
    const int n = row0 + r;
    if (n < N) {
      float x[8];
      values(c, x);
      int8_t q[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) q[e] = q8_of(__fmul_rn(x[e], f));
      uint2 o;
      o.x = pack4_s8(q[0], q[1], q[2], q[3]);
      o.y = pack4_s8(q[4], q[5], q[6], q[7]);
      *reinterpret_cast<uint2*>(dst8 + ((static_cast<int64_t>(b) * H + h) * N + n) * D + d0) = o;
    }
  }
}

// KRAW: the fused path's second pass (K blocks prepared from raw rows); a separate
// instance so the two-step quantizer keeps its own (smaller) register budget.
template <int D, bool KRAW = false>
__global__ void __launch_bounds__(128) quant_kernel(const QuantArgs a) {
  __shared__ float red[4];
  __shared__ __align__(16) uint8_t tile[D * kKvRows];
  int blk = blockIdx.x;
  if (blk < a.nq_blocks) {                               // ---- Q groups
    const int g = blk % a.G, bh = blk / a.G;
    const int h = bh % a.Hq, b = bh / a.Hq;
    quant_group<D, kQRows>(a.qp, nullptr, b, h, a.Hq, a.Nq, g * kQRows, a.q8,
                           a.q_scale + static_cast<int64_t>(bh) * a.G + g, red);
    return;
  }
  blk -= a.nq_blocks;
  if (blk < a.nk_blocks) {                               // ---- K blocks
    const int j = blk % a.nK_scale, bh = blk / a.nK_scale;
    const int h = bh % a.Hkv, b = bh / a.Hkv;
    const float* mean = a.k_mean + static_cast<int64_t>(bh) * D;
    float* sc = a.k_scale + static_cast<int64_t>(bh) * a.nK_scale + j;
    if constexpr (KRAW) {
      quant_group<D, kKvRows>(a.kp, mean, b, h, a.Hkv, a.Nkv, j * kKvRows, a.k8, sc, red, &a);
    } else {
      if (a.k_rows == kKvRows)
        quant_group<D, kKvRows>(a.kp, mean, b, h, a.Hkv, a.Nkv, j * kKvRows, a.k8, sc, red);
      else
        quant_group<D, kQRows>(a.kp, mean, b, h, a.Hkv, a.Nkv, j * kQRows, a.k8, sc, red);
    }
    return;
  }
  blk -= a.nk_blocks;
  if (blk < a.nv_blocks) {                               // ---- V tiles (transposed)
    const int j = blk % a.nK, bh = blk / a.nK;
    const int h = bh % a.Hkv, b = bh / a.Hkv;
    const float* fac = a.vfac + static_cast<int64_t>(bh) * D;
    // Thread (rg, dc) converts rows 4rg..4rg+3 x dims 8dc..8dc+7 of each 64-dim
    // slab and writes, per dim, the four rows' codes as one 32-bit word of the
    // dim-major tile (byte k = row 4rg+k).
    const int rg = threadIdx.x & 15, dc = threadIdx.x >> 4;
#pragma unroll
    for (int slab = 0; slab < D; slab += 64) {
      const int d0 = slab + 8 * dc;
      uint4 raw[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int n = j * kKvRows + 4 * rg + k;
        raw[k] = (n < a.Nkv) ? *reinterpret_cast<const uint4*>(row_ptr(a.v, b, n, h) + d0)
                             : make_uint4(0, 0, 0, 0);   // zero rows past the end
      }
      float fv[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) fv[e] = fac[d0 + e];
      uint32_t hw[4][4];                                  // [row][dim pair] e4m3 pairs
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        float x[8];
        unpack8(raw[k], x);
#pragma unroll
        for (int e = 0; e < 8; e += 2)
          hw[k][e / 2] = cvt_e4m3x2(__fmul_rn(x[e], fv[e]), __fmul_rn(x[e + 1], fv[e + 1]));
      }
      uint32_t* tw = reinterpret_cast<uint32_t*>(tile);
#pragma unroll
      for (int e2 = 0; e2 < 4; ++e2) {
        const uint32_t u01 = hw[0][e2] | (hw[1][e2] << 16);   // bytes: r0 d, r0 d+1, r1 d, r1 d+1
        const uint32_t u23 = hw[2][e2] | (hw[3][e2] << 16);
        const int d = d0 + 2 * e2;
        tw[(d * kKvRows) / 4 + rg] = __byte_perm(u01, u23, 0x6420);        // dim d, rows 0..3
        tw[((d + 1) * kKvRows) / 4 + rg] = __byte_perm(u01, u23, 0x7531);  // dim d+1
      }
    }
    __syncthreads();
    const int64_t npad = static_cast<int64_t>(a.nK) * kKvRows;
    uint8_t* dst = a.v8t + static_cast<int64_t>(bh) * D * npad + static_cast<int64_t>(j) * kKvRows;
    for (int id = threadIdx.x; id < D * (kKvRows / 16); id += 128) {
      const int d = id / (kKvRows / 16), c = id - d * (kKvRows / 16);
      *reinterpret_cast<uint4*>(dst + d * npad + c * 16) =
          *reinterpret_cast<const uint4*>(tile + d * kKvRows + c * 16);
    }
  }
}

// ---------------------------------------------------------------- fused prep + quant
// RoPE coefficient tables for positions pos_offset + n, n < N: BF16 cos / sin of
// pos * theta^(-2i/R) (FP64, rounded once), [N][R/2] each.
__global__ void rope_table_kernel(int N, int rotary_dim, double theta, int64_t pos_offset,
                                  uint16_t* cos_t, uint16_t* sin_t) {
  const int half = rotary_dim / 2;
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= static_cast<int64_t>(N) * half) return;
  const int n = static_cast<int>(idx / half), i = static_cast<int>(idx - static_cast<int64_t>(n) * half);
  float c, sv;
  prep::rope_coef(pos_offset + n, prep::rope_freq(theta, i, rotary_dim), &c, &sv);
  cos_t[idx] = static_cast<uint16_t>(__float_as_uint(c) >> 16);    // exact: c is a BF16 value
  sin_t[idx] = static_cast<uint16_t>(__float_as_uint(sv) >> 16);
}

struct PrepStatsArgs {
  BNHD q, k, v;                 // raw BF16 inputs
  const uint16_t* qw;
  const uint16_t* kw;
  float eps;
  int rotary_dim;
  const uint16_t* cos_t;
  const uint16_t* sin_t;
  int8_t* q8;
  float* q_scale;
  double* ksum;                 // [B, nK, Hkv*D]
  float* vmax;                  // [B, nK, Hkv*D]
  int B, N, Hq, Hkv, G, nK;
  int nq_ctas;                  // CTAs [0, nq_ctas) do Q, the rest K/V statistics
};

// First pass of the fused path, 128 threads per CTA, two kinds of CTA in one grid:
//  * Q CTA (64-row block j, batch, query head): the block's rows are prepared and
//    quantized at once, its two 32-row groups ("Q And K Quantization"); Q leaves
//    as INT8 with no BF16 copy.
//  * K/V CTA (64-row block j, batch, KV head): its K rows are prepared into shared
//    memory and their FP64 column sums taken over the block in ascending row order
//    (the partials of the K mean, "Preparation" step 4); its V rows give the
//    block's column maxima of |v| ("V And PV").  K is prepared again from the raw
//    rows by the second pass.
// Both stage the block's 64 RoPE coefficient rows in shared memory once.
// Dynamic shared memory: tables 2 x 64 x R/2 BF16, then (K/V CTAs) 64 x D BF16.
constexpr int kPrepStatsThreads = 256;

// D <= 128: at most 64 registers (four CTAs per SM), so a CTA also fits beside an
// attention CTA of another stream (the host pipeline overlaps the two)
template <int D>
__global__ void __launch_bounds__(kPrepStatsThreads, D <= 128 ? 4 : 1) prep_stats_kernel(const PrepStatsArgs a) {
  constexpr int L = D / 8, HPW = 32 / L;       // lanes per row, rows per warp
  constexpr int NW = kPrepStatsThreads / 32;
  constexpr int RPP = NW * HPW;                // rows per pass
  constexpr int PASSES = kKvRows / RPP;
  extern __shared__ __align__(16) uint16_t dyn[];
  __shared__ float red[2][NW];
  __shared__ unsigned vmx[D];                  // |v| column maxima (FP32 bits)
  const int half = a.rotary_dim / 2;
  uint16_t* s_tab = dyn;                       // [2][64][half]
  uint16_t* sK = dyn + 2 * kKvRows * half;     // [64][D]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int sub = lane / L, l = lane - sub * L;
  auto row_of = [&](int p) { return p * RPP + warp * HPW + sub; };
  const bool is_q = static_cast<int>(blockIdx.x) < a.nq_ctas;
  const int id = is_q ? blockIdx.x : blockIdx.x - a.nq_ctas;
  const int j = id % a.nK;
  const int bh = id / a.nK;                    // b * Hq + h (Q) or b * Hkv + hk (K/V)
  const int n0 = j * kKvRows;

  if (is_q) {
    const int h = bh % a.Hq, b = bh / a.Hq;
    uint4 y[PASSES];
#pragma unroll
    for (int p = 0; p < PASSES; ++p) {
      const int n = n0 + row_of(p);
      y[p] = n < a.N ? *reinterpret_cast<const uint4*>(row_ptr(a.q, b, n, h) + 8 * l)
                     : make_uint4(0, 0, 0, 0);
    }
    if (half > 0) stage_tables(a.cos_t, a.sin_t, n0, a.N, half, s_tab);
    __syncthreads();
    int rows[PASSES];
#pragma unroll
    for (int p = 0; p < PASSES; ++p) rows[p] = row_of(p);
    prep_chunks<D, PASSES>(y, rows, a.qw, a.eps, a.rotary_dim, s_tab, s_tab + kKvRows * half);
    float gmax[2] = {0.0f, 0.0f};
#pragma unroll
    for (int p = 0; p < PASSES; ++p) {
      const int n = n0 + row_of(p);
      if (n < a.N) {                                // rows past the end take no part
        float x[8];
        unpack8(y[p], x);
        const int g = (p * RPP) / kQRows;             // a pass lies inside one group
#pragma unroll
        for (int e = 0; e < 8; ++e) gmax[g] = fmaxf(gmax[g], fabsf(x[e]));
      }
    }
#pragma unroll
    for (int g = 0; g < 2; ++g) {
#pragma unroll
      for (int off = 16; off >= 1; off >>= 1) gmax[g] = fmaxf(gmax[g], __shfl_xor_sync(0xffffffffu, gmax[g], off));
      if (lane == 0) red[g][warp] = gmax[g];
    }
    __syncthreads();
    float f[2];
#pragma unroll
    for (int g = 0; g < 2; ++g) {
      float m = red[g][0];
#pragma unroll
      for (int w2 = 1; w2 < NW; ++w2) m = fmaxf(m, red[g][w2]);
      m = fmaxf(1e-7f, m);
      f[g] = __fdiv_rn(127.0f, m);                  // a group with no row: amax 1e-7f
      if (threadIdx.x == g)
        a.q_scale[static_cast<int64_t>(bh) * a.G + 2 * j + g] = __fdiv_rn(m, 127.0f);
    }
#pragma unroll
    for (int p = 0; p < PASSES; ++p) {
      const int n = n0 + row_of(p);
      if (n < a.N) {
        const float fg = f[(p * RPP) / kQRows];
        float x[8];
        unpack8(y[p], x);
        int8_t q[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) q[e] = q8_of(__fmul_rn(x[e], fg));
        uint2 o;
        o.x = pack4_s8(q[0], q[1], q[2], q[3]);
        o.y = pack4_s8(q[4], q[5], q[6], q[7]);
        *reinterpret_cast<uint2*>(a.q8 + (static_cast<int64_t>(bh) * a.N + n) * D + 8 * l) = o;
      }
    }
    // groups of the last 128-row tile past the last 64-row block hold no row
    if (j == a.nK - 1) {
      for (int g = 2 * a.nK + threadIdx.x; g < a.G; g += blockDim.x)
        a.q_scale[static_cast<int64_t>(bh) * a.G + g] = __fdiv_rn(1e-7f, 127.0f);
    }
    return;
  }

  // ---- K/V statistics
  const int hk = bh % a.Hkv, b = bh / a.Hkv;
  const int nv = min(kKvRows, a.N - n0);              // valid rows of the block
  uint4 kraw[PASSES], vraw[PASSES];
#pragma unroll
  for (int p = 0; p < PASSES; ++p) {
    const int n = n0 + row_of(p);
    kraw[p] = n < a.N ? *reinterpret_cast<const uint4*>(row_ptr(a.k, b, n, hk) + 8 * l)
                      : make_uint4(0, 0, 0, 0);
    vraw[p] = n < a.N ? *reinterpret_cast<const uint4*>(row_ptr(a.v, b, n, hk) + 8 * l)
                      : make_uint4(0, 0, 0, 0);
  }
  for (int d = threadIdx.x; d < D; d += blockDim.x) vmx[d] = 0u;
  if (half > 0) stage_tables(a.cos_t, a.sin_t, n0, a.N, half, s_tab);
  __syncthreads();
  {
    int rows[PASSES];
#pragma unroll
    for (int p = 0; p < PASSES; ++p) rows[p] = row_of(p);
    prep_chunks<D, PASSES>(kraw, rows, a.kw, a.eps, a.rotary_dim, s_tab, s_tab + kKvRows * half);
#pragma unroll
    for (int p = 0; p < PASSES; ++p)
      *reinterpret_cast<uint4*>(sK + rows[p] * D + 8 * l) = kraw[p];
  }
  float vm[8] = {0, 0, 0, 0, 0, 0, 0, 0};
#pragma unroll
  for (int p = 0; p < PASSES; ++p) {
    if (n0 + row_of(p) < a.N) {
      float x[8];
      unpack8(vraw[p], x);
#pragma unroll
      for (int e = 0; e < 8; ++e) vm[e] = fmaxf(vm[e], fabsf(x[e]));
    }
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) {
#pragma unroll
    for (int off = L; off < 32; off <<= 1) vm[e] = fmaxf(vm[e], __shfl_xor_sync(0xffffffffu, vm[e], off));
  }
  if (sub == 0) {
#pragma unroll
    for (int e = 0; e < 8; ++e) atomicMax(&vmx[8 * l + e], __float_as_uint(vm[e]));   // |v| >= 0
  }
  __syncthreads();                                  // sK written, every atomicMax landed
  // FP64 column sums over the block's valid rows, ascending (one column per thread)
  const int C = a.Hkv * D;
  const size_t o = (static_cast<size_t>(b) * a.nK + j) * C + static_cast<size_t>(hk) * D;
  for (int d = threadIdx.x; d < D; d += blockDim.x) {
    double sacc = 0.0;
    for (int r = 0; r < nv; ++r)
      sacc = __dadd_rn(sacc, static_cast<double>(__uint_as_float(static_cast<uint32_t>(sK[r * D + d]) << 16)));
    a.ksum[o + d] = sacc;
    a.vmax[o + d] = __uint_as_float(vmx[d]);
  }
}

// ---------------------------------------------------------------- FP16 V
// V for the FP16 P.V product: BF16 -> FP16 round to nearest even, no scale,
// stored dim-major [B, Hkv, D, cap] (keys contiguous).  One CTA per 64-key tile
// of one (batch, head): source rows 0 .. n_src-1 go to keys key0 .. of the
// destination; keys key0 + [n_src, n_write) are written as 0 (n_write a multiple
// of 8 and key0 + n_write <= cap, both checked by the caller), keys outside
// [key0, key0 + n_write) are not touched.
template <int D>
__global__ void __launch_bounds__(128) quant_v16_kernel(BNHD v, int n_src, int Hkv, int cap,
                                                        int key0, int n_write, uint16_t* v16t) {
  __shared__ __align__(16) uint16_t tile[D * kKvRows];   // [d][key]
  const int j = blockIdx.x, bh = blockIdx.y, b = bh / Hkv, h = bh - b * Hkv;
  constexpr int CPR = D / 8;
  for (int id = threadIdx.x; id < kKvRows * CPR; id += blockDim.x) {
    const int r = id / CPR, d0 = (id - r * CPR) * 8, n = j * kKvRows + r;
    const uint4 raw = n < n_src ? *reinterpret_cast<const uint4*>(row_ptr(v, b, n, h) + d0)
                                : make_uint4(0, 0, 0, 0);
    float x[8];
    unpack8(raw, x);
#pragma unroll
    for (int e = 0; e < 8; ++e) tile[(d0 + e) * kKvRows + r] = __half_as_ushort(__float2half_rn(x[e]));
  }
  __syncthreads();
  const int kmax = min(kKvRows, n_write - j * kKvRows);  // keys of this tile to write (multiple of 8)
  uint16_t* dst = v16t + static_cast<int64_t>(bh) * D * cap + key0 + j * kKvRows;
  for (int id = threadIdx.x; id < D * (kKvRows / 8); id += blockDim.x) {
    const int d = id / (kKvRows / 8), c = id - d * (kKvRows / 8);
    if (c * 8 < kmax)
      *reinterpret_cast<uint4*>(dst + static_cast<int64_t>(d) * cap + c * 8) =
          *reinterpret_cast<const uint4*>(tile + d * kKvRows + c * 8);
  }
}

// ---------------------------------------------------------------- Hadamard
// In-warp Walsh-Hadamard transform of one D-element row held as E = D/32
// consecutive elements per lane, stages h = 1, 2, ..., D/2 in order; each stage
// maps (a at i, b at i+h) to (a+b, a-b) in FP32.
template <int D>
__device__ __forceinline__ void fwht_row(float (&v)[D / 32]) {
  constexpr int E = D / 32;
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int h = 1; h < E; h <<= 1) {
#pragma unroll
    for (int k = 0; k < E; ++k) {
      if ((k & h) == 0) {
        const float a = v[k], b = v[k + h];
        v[k] = __fadd_rn(a, b);
        v[k + h] = __fsub_rn(a, b);
      }
    }
  }
#pragma unroll
  for (int h = E; h < D; h <<= 1) {
    const int lm = h / E;
    const bool lower = (lane & lm) == 0;
#pragma unroll
    for (int k = 0; k < E; ++k) {
      const float o = __shfl_xor_sync(0xffffffffu, v[k], lm);
      v[k] = lower ? __fadd_rn(v[k], o) : __fsub_rn(o, v[k]);
    }
  }
}

template <int D>
__device__ __forceinline__ void load_row_e(const BNHD& t, int b, int n, int h, float (&v)[D / 32]) {
  constexpr int E = D / 32;
  const int lane = threadIdx.x & 31;
  const uint16_t* p = row_ptr(t, b, n, h) + lane * E;
  if constexpr (E == 8) {
    unpack8(*reinterpret_cast<const uint4*>(p), v);
  } else {
    const uint32_t u = *reinterpret_cast<const uint32_t*>(p);  // E == 2
    v[0] = __uint_as_float(u << 16);
    v[1] = __uint_as_float(u & 0xFFFF0000u);
  }
}

template <int D>
__device__ __forceinline__ void store_q8_e(int8_t* dst, const float (&v)[D / 32], float f) {
  constexpr int E = D / 32;
  const int lane = threadIdx.x & 31;
  if constexpr (E == 8) {
    int8_t q[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) q[e] = q8_of(__fmul_rn(v[e], f));
    uint2 o;
    o.x = pack4_s8(q[0], q[1], q[2], q[3]);
    o.y = pack4_s8(q[4], q[5], q[6], q[7]);
    *reinterpret_cast<uint2*>(dst + lane * 8) = o;
  } else {
    const uint16_t o = static_cast<uint16_t>(static_cast<uint8_t>(q8_of(__fmul_rn(v[0], f)))) |
                       static_cast<uint16_t>(static_cast<uint8_t>(q8_of(__fmul_rn(v[1], f))) << 8);
    *reinterpret_cast<uint16_t*>(dst + lane * 2) = o;
  }
}

struct HadArgs {
  BNHD q, k;
  int8_t* q8;
  float* q_scale;
  int8_t* k8;
  uint16_t* k_scale16;
  int B, Nq, Nkv, Hq, Hkv, G;
  int nq_blocks, nk_blocks;
  int kcap, key0;      // K rows land at key0 + n of planes of kcap rows (a key cache)
};

// Q: one CTA (8 warps, 4 rows each) per 32-row group; K: one warp per token.
template <int D>
__global__ void __launch_bounds__(256) hadamard_quant_kernel(const HadArgs a) {
  constexpr int E = D / 32;
  constexpr float kNorm = (D == 256) ? 0.0625f : 0.125f;   // 1/sqrt(D), exact
  __shared__ float red[8];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int blk = blockIdx.x;
  if (blk < a.nq_blocks) {
    const int g = blk % a.G, bh = blk / a.G;
    const int h = bh % a.Hq, b = bh / a.Hq;
    float v[4][E];
    float amax = 0.0f;
#pragma unroll
    for (int rr = 0; rr < 4; ++rr) {
      const int n = g * kQRows + warp * 4 + rr;
      if (n < a.Nq) {                                  // warp-uniform
        load_row_e<D>(a.q, b, n, h, v[rr]);
        fwht_row<D>(v[rr]);
#pragma unroll
        for (int e = 0; e < E; ++e) {
          v[rr][e] = __fmul_rn(v[rr][e], kNorm);
          amax = fmaxf(amax, fabsf(v[rr][e]));
        }
      }
    }
    amax = fmaxf(1e-7f, block_max<256>(amax, red));
    const float f = __fdiv_rn(127.0f, amax);
    if (threadIdx.x == 0) a.q_scale[static_cast<int64_t>(bh) * a.G + g] = __fdiv_rn(amax, 127.0f);
#pragma unroll
    for (int rr = 0; rr < 4; ++rr) {
      const int n = g * kQRows + warp * 4 + rr;
      if (n < a.Nq) store_q8_e<D>(a.q8 + ((static_cast<int64_t>(bh)) * a.Nq + n) * D, v[rr], f);
    }
    return;
  }
  blk -= a.nq_blocks;
  const int64_t tok = static_cast<int64_t>(blk) * 8 + warp;   // (b, hkv, n) flattened
  if (tok >= static_cast<int64_t>(a.B) * a.Hkv * a.Nkv) return;
  const int n = static_cast<int>(tok % a.Nkv);
  const int bh = static_cast<int>(tok / a.Nkv);
  const int h = bh % a.Hkv, b = bh / a.Hkv;
  float v[E];
  load_row_e<D>(a.k, b, n, h, v);
  fwht_row<D>(v);
  float amax = 0.0f;
#pragma unroll
  for (int e = 0; e < E; ++e) {
    v[e] = __fmul_rn(v[e], kNorm);
    amax = fmaxf(amax, fabsf(v[e]));
  }
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
  amax = fmaxf(1e-7f, amax);
  const float f = __fdiv_rn(127.0f, amax);
  const int64_t slot = static_cast<int64_t>(bh) * a.kcap + a.key0 + n;   // destination row
  if (lane == 0) a.k_scale16[slot] = __half_as_ushort(__float2half_rn(__fdiv_rn(amax, 127.0f)));
  store_q8_e<D>(a.k8 + slot * D, v, f);
}

// ---------------------------------------------------------------- rotated INT8 V
// V' = V H/sqrt(D) per token (fwht_row, the rotation of the K path), INT8 with one
// scale per (batch, head, channel).  Statistics: one CTA (8 warps) per (64-row
// block j, batch, head), a warp per row, |v'| column maxima of the block.
template <int D>
__global__ void __launch_bounds__(256) vrot_stats_kernel(BNHD v, int Nkv, int Hkv, int nK,
                                                         float* vmax) {
  constexpr int E = D / 32;
  constexpr float kNorm = (D == 256) ? 0.0625f : 0.125f;   // 1/sqrt(D), exact
  __shared__ unsigned cmax[D];
  const int j = blockIdx.x, bh = blockIdx.y, b = bh / Hkv, h = bh - b * Hkv;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int d = threadIdx.x; d < D; d += blockDim.x) cmax[d] = 0u;
  __syncthreads();
  float m[E];
#pragma unroll
  for (int e = 0; e < E; ++e) m[e] = 0.0f;
  for (int r = warp; r < kKvRows; r += 8) {
    const int n = j * kKvRows + r;
    if (n >= Nkv) break;                             // warp-uniform
    float x[E];
    load_row_e<D>(v, b, n, h, x);
    fwht_row<D>(x);
#pragma unroll
    for (int e = 0; e < E; ++e) m[e] = fmaxf(m[e], fabsf(__fmul_rn(x[e], kNorm)));
  }
#pragma unroll
  for (int e = 0; e < E; ++e) atomicMax(&cmax[lane * E + e], __float_as_uint(m[e]));
  __syncthreads();
  const size_t o = (static_cast<size_t>(b) * nK + j) * Hkv * D + static_cast<size_t>(h) * D;
  for (int d = threadIdx.x; d < D; d += blockDim.x) vmax[o + d] = __uint_as_float(cmax[d]);
}

// Codes: one CTA per (64-row block, batch, head): rows rotated again (the same
// arithmetic), times 127/amax of their channel, rint-sat to INT8, transposed into
// the dim-major [B, H, D, 64 nK] tile (keys past Nkv are 0).
template <int D>
__global__ void __launch_bounds__(256) vrot_quant_kernel(BNHD v, int Nkv, int Hkv, int nK,
                                                         const float* vfac, int8_t* v8t) {
  constexpr int E = D / 32;
  constexpr float kNorm = (D == 256) ? 0.0625f : 0.125f;
  __shared__ __align__(16) int8_t tile[D * kKvRows];   // [d][key]
  const int j = blockIdx.x, bh = blockIdx.y, b = bh / Hkv, h = bh - b * Hkv;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const float* fac = vfac + static_cast<int64_t>(bh) * D;
  float f[E];
#pragma unroll
  for (int e = 0; e < E; ++e) f[e] = fac[lane * E + e];
  for (int r = warp; r < kKvRows; r += 8) {
    const int n = j * kKvRows + r;
    float x[E];
    if (n < Nkv) {
      load_row_e<D>(v, b, n, h, x);
      fwht_row<D>(x);
    }
#pragma unroll
    for (int e = 0; e < E; ++e)
      tile[(lane * E + e) * kKvRows + r] = n < Nkv ? q8_of(__fmul_rn(__fmul_rn(x[e], kNorm), f[e])) : 0;
  }
  __syncthreads();
  const int64_t npad = static_cast<int64_t>(nK) * kKvRows;
  int8_t* dst = v8t + static_cast<int64_t>(bh) * D * npad + static_cast<int64_t>(j) * kKvRows;
  for (int id = threadIdx.x; id < D * (kKvRows / 16); id += blockDim.x) {
    const int d = id / (kKvRows / 16), c = id - d * (kKvRows / 16);
    *reinterpret_cast<uint4*>(dst + d * npad + c * 16) =
        *reinterpret_cast<const uint4*>(tile + d * kKvRows + c * 16);
  }
}

}  // namespace

cudaError_t launch_quant_v_rotated(int B, int Nkv, int Hkv, int D, BNHD v, QuantWorkspace ws,
                                   int8_t* v8t, float* v_scale, cudaStream_t st) {
  const int nK = (Nkv + kKvRows - 1) / kKvRows;
  const dim3 grid(nK, B * Hkv);
  switch (D) {
    case 64: vrot_stats_kernel<64><<<grid, 256, 0, st>>>(v, Nkv, Hkv, nK, ws.vmax); break;
    case 256: vrot_stats_kernel<256><<<grid, 256, 0, st>>>(v, Nkv, Hkv, nK, ws.vmax); break;
    default: return cudaErrorInvalidValue;
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int C = Hkv * D;
  const int64_t cols = static_cast<int64_t>(B) * C;
  kv_finalize_kernel<<<static_cast<unsigned>((cols + 255) / 256), 256, 0, st>>>(
      B, Nkv, nK, C, false, nullptr, ws.vmax, nullptr, v_scale, ws.vfac, 127.0f);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  switch (D) {
    case 64: vrot_quant_kernel<64><<<grid, 256, 0, st>>>(v, Nkv, Hkv, nK, ws.vfac, v8t); break;
    case 256: vrot_quant_kernel<256><<<grid, 256, 0, st>>>(v, Nkv, Hkv, nK, ws.vfac, v8t); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

size_t quant_workspace_bytes(int B, int Nkv, int Hkv, int D) {
  const size_t nK = (static_cast<size_t>(Nkv) + kKvRows - 1) / kKvRows;
  const size_t C = static_cast<size_t>(Hkv) * D;
  auto up = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
  return up(B * nK * C * sizeof(double)) + up(B * nK * C * sizeof(float)) +
         up(B * C * sizeof(float));
}

QuantWorkspace carve_workspace(void* ws, int B, int Nkv, int Hkv, int D) {
  const size_t nK = (static_cast<size_t>(Nkv) + kKvRows - 1) / kKvRows;
  const size_t C = static_cast<size_t>(Hkv) * D;
  auto up = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
  char* p = static_cast<char*>(ws);
  QuantWorkspace w;
  w.ksum = reinterpret_cast<double*>(p);
  p += up(B * nK * C * sizeof(double));
  w.vmax = reinterpret_cast<float*>(p);
  p += up(B * nK * C * sizeof(float));
  w.vfac = reinterpret_cast<float*>(p);
  return w;
}

cudaError_t launch_kv_stats(int B, int Nkv, int Hkv, int D, const BNHD* kp, BNHD v,
                            QuantWorkspace ws, float* k_mean, float* v_scale, cudaStream_t st) {
  const int nK = (Nkv + kKvRows - 1) / kKvRows;
  const int C = Hkv * D;
  const bool has_k = kp != nullptr;
  kv_reduce_kernel<<<dim3(nK, B), 256, 0, st>>>(Nkv, Hkv, D, has_k ? *kp : v, has_k, v, ws.ksum,
                                                ws.vmax);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int64_t cols = static_cast<int64_t>(B) * C;
  kv_finalize_kernel<<<static_cast<unsigned>((cols + 255) / 256), 256, 0, st>>>(
      B, Nkv, nK, C, has_k, ws.ksum, ws.vmax, k_mean, v_scale, ws.vfac);
  return cudaGetLastError();
}

cudaError_t launch_quant(int B, int Nq, int Nkv, int Hq, int Hkv, int D, BNHD qp, BNHD kp,
                         BNHD v, const float* k_mean, const float* vfac, int8_t* q8,
                         float* q_scale, int8_t* k8, float* k_scale, uint8_t* v8t,
                         cudaStream_t st, int k_rows) {
  QuantArgs a{};
  a.k_rows = k_rows;
  a.nK_scale = (Nkv + k_rows - 1) / k_rows;
  a.qp = qp; a.kp = kp; a.v = v;
  a.k_mean = k_mean; a.vfac = vfac;
  a.q8 = q8; a.q_scale = q_scale; a.k8 = k8; a.k_scale = k_scale; a.v8t = v8t;
  a.B = B; a.Nq = Nq; a.Nkv = Nkv; a.Hq = Hq; a.Hkv = Hkv;
  a.G = 4 * ((Nq + 127) / 128);
  a.nK = (Nkv + kKvRows - 1) / kKvRows;
  a.nq_blocks = q8 ? B * Hq * a.G : 0;
  a.nk_blocks = k8 ? B * Hkv * a.nK_scale : 0;
  a.nv_blocks = v8t ? B * Hkv * a.nK : 0;
  const unsigned grid = static_cast<unsigned>(a.nq_blocks + a.nk_blocks + a.nv_blocks);
  switch (D) {
    case 64: quant_kernel<64><<<grid, 128, 0, st>>>(a); break;
    case 128: quant_kernel<128><<<grid, 128, 0, st>>>(a); break;
    case 256: quant_kernel<256><<<grid, 128, 0, st>>>(a); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

// Launch with `smem` bytes of dynamic shared memory (raising the kernel's limit
// when it exceeds the default 48 KB).
template <typename Args>
cudaError_t launch_dyn(void (*kern)(const Args), unsigned grid, unsigned block, int smem,
                       cudaStream_t st, const Args& a) {
  if (smem > 48 * 1024) {
    const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
  }
  kern<<<grid, block, smem, st>>>(a);
  return cudaGetLastError();
}

size_t prep_quant_table_bytes(int N, int rotary_dim) {
  return ((static_cast<size_t>(N) * (rotary_dim / 2) * sizeof(uint16_t) + 255) & ~static_cast<size_t>(255)) * 2;
}

cudaError_t launch_prep_quant(int B, int N, int Hq, int Hkv, int D, BNHD q, BNHD k, BNHD v,
                              const uint16_t* qw, const uint16_t* kw, float eps, int rotary_dim,
                              double theta, int64_t pos_offset, int8_t* q8, float* q_scale,
                              int8_t* k8, float* k_scale, float* k_mean, uint8_t* v8t,
                              float* v_scale, void* ws, cudaStream_t st) {
  const int nK = (N + kKvRows - 1) / kKvRows;
  QuantWorkspace w = carve_workspace(ws, B, N, Hkv, D);
  uint16_t* cos_t = reinterpret_cast<uint16_t*>(static_cast<char*>(ws) + quant_workspace_bytes(B, N, Hkv, D));
  uint16_t* sin_t = cos_t + prep_quant_table_bytes(N, rotary_dim) / 2 / sizeof(uint16_t);
  cudaError_t e;
  if (rotary_dim > 0) {
    const int64_t cnt = static_cast<int64_t>(N) * (rotary_dim / 2);
    rope_table_kernel<<<static_cast<unsigned>((cnt + 255) / 256), 256, 0, st>>>(
        N, rotary_dim, theta, pos_offset, cos_t, sin_t);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  PrepStatsArgs pa{q, k, v, qw, kw, eps, rotary_dim, cos_t, sin_t, q8, q_scale, w.ksum, w.vmax,
                   B, N, Hq, Hkv, 4 * ((N + 127) / 128), nK, nK * B * Hq};
  const unsigned grid1 = static_cast<unsigned>(nK) * B * (Hq + Hkv);
  const int tab_bytes = 2 * kKvRows * (rotary_dim / 2) * 2;
  const int smem1 = tab_bytes + kKvRows * D * 2;
  switch (D) {
    case 64: e = launch_dyn(prep_stats_kernel<64>, grid1, kPrepStatsThreads, smem1, st, pa); break;
    case 128: e = launch_dyn(prep_stats_kernel<128>, grid1, kPrepStatsThreads, smem1, st, pa); break;
    case 256: e = launch_dyn(prep_stats_kernel<256>, grid1, kPrepStatsThreads, smem1, st, pa); break;
    default: return cudaErrorInvalidValue;
  }
  if (e != cudaSuccess) return e;
  const int C = Hkv * D;
  const int64_t cols = static_cast<int64_t>(B) * C;
  kv_finalize_kernel<<<static_cast<unsigned>((cols + 255) / 256), 256, 0, st>>>(
      B, N, nK, C, true, w.ksum, w.vmax, k_mean, v_scale, w.vfac);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  QuantArgs a{};
  a.kp = k; a.v = v; a.qp = q;
  a.k_mean = k_mean; a.vfac = w.vfac;
  a.k8 = k8; a.k_scale = k_scale; a.v8t = v8t;
  a.B = B; a.Nq = N; a.Nkv = N; a.Hq = Hq; a.Hkv = Hkv;
  a.G = 4 * ((N + 127) / 128);
  a.nK = nK;
  a.nq_blocks = 0;
  a.k_rows = kKvRows;
  a.nK_scale = nK;
  a.nk_blocks = B * Hkv * nK;
  a.nv_blocks = B * Hkv * nK;
  a.k_raw = true; a.kw = kw; a.eps = eps; a.rotary_dim = rotary_dim; a.cos_t = cos_t; a.sin_t = sin_t;
  const unsigned g2 = static_cast<unsigned>(a.nk_blocks + a.nv_blocks);
  switch (D) {   // dynamic shared memory: the staged RoPE tables of a raw-K block
    case 64: return launch_dyn(quant_kernel<64, true>, g2, 128, tab_bytes, st, a);
    case 128: return launch_dyn(quant_kernel<128, true>, g2, 128, tab_bytes, st, a);
    case 256: return launch_dyn(quant_kernel<256, true>, g2, 128, tab_bytes, st, a);
    default: return cudaErrorInvalidValue;
  }
}

// Rotated INT8 Q only (q8 [B,Hq,Nq,D], one scale per 32-row group), or rotated
// per-token INT8 K only, written at rows key0 .. key0+Nkv-1 of [B,Hkv,kcap,D]
// (scales [B,Hkv,kcap]): the pieces of the chunked key-cache path.
cudaError_t launch_hadamard_part(int B, int N, int H, int D, BNHD x, bool is_q, int8_t* x8,
                                 void* scale, int kcap, int key0, cudaStream_t st) {
  HadArgs a{};
  a.B = B; a.Hq = H; a.Hkv = H; a.Nq = N; a.Nkv = N;
  a.kcap = kcap; a.key0 = key0;
  a.G = 4 * ((N + 127) / 128);
  if (is_q) {
    a.q = x; a.q8 = x8; a.q_scale = static_cast<float*>(scale);
    a.nq_blocks = B * H * a.G;
    a.nk_blocks = 0;
  } else {
    a.k = x; a.k8 = x8; a.k_scale16 = static_cast<uint16_t*>(scale);
    a.nq_blocks = 0;
    a.nk_blocks = static_cast<int>((static_cast<int64_t>(B) * H * N + 7) / 8);
  }
  const unsigned grid = static_cast<unsigned>(a.nq_blocks + a.nk_blocks);
  switch (D) {
    case 64: hadamard_quant_kernel<64><<<grid, 256, 0, st>>>(a); break;
    case 256: hadamard_quant_kernel<256><<<grid, 256, 0, st>>>(a); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t launch_quant_v16(int B, int n_src, int Hkv, int D, BNHD v, int cap, int key0,
                             int n_write, uint16_t* v16t, cudaStream_t st) {
  const dim3 grid((n_write + kKvRows - 1) / kKvRows, B * Hkv);
  switch (D) {
    case 64: quant_v16_kernel<64><<<grid, 128, 0, st>>>(v, n_src, Hkv, cap, key0, n_write, v16t); break;
    case 128: quant_v16_kernel<128><<<grid, 128, 0, st>>>(v, n_src, Hkv, cap, key0, n_write, v16t); break;
    case 256: quant_v16_kernel<256><<<grid, 128, 0, st>>>(v, n_src, Hkv, cap, key0, n_write, v16t); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t launch_quant_hadamard(int B, int Nq, int Nkv, int Hq, int Hkv, int D, BNHD q,
                                  BNHD k, BNHD v, const float* vfac, int8_t* q8,
                                  float* q_scale, int8_t* k8, uint16_t* k_scale16,
                                  uint8_t* v8t, cudaStream_t st) {
  HadArgs a{};
  a.q = q; a.k = k; a.q8 = q8; a.q_scale = q_scale; a.k8 = k8; a.k_scale16 = k_scale16;
  a.B = B; a.Nq = Nq; a.Nkv = Nkv; a.Hq = Hq; a.Hkv = Hkv;
  a.kcap = Nkv; a.key0 = 0;
  a.G = 4 * ((Nq + 127) / 128);
  a.nq_blocks = B * Hq * a.G;
  const int64_t toks = static_cast<int64_t>(B) * Hkv * Nkv;
  a.nk_blocks = static_cast<int>((toks + 7) / 8);
  const unsigned grid = static_cast<unsigned>(a.nq_blocks + a.nk_blocks);
  switch (D) {
    case 64: hadamard_quant_kernel<64><<<grid, 256, 0, st>>>(a); break;
    case 256: hadamard_quant_kernel<256><<<grid, 256, 0, st>>>(a); break;
    default: return cudaErrorInvalidValue;
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  // V: per-channel FP8, same tiles as the standard quantizer (no Q, no K part)
  return launch_quant(B, Nq, Nkv, Hq, Hkv, D, q, k, v, nullptr, vfac, nullptr, nullptr, nullptr,
                      nullptr, v8t, st, kKvRows);
}

}  // namespace qattn
