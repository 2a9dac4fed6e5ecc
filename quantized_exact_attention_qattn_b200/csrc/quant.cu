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
                                   float* v_scale, float* vfac) {
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
  v_scale[idx] = __fdiv_rn(a, 2.25f);
  vfac[idx] = __fdiv_rn(2.25f, a);
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
};

// A group of ROWS rows x D dims of one (batch, head): amax over valid rows,
// one scale, int8 rows written head-major [B, H, N, D].
template <int D, int ROWS>
__device__ __forceinline__ void quant_group(const BNHD& src, const float* mean, int b, int h,
                                            int H, int N, int row0, int8_t* dst8, float* scale_out,
                                            float* red) {
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

template <int D>
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
    const int j = blk % a.nK, bh = blk / a.nK;
    const int h = bh % a.Hkv, b = bh / a.Hkv;
    quant_group<D, kKvRows>(a.kp, a.k_mean + static_cast<int64_t>(bh) * D, b, h, a.Hkv, a.Nkv,
                            j * kKvRows, a.k8, a.k_scale + static_cast<int64_t>(bh) * a.nK + j,
                            red);
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
  if (lane == 0) a.k_scale16[tok] = __half_as_ushort(__float2half_rn(__fdiv_rn(amax, 127.0f)));
  store_q8_e<D>(a.k8 + tok * D, v, f);
}

}  // namespace

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
                         cudaStream_t st) {
  QuantArgs a{};
  a.qp = qp; a.kp = kp; a.v = v;
  a.k_mean = k_mean; a.vfac = vfac;
  a.q8 = q8; a.q_scale = q_scale; a.k8 = k8; a.k_scale = k_scale; a.v8t = v8t;
  a.B = B; a.Nq = Nq; a.Nkv = Nkv; a.Hq = Hq; a.Hkv = Hkv;
  a.G = 4 * ((Nq + 127) / 128);
  a.nK = (Nkv + kKvRows - 1) / kKvRows;
  a.nq_blocks = q8 ? B * Hq * a.G : 0;
  a.nk_blocks = k8 ? B * Hkv * a.nK : 0;
  a.nv_blocks = B * Hkv * a.nK;
  const unsigned grid = static_cast<unsigned>(a.nq_blocks + a.nk_blocks + a.nv_blocks);
  switch (D) {
    case 64: quant_kernel<64><<<grid, 128, 0, st>>>(a); break;
    case 128: quant_kernel<128><<<grid, 128, 0, st>>>(a); break;
    case 256: quant_kernel<256><<<grid, 128, 0, st>>>(a); break;
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
                      nullptr, v8t, st);
}

}  // namespace qattn
