// attn_common.cuh — building blocks of the attention mainloop (attn_fwd.cu): the
// softmax constants of the "Online Softmax" section, the launch parameters, the
// exponential, the score bias, the O rescale, and the TMA tensor-map encoder.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <mutex>

#include "qattn_device.cuh"
#include "qattn_internal.h"

namespace qattn {
namespace attn {

constexpr int BM = 128;   // query rows per tile (TMEM lanes)
constexpr float kMInit = -5000000.0f;
constexpr float kFp8Offset = 8.807f;

struct FwdParams {
  const int8_t* q8;     // [B,Hq,Nq,D]: read directly when Q lives in tensor memory
  const float* q_scale;
  const void* k_scale;
  const float* v_scale;
  uint16_t* out;
  int* dev_err;
  int B, Nq, Nkv, Hq, Hkv, G, nK, nQ, n_groups;
  float c;
  int stall_tile;   // test hook: K/V tile whose copy is never issued (-1: none)
  int kcap;         // K rows per (batch, head) plane of k8 (>= Nkv)
  int ks_stride;    // K scales per (batch, head) in k_scale
  // score copy-out (qattn_scores only): n_dump requested (b, h, q_tile, k_tile)
  // quads and one [128][64] INT32 slot per quad
  const int4* dump_tiles;
  int32_t* dump_out;
  int n_dump;
};

// Score copy-out of the debug build of the mainloop (qattn_scores).  The thread
// owning query row `row` holds NCOL consecutive scores of key tile t, starting at
// column col0, as the softmax reads them: x[j] - bias is the exact INT32 score
// (bias = kSBias, the output of the bias MMA that the scores accumulate onto).  Every slot whose request names (b, h, qt, t) receives them; the
// warp's lanes scan the request list 32 entries at a time.
template <int NCOL>
__device__ __forceinline__ void dump_scores(const FwdParams& p, int b, int h, int qt, int t,
                                            int row, int col0, const float (&x)[NCOL],
                                            float bias) {
  const int lane = threadIdx.x & 31;
  for (int base = 0; base < p.n_dump; base += 32) {
    bool hit = false;
    if (base + lane < p.n_dump) {
      const int4 r = p.dump_tiles[base + lane];
      hit = r.x == b && r.y == h && r.z == qt && r.w == t;
    }
    uint32_t m = __ballot_sync(0xffffffffu, hit);
    while (m) {
      const int slot = base + __ffs(m) - 1;
      m &= m - 1;
      int4* dst = reinterpret_cast<int4*>(p.dump_out + (static_cast<int64_t>(slot) * BM + row) * 64 + col0);
#pragma unroll
      for (int j = 0; j < NCOL; j += 4)
        dst[j / 4] = make_int4(__float2int_rn(__fsub_rn(x[j], bias)), __float2int_rn(__fsub_rn(x[j + 1], bias)),
                               __float2int_rn(__fsub_rn(x[j + 2], bias)), __float2int_rn(__fsub_rn(x[j + 3], bias)));
    }
  }
}

// ---------------------------------------------------------------- exp2
// Columns j with (j % 8) < kPolyPer8 evaluate 2^t with an FMA-pipe polynomial,
// the rest with the MUFU ex2.approx, so both pipes share the exponentials.
#ifndef QATTN_POLY_PER8
#define QATTN_POLY_PER8 2
#endif
constexpr int kPolyPer8 = QATTN_POLY_PER8;
constexpr float kMagic = 12582912.0f;   // 1.5 * 2^23: x + kMagic rounds x to an integer
// Score bias.  Before each QK the tensor core writes kSBias = 16 * 888^2 =
// 12616704 = 2^23 + 0x408400 into S (one BF16 MMA, K = 16, every operand element
// 888.0, an exact FP32 sum), and the INT8 MMAs then add the INT32 score S onto
// those bits.  The mantissa field 0x408400 + S stays inside [0, 2^23) for
// -4228096 <= S < 4160512, which holds every score of INT8 codes in [-127, 127]
// up to D = 256 (|S| <= 256 * 127 * 127 = 4129024), so the word read back as FP32
// is exactly kSBias + S: one subtraction recovers S, no integer-to-float conversion.
constexpr float kSBias = 12616704.0f;
constexpr uint32_t kSBiasRootBf16x2 = 0x445E445Eu;   // two BF16 888.0
// 2^f on [-1/2, 1/2], degree 5, relative minimax (fit_exp2.py), max relative error
// 2.3e-7 in FP32: about that of ex2.approx, so both paths round P to E4M3 alike.
constexpr float kC0 = 1.000000119e+00f, kC1 = 6.931469440e-01f, kC2 = 2.402212024e-01f,
                kC3 = 5.550713092e-02f, kC4 = 9.675540961e-03f, kC5 = 1.327647245e-03f;

// 2^t for two values at once: n = round(t), f = t - n, 2^t = poly(f) * 2^n with
// n added to the exponent field.  t is clamped at -126 so that the exponent of
// the result stays >= 0 (a tiny or subnormal positive value, never a wrap).
__device__ __forceinline__ float2 exp2_poly2(float2 t) {
  t.x = fmaxf(t.x, -126.0f);
  t.y = fmaxf(t.y, -126.0f);
  const float2 j = fadd2(t, make_float2(kMagic, kMagic));          // round to integer
  const float2 n = fadd2(j, make_float2(-kMagic, -kMagic));        // exact
  const float2 f = ffma2(n, make_float2(-1.0f, -1.0f), t);         // t - n, exact
  float2 q = ffma2(make_float2(kC5, kC5), f, make_float2(kC4, kC4));
  q = ffma2(q, f, make_float2(kC3, kC3));
  q = ffma2(q, f, make_float2(kC2, kC2));
  q = ffma2(q, f, make_float2(kC1, kC1));
  q = ffma2(q, f, make_float2(kC0, kC0));
  return make_float2(__uint_as_float(__float_as_uint(q.x) + (__float_as_uint(j.x) << 23)),
                     __uint_as_float(__float_as_uint(q.y) + (__float_as_uint(j.y) << 23)));
}

template <int J>
__device__ __forceinline__ float2 exp2_pair(float2 t) {
  if constexpr ((J % 8) < kPolyPer8) {
    return exp2_poly2(t);
  } else {
    return make_float2(ex2_approx(t.x), ex2_approx(t.y));
  }
}

// x[j] holds the exact FP32 score S_j; the exponent is fma(S_j, A, -mn).  Columns
// J .. END-1 of the row's N values, two at a time.
template <int J, int END, int N>
__device__ __forceinline__ void exp_block(float (&x)[N], float2 a2, float2 nb2) {
  if constexpr (J < END) {
    const float2 t = ffma2(make_float2(x[J], x[J + 1]), a2, nb2);
    const float2 e = exp2_pair<J>(t);
    x[J] = e.x;
    x[J + 1] = e.y;
    exp_block<J + 2, END>(x, a2, nb2);
  }
}

// Per-token K scales.  The warp stages the tile's score scales A_j = (q_scale *
// k_j) * c in shared memory (q_scale is the same for all rows of a warp); every
// lane reads the same addresses, a broadcast.  max_j S_j * A_j over all N keys
// (every key valid), four independent chains.
template <int N>
__device__ __forceinline__ float kt_tile_max(const float (&x)[N], const float* as) {
  float mq[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
  for (int j = 0; j < N; j += 4) {
    const float2 s01 = fmul2(make_float2(x[j], x[j + 1]), *reinterpret_cast<const float2*>(as + j));
    const float2 s23 = fmul2(make_float2(x[j + 2], x[j + 3]), *reinterpret_cast<const float2*>(as + j + 2));
    const int q = (j / 4) & 1;
    mq[q] = fmax3(mq[q], s01.x, s01.y);
    mq[2 + q] = fmax3(mq[2 + q], s23.x, s23.y);
  }
  return fmaxf(fmaxf(mq[0], mq[1]), fmaxf(mq[2], mq[3]));
}

// x[j] holds the exact FP32 score S_j; p_j = 2^fma(S_j, A_j, -mn), columns J .. END-1.
template <int J, int END, int N>
__device__ __forceinline__ void exp_block_kt(float (&x)[N], const float* as, float2 nb2) {
  if constexpr (J < END) {
    const float2 t = ffma2(make_float2(x[J], x[J + 1]), *reinterpret_cast<const float2*>(as + J), nb2);
    const float2 e = exp2_pair<J>(t);
    x[J] = e.x;
    x[J + 1] = e.y;
    exp_block_kt<J + 2, END>(x, as, nb2);
  }
}

// O <- O * o for this warp's 32 rows and NCOL columns of O (tensor memory), 64
// (or, for a 32-column block, 32) columns at a time.
template <int NCOL>
__device__ __forceinline__ void rescale_rows(uint32_t tO, float o) {
  constexpr int CH = (NCOL % 64 == 0) ? 64 : 32;
#pragma unroll 1
  for (int c0 = 0; c0 < NCOL; c0 += CH) {
    uint32_t r[CH];
#pragma unroll
    for (int c = 0; c < CH; c += 32)
      tmem_ld32(tO + c0 + c, *reinterpret_cast<uint32_t(*)[32]>(&r[c]));
    tmem_wait_ld();
#pragma unroll
    for (int j = 0; j < CH; j += 2) {
      const float2 v = fmul2(make_float2(__uint_as_float(r[j]), __uint_as_float(r[j + 1])),
                             make_float2(o, o));
      r[j] = __float_as_uint(v.x);
      r[j + 1] = __float_as_uint(v.y);
    }
#pragma unroll
    for (int c = 0; c < CH; c += 32)
      tmem_st32(tO + c0 + c, *reinterpret_cast<uint32_t(*)[32]>(&r[c]));
  }
}

// O <- O * o for the HALF O columns a thread owns in the two-threads-per-row
// layout (16x32bx2 accesses: threads 0-15 columns 0 .. HALF-1 of their lanes,
// threads 16-31 columns HALF .. 2 HALF-1), 32 columns at a time.
template <int HALF>
__device__ __forceinline__ void rescale_halves(uint32_t tO, float o) {
  static_assert(HALF % 64 == 0, "64-column round trips");
#pragma unroll 1
  for (int c0 = 0; c0 < HALF; c0 += 64) {           // two 32-column loads per round trip
    uint32_t r[64];
    tmem_ld16x2_x32<HALF>(tO + c0, *reinterpret_cast<uint32_t(*)[32]>(&r[0]));
    tmem_ld16x2_x32<HALF>(tO + c0 + 32, *reinterpret_cast<uint32_t(*)[32]>(&r[32]));
    tmem_wait_ld();
#pragma unroll
    for (int j = 0; j < 64; j += 2) {
      const float2 v = fmul2(make_float2(__uint_as_float(r[j]), __uint_as_float(r[j + 1])),
                             make_float2(o, o));
      r[j] = __float_as_uint(v.x);
      r[j + 1] = __float_as_uint(v.y);
    }
    tmem_st16x2_x32<HALF>(tO + c0, *reinterpret_cast<uint32_t(*)[32]>(&r[0]));
    tmem_st16x2_x32<HALF>(tO + c0 + 32, *reinterpret_cast<uint32_t(*)[32]>(&r[32]));
  }
}

// ------------------------------------------------------------------ host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

// 3-D uint8 tensor map with explicit pitches (bytes): extents {inner, rows, planes},
// row_pitch and plane_pitch multiples of 16; reads past an extent return zeros.
inline bool make_map_pitched(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows,
                             uint64_t planes, uint64_t row_pitch, uint64_t plane_pitch,
                             uint32_t box_inner, uint32_t box_rows, CUtensorMapSwizzle sw) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {inner, rows, planes};
  const cuuint64_t strides[2] = {row_pitch, plane_pitch};
  const cuuint32_t box[3] = {box_inner, box_rows, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D uint8 tensor map: dims {inner, rows, planes}, row pitch = inner bytes.
inline bool make_map(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint64_t planes,
              uint32_t box_inner, uint32_t box_rows, CUtensorMapSwizzle sw) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {inner, rows, planes};
  const cuuint64_t strides[2] = {inner, inner * rows};
  const cuuint32_t box[3] = {box_inner, box_rows, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace attn
}  // namespace qattn
