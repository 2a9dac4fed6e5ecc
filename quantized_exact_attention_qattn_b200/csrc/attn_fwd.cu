// attn_fwd.cu — fused INT8-QK / FP8-PV attention mainloop for sm_100a.
//
// Numerics: "Exact Numerical Contract", sections "INT8 QK And Score Domain",
// "Online Softmax", "V And PV", "Finalization And Tails".  Per query row and
// per 64-key tile t (ascending), S = Q8 K8^T exact in INT32:
//   A = (q_scale * k_scale) * c;  s = S * A          (FP32, c = log2(e) / sqrt(D))
//   mn = max(m, max(s) - 8.807);  old = ex2(m - mn);  d *= old;  O *= old
//   p = ex2(fma(S, A, -mn));  d += p;  P8 = e4m3(p);  O += P8 V8;  m = mn
//   out = bf16(O * rcp(d) * v_scale)
//
// Blackwell mapping (one CTA = NQT query tiles of 128 rows of one (b, h)):
//   warp 0      TMA producer: (D = 64) the Q tiles once, K/V tiles into a STAGES ring
//   warp 1+i    single-thread tcgen05.mma issuer of query tile i: QK^T as
//               kind::i8 (M=128, N=64, K=32 steps; for D >= 128 the Q tile is
//               operand A in TMEM, stored there once by the softmax warps) into
//               TMEM S[i] as soon as the softmax warps have read S[i], then P.V
//               (kind::f8f6f4 for FP8 P and V, kind::f16 for the FP16 variant) with
//               P read from TMEM, accumulating into TMEM O[i]
//   warps 4..   D <= 128: one 128-thread softmax warpgroup per query tile;
//               thread r owns query row r (TMEM lane r): tcgen05.ld of its 64
//               scores, the online-softmax update, tcgen05.st of its 64
//               probabilities, the O rescale of its row (only in warps where some
//               row's maximum moved, after the previous P.V completed), and the
//               final normalisation + BF16 store.  Each QK starts with a BF16
//               MMA that writes the FP32 bias kSBias = 16 * 888^2 into S and the INT8
//               MMAs accumulate onto its bits, so the scores read back as FP32
//               with one packed subtract per pair and no conversion, and the
//               reader releases S to the next QK right after its load.
//               D = 256: eight warps per query tile, two threads per row of the
//               same warp (16x32bx2 accesses): each owns 32 of the tile's keys and
//               half of the O columns, the row maximum is one shuffle between the
//               two, and each keeps a partial denominator added at the end.
// The query tiles' chains (two per CTA at D = 128, three at D = 64, where the
// smaller O leaves TMEM room for a third) are independent, so while one warpgroup
// runs the softmax of its tile the tensor core works for the others.  Every wait is
// bounded; a timeout sets a device error bit and all roles drain.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cmath>
#include <atomic>
#include <mutex>

#include "attn_common.cuh"

namespace qattn {

// Test hook (qattn_debug_stall_kv_tile): read at each attention launch.
static std::atomic<int> g_stall_tile{-1};
int stall_tile() { return g_stall_tile.load(); }

namespace {
using namespace attn;

constexpr int BN = 64;    // keys per tile ("Online Softmax": 64-key tiles)

// PV 0: FP8 E4M3 P and V (kind::f8f6f4), two P buffers of 16 columns per query
// tile; PV 1: FP16 P and V (kind::f16), one P buffer of 32 columns (the same
// tensor-memory columns) and V tiles of 64 keys x 2 bytes per dim row; PV 2 (D =
// 256): as PV 1, with V arriving as rotated INT8 in a staging buffer that two
// converter warps widen to the FP16 tile (exact), and the inverse rotation of the
// output in the epilogue.
template <int D, int NQT, int PV = 0>
struct Cfg {
  static constexpr int STAGES = (D == 256) ? 3 : 4;
  static constexpr int KCH = (D >= 128) ? 128 : 64;        // K-major swizzle row width (bytes)
  static constexpr int NCH = D / KCH;                       // column chunks per row
  static constexpr uint32_t SW_QK = (KCH == 128) ? 2u : 4u; // 128B or 64B swizzle
  static constexpr int Q_BYTES = BM * D;
  static constexpr int K_BYTES = BN * D;
  static constexpr int VB = PV ? 2 : 1;                     // bytes per V element in the MMA tile
  static constexpr int V_BYTES = D * BN * VB;
  static constexpr int VST_BYTES = (PV == 2) ? D * BN : 0;    // INT8 V staging (PV 2)
  // Q in tensor memory (A operand of QK read from TMEM, so each QK MMA reads only
  // its K tile from shared memory) wherever the columns allow: D = 128 with two
  // query tiles, D = 256 with one; D = 64 with three keeps Q in shared memory.
  static constexpr bool Q_TMEM = (D != 64);
  static constexpr int SMEM_Q = 0;
  static constexpr int SMEM_K = SMEM_Q + (Q_TMEM ? 0 : NQT * Q_BYTES);
  static constexpr int SMEM_V = SMEM_K + STAGES * K_BYTES;
  // Softmax layout: one thread per query row (one warpgroup per query tile), or,
  // for D = 256, two threads per row inside one warp (16x32bx2 tensor-memory
  // accesses), eight warps per query tile
  static constexpr bool HALVES = (D == 256);
  static constexpr int SM_WARPS = (HALVES ? 8 : 4) * NQT;           // softmax warps
  static constexpr int ARRIVALS = HALVES ? 8 : 4;                   // softmax warps per query tile
  static constexpr int SMEM_VST = SMEM_V + STAGES * V_BYTES;
  // The constant BF16 operand tile of the score-bias MMA that starts every QK (128
  // rows of 128 bytes, 128-byte swizzle; every element 888.0, so the layout does
  // not matter)
  static constexpr int SMEM_CB = SMEM_VST + STAGES * VST_BYTES;
  static constexpr int CB_BYTES = BM * 128;
  static constexpr int SMEM_KS = SMEM_CB + CB_BYTES;               // float [softmax warps][64]
  static constexpr int SMEM_BAR = SMEM_KS + SM_WARPS * BN * 4;
  static constexpr int N_BARS = 1 + 2 * STAGES + 8 * NQT + (PV == 2 ? STAGES : 0);
  static constexpr int SMEM_BYTES = SMEM_BAR + N_BARS * 8 + 16;
  // warps 0..: producer, one MMA issuer per query tile (then a spare warp or two),
  // then the softmax warps; any four consecutive warps cover the four TMEM lane
  // quadrants (warp % 4)
  static constexpr int SOFTMAX_WARP0 = 4;
  static constexpr int THREADS = 32 * (SOFTMAX_WARP0 + SM_WARPS);
  // tensor memory columns: O[NQT] (D each), S[NQT] (64 each), P[NQT][2] (16 each)
  static constexpr uint32_t O_COL = 0;
  static constexpr uint32_t S_COL = NQT * D;
  static constexpr uint32_t P_COL = S_COL + NQT * BN;
  static constexpr uint32_t Q_COL = P_COL + NQT * 2 * (BN / 4);   // Q[NQT] (D/4 each)
  static constexpr uint32_t TMEM_COLS = 512;
  static_assert(Q_COL + (Q_TMEM ? NQT * (D / 4) : 0) <= TMEM_COLS, "tensor memory budget");
  static constexpr uint32_t IDESC_QK = instr_desc(2, 1, BM, BN);   // s8 x s8 -> s32
  static constexpr uint32_t IDESC_SB = instr_desc(1, 1, BM, BN);   // bf16 x bf16 -> f32 (score bias)
  // e4m3 x e4m3 -> f32 (kind::f8f6f4) or f16 x f16 -> f32 (kind::f16): format code 0 both
  static constexpr uint32_t IDESC_PV = instr_desc(1, 0, BM, D);
};

// Bytes b0 .. b0+127 of query row n (head bh) into 32 tensor-memory columns at taddr
// (this warp's lanes), four bytes per column in order; rows past Nq are zero.
__device__ __forceinline__ void store_q_row(const FwdParams& p, int bh, int n, int D, int b0,
                                            uint32_t taddr) {
  uint32_t r[32];
  if (n < p.Nq) {
    const uint4* src =
        reinterpret_cast<const uint4*>(p.q8 + (static_cast<int64_t>(bh) * p.Nq + n) * D + b0);
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const uint4 v = __ldg(src + c);
      r[4 * c] = v.x;
      r[4 * c + 1] = v.y;
      r[4 * c + 2] = v.z;
      r[4 * c + 3] = v.w;
    }
  } else {
#pragma unroll
    for (int c = 0; c < 32; ++c) r[c] = 0u;
  }
  tmem_st32(taddr, r);
}

// DUMP: the debug build behind qattn_scores; it also copies the requested score
// tiles out as the softmax warps recover them (dump_scores), and is otherwise the
// same kernel.
template <int D, int NQT, int KMODE, bool DUMP, int PV>
__global__ void __launch_bounds__(Cfg<D, NQT, PV>::THREADS, 1)
attn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmV, const FwdParams p) {
  using C = Cfg<D, NQT, PV>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  float* ks_stage = reinterpret_cast<float*>(smem + C::SMEM_KS);   // per-token score scales A_j
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::SMEM_BAR);
  uint64_t* q_full = bars;
  uint64_t* kv_full = q_full + 1;
  uint64_t* kv_empty = kv_full + C::STAGES;
  // A parity wait for phase k is only sound if phase k-1 has completed and phase
  // k+1 cannot complete before the waiter is through.  P buffers, P-full and
  // PV-done are replicated per tile parity, [i][t & 1]: softmax writes P_i(t+2)
  // only after PV_i(t+1) (and so PV_i(t)) completed, PV_i(t+2) needs P_i(t+2),
  // and every waiter waits for every phase in order.  Every other barrier's next
  // phase depends on its waiter having passed.
  uint64_t* s_full = kv_empty + C::STAGES;   // MMA -> softmax: S_i(t) in TMEM
  uint64_t* s_free = s_full + NQT;           // softmax -> MMA: S_i read
  uint64_t* p_full = s_free + NQT;           // [NQT][2] softmax -> MMA: P_i(t) written, O_i rescaled
  uint64_t* pv_done = p_full + 2 * NQT;      // [NQT][2] MMA -> softmax: PV_i(t) done
  uint64_t* drain = pv_done + 2 * NQT;
  uint64_t* q_ready = drain + NQT;           // [NQT] softmax -> MMA: Q_i stored in tensor memory
  uint64_t* v_ready = q_ready + NQT;         // [STAGES] (PV 2) converters -> MMA: FP16 V tile written
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_flag;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  const int item = blockIdx.x;
  const int grp = item % p.n_groups;
  const int bh = item / p.n_groups;
  const int h = bh % p.Hq;
  const int b = bh / p.Hq;
  const int hkv = h / (p.Hq / p.Hkv);
  const int bhkv = b * p.Hkv + hkv;
  const int qt0 = grp * NQT;
  const int nvalid = min(NQT, p.nQ - qt0);
  const int nK = p.nK;

  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(q_full, 1);
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(kv_full + s, 1);
      mbar_init(kv_empty + s, nvalid);      // one commit per P.V issuer
    }
    for (int i = 0; i < NQT; ++i) {
      mbar_init(s_full + i, 1);
      for (int bb = 0; bb < 2; ++bb) {
        mbar_init(p_full + 2 * i + bb, C::ARRIVALS);   // one lane per softmax warp
        mbar_init(pv_done + 2 * i + bb, 1);
      }
      mbar_init(s_free + i, C::ARRIVALS);             // one lane per softmax warp
      mbar_init(q_ready + i, C::ARRIVALS);            // one lane per softmax warp
    }
    for (int i = 0; i < NQT; ++i) mbar_init(drain + i, 1);
    if constexpr (PV == 2)
      for (int s = 0; s < C::STAGES; ++s) mbar_init(v_ready + s, 2);   // two converter warps
    fence_barrier_init();
  }
  {   // operand tile of the score-bias MMA, read by the tensor core
    uint32_t* cb = reinterpret_cast<uint32_t*>(smem + C::SMEM_CB);
    for (int i = threadIdx.x; i < C::CB_BYTES / 4; i += C::THREADS) cb[i] = kSBiasRootBf16x2;
    fence_proxy_async_smem();
  }
  if (warp == 1) {
    tmem_alloc(&tmem_base_sh, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  volatile int* abort = &abort_flag;

  if (warp == 0) {
    // ================================================================ producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      if (!C::Q_TMEM) {
        mbar_arrive_expect_tx(q_full, static_cast<uint32_t>(nvalid * C::Q_BYTES));
        for (int i = 0; i < nvalid; ++i)
          for (int ch = 0; ch < C::NCH; ++ch)
            tma_load_3d(smem + C::SMEM_Q + i * C::Q_BYTES + ch * (BM * C::KCH), &tmQ, q_full,
                        ch * C::KCH, (qt0 + i) * BM, bh);
      }
      int issued = 0;
      for (int t = 0; t < nK; ++t) {
        const int s = t % C::STAGES;
        if (t >= C::STAGES &&
            !mbar_wait(kv_empty + s, ((t / C::STAGES) - 1) & 1, abort, p.dev_err, kErrTimeoutKV))
          break;
        if (t == p.stall_tile) {   // test hook: this stage's waiters time out
          issued = t + 1;
          continue;
        }
        mbar_arrive_expect_tx(kv_full + s, static_cast<uint32_t>(C::K_BYTES + (PV == 2 ? C::VST_BYTES : C::V_BYTES)));
        for (int ch = 0; ch < C::NCH; ++ch)
          tma_load_3d(smem + C::SMEM_K + s * C::K_BYTES + ch * (BN * C::KCH), &tmK, kv_full + s,
                      ch * C::KCH, t * BN, bhkv);
        if constexpr (PV == 2)   // INT8 tile into the staging buffer (unswizzled, 64 B rows)
          tma_load_3d(smem + C::SMEM_VST + s * C::VST_BYTES, &tmV, kv_full + s, t * BN, 0, bhkv);
        else
          tma_load_3d(smem + C::SMEM_V + s * C::V_BYTES, &tmV, kv_full + s, t * BN * C::VB, 0, bhkv);
        issued = t + 1;
      }
      int dummy = 0;      // drain: every issued copy must land before the CTA may exit
      if (!C::Q_TMEM) mbar_wait(q_full, 0, &dummy, p.dev_err, kErrTimeoutDrain);
      for (int u = max(0, issued - C::STAGES); u < issued; ++u)
        if (u != p.stall_tile)
          mbar_wait(kv_full + (u % C::STAGES), (u / C::STAGES) & 1, &dummy, p.dev_err,
                    kErrTimeoutDrain);
    }
  } else if (warp <= NQT) {
    // ================================================================ MMA issuers
    // One issuing thread per query tile i (warp 1 + i), so the two tiles' chains
    // never wait on each other: QK_i(t+1) as soon as S_i(t) has been read, then
    // PV_i(t) once the softmax warps have written P_i(t) and rescaled O_i.
    const int i = warp - 1;
    if (lane == 0 && i < nvalid) {
      const uint32_t sQ = smem_u32(smem + C::SMEM_Q) + i * C::Q_BYTES;
      const uint32_t sK = smem_u32(smem + C::SMEM_K);
      const uint32_t sV = smem_u32(smem + C::SMEM_V);
      const uint32_t tS = tmem + C::S_COL + i * BN;
      const uint32_t tO = tmem + C::O_COL + i * D;
      const uint64_t cbd = smem_desc(smem_u32(smem + C::SMEM_CB), 8 * 128, 2u);
      auto issue_qk = [&](int s) {
        // S <- kSBias first (overwrite), the INT8 steps then accumulate onto it
        mma_f16_ss(tS, cbd, cbd, C::IDESC_SB, 0u);
#pragma unroll
        for (int kk = 0; kk < D / 32; ++kk) {
          const int ch = (kk * 32) / C::KCH, off = (kk * 32) % C::KCH;
          const uint64_t bd = smem_desc(sK + s * C::K_BYTES + ch * (BN * C::KCH) + off,
                                        8 * C::KCH, C::SW_QK);
          if constexpr (C::Q_TMEM)   // Q_i row r in lane r, 4 bytes per column, 8 columns per K step
            mma_i8_ts(tS, tmem + C::Q_COL + i * (D / 4) + kk * 8, bd, C::IDESC_QK, 1u);
          else
            mma_i8_ss(tS, smem_desc(sQ + ch * (BM * C::KCH) + off, 8 * C::KCH, C::SW_QK), bd,
                      C::IDESC_QK, 1u);
        }
        tc_commit(s_full + i);
      };
      bool ok = (C::Q_TMEM ? mbar_wait(q_ready + i, 0, abort, p.dev_err, kErrTimeoutQ)
                           : mbar_wait(q_full, 0, abort, p.dev_err, kErrTimeoutQ)) &&
                mbar_wait(kv_full, 0, abort, p.dev_err, kErrTimeoutKV) &&
                mbar_wait(s_free + i, 0, abort, p.dev_err, kErrTimeoutS);
      if (ok) {
        tc_fence_after();
        issue_qk(0);
      }
      for (int t = 0; ok && t < nK; ++t) {
        const int s = t % C::STAGES;
        if (t + 1 < nK) {
          const int s1 = (t + 1) % C::STAGES;
          ok = mbar_wait(kv_full + s1, ((t + 1) / C::STAGES) & 1, abort, p.dev_err, kErrTimeoutKV) &&
               mbar_wait(s_free + i, (t + 1) & 1, abort, p.dev_err, kErrTimeoutS);
          if (!ok) break;
          tc_fence_after();
          issue_qk(s1);
        }
        ok = mbar_wait(p_full + 2 * i + (t & 1), (t >> 1) & 1, abort, p.dev_err, kErrTimeoutP);
        if (!ok) break;
        tc_fence_after();
        if constexpr (PV == 0) {   // P_i(t) in buffer t & 1; V rows of 64 keys, 64-byte swizzle
          const uint32_t a_tm = tmem + C::P_COL + (i * 2 + (t & 1)) * (BN / 4);
#pragma unroll
          for (int kk = 0; kk < BN / 32; ++kk) {
            const uint64_t bd = smem_desc(sV + s * C::V_BYTES + kk * 32, 8 * 64, 4u);
            mma_f8_ts(tO, a_tm + kk * 8, bd, C::IDESC_PV, (t > 0 || kk > 0) ? 1u : 0u);
          }
        } else {                   // one FP16 P buffer; V rows of 128 bytes, 128-byte swizzle
          if constexpr (PV == 2) {  // the converter warps have written this stage's FP16 V
            ok = mbar_wait(v_ready + s, (t / C::STAGES) & 1, abort, p.dev_err, kErrTimeoutKV);
            if (!ok) break;
            tc_fence_after();
          }
          const uint32_t a_tm = tmem + C::P_COL + i * (BN / 2);
#pragma unroll
          for (int kk = 0; kk < BN / 16; ++kk) {   // K = 16 FP16 (32 bytes, 8 columns) per MMA
            const uint64_t bd = smem_desc(sV + s * C::V_BYTES + kk * 32, 8 * 128, 2u);
            mma_f16_ts(tO, a_tm + kk * 8, bd, C::IDESC_PV, (t > 0 || kk > 0) ? 1u : 0u);
          }
        }
        tc_commit(pv_done + 2 * i + (t & 1));
        tc_commit(kv_empty + s);   // stage s is free once every issuer's reads finished
      }
      tc_commit(drain + i);        // drain: every issued tensor-core op before tear-down
      int dummy = 0;
      mbar_wait(drain + i, 0, &dummy, p.dev_err, kErrTimeoutDrain);
    }
    __syncwarp();
  } else if (PV == 2 && warp < C::SOFTMAX_WARP0) {
    // ================================================================ V converters (PV 2)
    // Warps NQT+1 and NQT+2 widen each stage's INT8 V tile (dims x 64 keys,
    // unswizzled) to the FP16 tile the P.V MMA reads (dims x 128 bytes, 128-byte
    // swizzle: 16-byte chunk c of row d at c ^ (d & 7)), half of the dims each.
    // b -> fp16: the bytes of (b ^ 0x80) under an exponent byte 0x64 are the FP16
    // value 1024 + b + 128; subtracting 1152 leaves b exactly.
    if constexpr (PV == 2) {
      const int cw = warp - (NQT + 1);
      const __half2 k1152 = __half2half2(__ushort_as_half(0x6480));
      for (int t = 0; t < nK; ++t) {
        const int s = t % C::STAGES;
        if (!__all_sync(0xffffffffu, mbar_wait(kv_full + s, (t / C::STAGES) & 1, abort, p.dev_err,
                                                kErrTimeoutKV)))
          break;
        const uint8_t* src = smem + C::SMEM_VST + s * C::VST_BYTES;
        uint8_t* dst = smem + C::SMEM_V + s * C::V_BYTES;
#pragma unroll 4
        for (int k = 0; k < (D / 2) * 8 / 32; ++k) {
          const int id = lane + 32 * k;
          const int d = cw * (D / 2) + (id >> 3), c = id & 7;
          const uint2 w = *reinterpret_cast<const uint2*>(src + d * BN + c * 8);
          uint32_t o[4];
          const uint32_t u0 = w.x ^ 0x80808080u, u1 = w.y ^ 0x80808080u;
          const uint32_t raw[4] = {__byte_perm(u0, 0x64646464u, 0x4140), __byte_perm(u0, 0x64646464u, 0x4342),
                                   __byte_perm(u1, 0x64646464u, 0x4140), __byte_perm(u1, 0x64646464u, 0x4342)};
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const __half2 hv = __hsub2(*reinterpret_cast<const __half2*>(&raw[q]), k1152);
            o[q] = *reinterpret_cast<const uint32_t*>(&hv);
          }
          *reinterpret_cast<uint4*>(dst + d * (BN * 2) + ((c ^ (d & 7)) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
        }
        fence_proxy_async_smem();                   // generic writes -> the tensor core's reads
        __syncwarp();
        if (lane == 0) mbar_arrive(v_ready + s);
      }
    }
  } else if (warp >= C::SOFTMAX_WARP0) {
    if constexpr (C::HALVES) {
      // ================================================================ softmax, two threads per row
      // Eight warps per query tile, two threads per row of the same warp.  Warp
      // slot s = 0..7 of tile i covers lanes 32 (s % 4) + 16 (s / 4) .. +15 (its
      // sub-partition's quadrant); of lane r's two threads, the first (thread r)
      // owns keys 0-31 of each tile and O columns 0 .. D/2-1, the second (thread
      // r + 16) keys 32-63 and O columns D/2 .. D-1 (16x32bx2 accesses).  The row's tile
      // maximum is one shuffle between the two; each keeps its own partial
      // denominator, added at the end.
      const int slot = warp - C::SOFTMAX_WARP0;
      const int i = slot >> 3;
      const int q4 = warp & 3;
      const int hb = (slot >> 2) & 1;
      const int kh = lane >> 4;
      const int row = q4 * 32 + hb * 16 + (lane & 15);
      if (i < nvalid) {
        const int qt = qt0 + i;
        const uint32_t lane_off = static_cast<uint32_t>(q4 * 32 + hb * 16) << 16;
        const uint32_t tS = tmem + lane_off + C::S_COL + i * BN;
        const uint32_t tP = tmem + lane_off + C::P_COL + (i * 2) * (BN / 4);
        const uint32_t tO = tmem + lane_off + C::O_COL + i * D;
        const float qs = p.q_scale[static_cast<int64_t>(bh) * p.G + qt * 4 + q4];
        const int last_valid = p.Nkv - (nK - 1) * BN;
        const float* ks32 = static_cast<const float*>(p.k_scale) + static_cast<int64_t>(bhkv) * p.ks_stride;
        const __half* ks16 = static_cast<const __half*>(p.k_scale) + static_cast<int64_t>(bhkv) * p.ks_stride;
        const int n_groups32 = (p.Nkv + 31) / 32;        // scales per 32-row group (mode 2)
        float m = kMInit;
        float den = (kh == 0) ? 1.0f : 0.0f;   // the two halves' partial sums add up to d
        float ks_next = (KMODE == 0) ? ks32[0] : 0.0f;
        // per-key scales: lane l holds those of tokens 2l, 2l+1 of a tile (0 past the
        // end): their own (mode 1) or their 32-row group's (mode 2)
        // The loads are issued a tile ahead into raw registers (predicated, nothing
        // depends on them until the next tile stages its scales): a conversion right
        // after the load would stall the warp for the load's whole latency.
        auto load_kraw = [&](int tt) {
          uint32_t a = 0, b = 0;
          if constexpr (KMODE == 2) {
            const int g = 2 * tt + (lane >> 4);
            if (g < n_groups32) a = __float_as_uint(__ldg(ks32 + g));
          } else {
            const int j = tt * BN + 2 * lane;
            const unsigned short* k16 = reinterpret_cast<const unsigned short*>(ks16);
            if (j < p.Nkv) a = __ldg(k16 + j);
            if (j + 1 < p.Nkv) b = __ldg(k16 + j + 1);
          }
          return make_uint2(a, b);
        };
        auto kraw_pair = [&](uint2 r) {
          if constexpr (KMODE == 2) {
            return make_float2(__uint_as_float(r.x), __uint_as_float(r.x));
          } else {
            return make_float2(__half2float(__ushort_as_half(static_cast<unsigned short>(r.x))),
                               __half2float(__ushort_as_half(static_cast<unsigned short>(r.y))));
          }
        };
        uint2 kraw_next = make_uint2(0u, 0u);
        if constexpr (KMODE != 0) kraw_next = load_kraw(0);
        {   // this thread's D/2 bytes of its Q row into tensor memory (D/8 columns)
          const int n = qt * BM + row;
          constexpr int QW = D / 8;                       // 32-bit words per thread
          uint32_t r[QW];
          if (n < p.Nq) {
            const uint4* src = reinterpret_cast<const uint4*>(
                p.q8 + (static_cast<int64_t>(bh) * p.Nq + n) * D + kh * (D / 2));
#pragma unroll
            for (int c = 0; c < QW / 4; ++c) {
              const uint4 v = __ldg(src + c);
              r[4 * c] = v.x;
              r[4 * c + 1] = v.y;
              r[4 * c + 2] = v.z;
              r[4 * c + 3] = v.w;
            }
          } else {
#pragma unroll
            for (int c = 0; c < QW; ++c) r[c] = 0u;
          }
          if constexpr (QW == 16)
            tmem_st16x2_x16<16>(tmem + lane_off + C::Q_COL + i * (D / 4), r);
          else
            tmem_st16x2_x32<32>(tmem + lane_off + C::Q_COL + i * (D / 4), r);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(q_ready + i);
          mbar_arrive(s_free + i);                  // s_free phase t: QK_i(t) may accumulate
        }
        bool ok = true;
        for (int t = 0; ok && t < nK; ++t) {
          const float ks_cur = ks_next;
          if (KMODE == 0 && t + 1 < nK) ks_next = ks32[t + 1];   // prefetch next tile's scale
          const uint2 kraw = kraw_next;
          if constexpr (KMODE != 0) {
            if (t + 1 < nK) kraw_next = load_kraw(t + 1);
          }
          ok = __all_sync(0xffffffffu, mbar_wait(s_full + i, t & 1, abort, p.dev_err, kErrTimeoutS));
          if (!ok) break;
          tc_fence_after();
          float x[32];                                    // keys 32 kh .. 32 kh + 31
          tmem_ld16x2_x32<32>(tS, *reinterpret_cast<uint32_t(*)[32]>(&x[0]));
          tmem_wait_ld();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(s_free + i);
          if constexpr (DUMP) dump_scores<32>(p, b, h, qt, t, row, kh * 32, x, kSBias);
          const bool last = (t == nK - 1);
          const int k0 = kh * 32;                         // first key of this half
          float mn;
          float2 a2, nb2;
          if constexpr (KMODE == 0) {
            if (last) {
#pragma unroll
              for (int j = 0; j < 32; ++j)
                if (k0 + j >= last_valid) x[j] = -INFINITY;   // masked key: p = 0
            }
            float mq[2];
#pragma unroll
            for (int q = 0; q < 2; ++q) {
              mq[q] = fmaxf(x[16 * q], x[16 * q + 15]);
#pragma unroll
              for (int j = 1; j < 15; j += 2) mq[q] = fmax3(mq[q], x[16 * q + j], x[16 * q + j + 1]);
            }
            float xmax = fmaxf(mq[0], mq[1]);
            xmax = fmaxf(xmax, __shfl_xor_sync(0xffffffffu, xmax, 16));   // the row's other half
#pragma unroll
            for (int j = 0; j < 32; j += 2) {
              const float2 sj = fadd2(make_float2(x[j], x[j + 1]), make_float2(-kSBias, -kSBias));
              x[j] = sj.x;
              x[j + 1] = sj.y;
            }
            const float a = __fmul_rn(__fmul_rn(qs, ks_cur), p.c);
            const float smax = __fmul_rn(__fsub_rn(xmax, kSBias), a);
            mn = fmaxf(m, __fsub_rn(smax, kFp8Offset));
            a2 = make_float2(a, a);
            nb2 = make_float2(-mn, -mn);
          } else {
            // per-token K scales: the warp stages the tile's 64 score scales
            // A_j = (q_scale * k_j) * c (two per lane); each half reads its own 32
            const int nv = last ? last_valid : BN;
            float* kss = ks_stage + slot * BN;
            *reinterpret_cast<float2*>(kss + 2 * lane) =
                fmul2(fmul2(make_float2(qs, qs), kraw_pair(kraw)), make_float2(p.c, p.c));
            __syncwarp();
#pragma unroll
            for (int j = 0; j < 32; j += 2) {
              const float2 sj = fadd2(make_float2(x[j], x[j + 1]), make_float2(-kSBias, -kSBias));
              x[j] = sj.x;
              x[j + 1] = sj.y;
            }
            float smx = -INFINITY;
            if (!last) {
              smx = kt_tile_max<32>(x, kss + k0);
            } else {
#pragma unroll
              for (int j = 0; j < 32; ++j)
                if (k0 + j < nv) smx = fmaxf(smx, __fmul_rn(x[j], kss[k0 + j]));
            }
            smx = fmaxf(smx, __shfl_xor_sync(0xffffffffu, smx, 16));
            mn = fmaxf(m, __fsub_rn(smx, kFp8Offset));
            nb2 = make_float2(-mn, -mn);
          }
          const float old = ex2_approx(__fsub_rn(m, mn));
          if constexpr (KMODE == 0) {
            exp_block<0, 32>(x, a2, nb2);
          } else {
            exp_block_kt<0, 32>(x, ks_stage + slot * BN + k0, nb2);
            __syncwarp();                                 // kss is rewritten next tile
            if (last) {
#pragma unroll
              for (int j = 0; j < 32; ++j)
                if (k0 + j >= last_valid) x[j] = 0.0f;    // masked key: p = 0
            }
          }
          // partial denominator: unquantized probabilities, four independent pair sums
          float2 acc[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) acc[q] = make_float2(x[2 * q], x[2 * q + 1]);
#pragma unroll
          for (int j = 8; j < 32; j += 8) {
#pragma unroll
            for (int q = 0; q < 4; ++q) acc[q] = fadd2(acc[q], make_float2(x[j + 2 * q], x[j + 2 * q + 1]));
          }
          acc[0] = fadd2(acc[0], acc[1]);
          acc[2] = fadd2(acc[2], acc[3]);
          acc[0] = fadd2(acc[0], acc[2]);
          den = __fadd_rn(__fmul_rn(den, old), __fadd_rn(acc[0].x, acc[0].y));
          uint32_t pk[PV ? 16 : 8];
          if constexpr (PV == 0) {
#pragma unroll
            for (int j = 0; j < 32; j += 4) pk[j / 4] = cvt_e4m3x4(x[j], x[j + 1], x[j + 2], x[j + 3]);
          } else {
#pragma unroll
            for (int j = 0; j < 32; j += 2) pk[j / 2] = cvt_f16x2(x[j], x[j + 1]);
          }
          if (t >= 1) {
            // PV_i(t-1) frees P buffer (t & 1), last read by PV_i(t-2), and must land
            // before this thread rescales its half of the row's O by old
            ok = __all_sync(0xffffffffu, mbar_wait(pv_done + 2 * i + ((t - 1) & 1), ((t - 1) >> 1) & 1,
                                                   abort, p.dev_err, kErrTimeoutO));
            if (!ok) break;
            tc_fence_after();
            if (__any_sync(0xffffffffu, old != 1.0f)) rescale_halves<D / 2>(tO, old);
          }
          if constexpr (PV == 0)
            tmem_st16x2_x8<8>(tP + (t & 1) * (BN / 4), pk);   // keys 32 kh .. : columns 8 kh ..
          else
            tmem_st16x2_x16<16>(tP, pk);                     // keys 32 kh .. : columns 16 kh ..
          tmem_wait_st();                                 // P and any O rescale have landed
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(p_full + 2 * i + (t & 1));
          m = mn;
        }
        // ---- finalize: O * rcp(d) * v_scale -> BF16, valid rows only ("Finalization")
        if (ok)
          ok = __all_sync(0xffffffffu, mbar_wait(pv_done + 2 * i + ((nK - 1) & 1), ((nK - 1) >> 1) & 1,
                                                 abort, p.dev_err, kErrTimeoutO));
        den = __fadd_rn(den, __shfl_xor_sync(0xffffffffu, den, 16));   // d = d_0 + d_1
        if (ok) {
          tc_fence_after();
          const float inv = rcp_approx(den);
          const int n = qt * BM + row;
          const float* vs = PV == 1 ? nullptr : p.v_scale + static_cast<int64_t>(bhkv) * D + kh * (D / 2);
          uint16_t* dst = p.out + ((static_cast<int64_t>(b) * p.Nq + n) * p.Hq + h) * D + kh * (D / 2);
          if constexpr (PV == 2) {
            // rotated V: o' = O * rcp(d) * v_scale (per rotated channel), then the
            // inverse rotation out = FWHT(o') / sqrt(D): stages h = 1 .. D/4 inside
            // this thread's D/2 columns, the last (h = D/2) against the row's other
            // thread, in the oracle's stage order
            constexpr int HC = D / 2;
            float o[HC];
#pragma unroll
            for (int c0 = 0; c0 < HC; c0 += 32) {
              uint32_t r[32];
              tmem_ld16x2_x32<HC>(tO + c0, r);
              tmem_wait_ld();
#pragma unroll
              for (int j = 0; j < 32; ++j)
                o[c0 + j] = __fmul_rn(__fmul_rn(__uint_as_float(r[j]), inv), vs[c0 + j]);
            }
#pragma unroll
            for (int hh = 1; hh < HC; hh <<= 1) {
#pragma unroll
              for (int k2 = 0; k2 < HC; ++k2) {
                if ((k2 & hh) == 0) {
                  const float a0 = o[k2], b0 = o[k2 + hh];
                  o[k2] = __fadd_rn(a0, b0);
                  o[k2 + hh] = __fsub_rn(a0, b0);
                }
              }
            }
            constexpr float kInvSqrtD = (D == 256) ? 0.0625f : 0.125f;   // exact
#pragma unroll
            for (int k2 = 0; k2 < HC; ++k2) {
              const float other = __shfl_xor_sync(0xffffffffu, o[k2], 16);
              o[k2] = __fmul_rn(kh == 0 ? __fadd_rn(o[k2], other) : __fsub_rn(other, o[k2]), kInvSqrtD);
            }
            if (n < p.Nq) {
#pragma unroll
              for (int c0 = 0; c0 < HC; c0 += 8) {
                uint32_t w4[4];
#pragma unroll
                for (int q = 0; q < 4; ++q)
                  w4[q] = static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(o[c0 + 2 * q]))) |
                          (static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(o[c0 + 2 * q + 1]))) << 16);
                *reinterpret_cast<uint4*>(dst + c0) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
              }
            }
          } else {
#pragma unroll 1
          for (int c0 = 0; c0 < D / 2; c0 += 32) {
            uint32_t o[32];
            tmem_ld16x2_x32<D / 2>(tO + c0, o);
            tmem_wait_ld();
            if (n < p.Nq) {
              uint32_t w[16];
#pragma unroll
              for (int j = 0; j < 32; j += 2) {
                float2 v = fmul2(make_float2(__uint_as_float(o[j]), __uint_as_float(o[j + 1])),
                                 make_float2(inv, inv));
                if constexpr (PV != 1) v = fmul2(v, make_float2(vs[c0 + j], vs[c0 + j + 1]));
                w[j / 2] = static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(v.x))) |
                           (static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(v.y))) << 16);
              }
              uint4* d4 = reinterpret_cast<uint4*>(dst + c0);
              d4[0] = make_uint4(w[0], w[1], w[2], w[3]);
              d4[1] = make_uint4(w[4], w[5], w[6], w[7]);
              d4[2] = make_uint4(w[8], w[9], w[10], w[11]);
              d4[3] = make_uint4(w[12], w[13], w[14], w[15]);
            }
          }
          }
        }
      }
    } else {
      // ================================================================ softmax
      const int wg = (warp - C::SOFTMAX_WARP0) >> 2;
      const int q4 = warp & 3;
      const int row = q4 * 32 + lane;
      if (wg < nvalid) {
        const int qt = qt0 + wg;
        const uint32_t lane_off = static_cast<uint32_t>(q4 * 32) << 16;
        const uint32_t tS = tmem + lane_off + C::S_COL + wg * BN;
        const uint32_t tP = tmem + lane_off + C::P_COL + (wg * 2) * (BN / 4);
        const uint32_t tO = tmem + lane_off + C::O_COL + wg * D;
        const float qs = p.q_scale[static_cast<int64_t>(bh) * p.G + qt * 4 + q4];
        const int last_valid = p.Nkv - (nK - 1) * BN;
        const float* ks32 = static_cast<const float*>(p.k_scale) + static_cast<int64_t>(bhkv) * p.ks_stride;
        const __half* ks16 = static_cast<const __half*>(p.k_scale) + static_cast<int64_t>(bhkv) * p.ks_stride;
        const int n_groups32 = (p.Nkv + 31) / 32;        // scales per 32-row group (mode 2)
        float m = kMInit, den = 1.0f;
        float ks_next = (KMODE == 0) ? ks32[0] : 0.0f;
        // per-key scales: lane l holds those of tokens 2l, 2l+1 of a tile (0 past the
        // end): their own (mode 1) or their 32-row group's (mode 2)
        // The loads are issued a tile ahead into raw registers (predicated, nothing
        // depends on them until the next tile stages its scales): a conversion right
        // after the load would stall the warp for the load's whole latency.
        auto load_kraw = [&](int tt) {
          uint32_t a = 0, b = 0;
          if constexpr (KMODE == 2) {
            const int g = 2 * tt + (lane >> 4);
            if (g < n_groups32) a = __float_as_uint(__ldg(ks32 + g));
          } else {
            const int j = tt * BN + 2 * lane;
            const unsigned short* k16 = reinterpret_cast<const unsigned short*>(ks16);
            if (j < p.Nkv) a = __ldg(k16 + j);
            if (j + 1 < p.Nkv) b = __ldg(k16 + j + 1);
          }
          return make_uint2(a, b);
        };
        auto kraw_pair = [&](uint2 r) {
          if constexpr (KMODE == 2) {
            return make_float2(__uint_as_float(r.x), __uint_as_float(r.x));
          } else {
            return make_float2(__half2float(__ushort_as_half(static_cast<unsigned short>(r.x))),
                               __half2float(__ushort_as_half(static_cast<unsigned short>(r.y))));
          }
        };
        uint2 kraw_next = make_uint2(0u, 0u);
        if constexpr (KMODE != 0) kraw_next = load_kraw(0);
        if constexpr (C::Q_TMEM) {   // this warp's rows of Q_i (D = 128: 32 columns)
          static_assert(!C::Q_TMEM || D == 128, "one 32-column store per row");
          store_q_row(p, bh, qt * BM + row, D, 0, tmem + lane_off + C::Q_COL + wg * (D / 4));
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(q_ready + wg);
        }
        // S arrives as kSBias + S (the issuer's bias MMA precedes each QK), read back
        // as FP32 exactly; one subtraction recovers S
        __syncwarp();
        if (lane == 0) mbar_arrive(s_free + wg);      // s_free phase t: QK_i(t) may write S
        bool ok = true;
        for (int t = 0; ok && t < nK; ++t) {
          float ks_cur = ks_next;
          if (KMODE == 0 && t + 1 < nK) ks_next = ks32[t + 1];   // prefetch next tile's scale
          const uint2 kraw = kraw_next;
          if constexpr (KMODE != 0) {
            if (t + 1 < nK) kraw_next = load_kraw(t + 1);
          }
          ok = __all_sync(0xffffffffu, mbar_wait(s_full + wg, t & 1, abort, p.dev_err, kErrTimeoutS));
          if (!ok) break;
          tc_fence_after();
          float x[64];
          tmem_ld32(tS, *reinterpret_cast<uint32_t(*)[32]>(&x[0]));
          tmem_ld32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&x[32]));
          tmem_wait_ld();                                 // S is in registers: release it
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(s_free + wg);
          if constexpr (DUMP) dump_scores<64>(p, b, h, qt, t, row, 0, x, kSBias);
          const bool last = (t == nK - 1);
          float mn;
          float2 a2, nb2;
          if constexpr (KMODE == 0) {
            // A = (q_scale * k_scale) * c; tile max of S*A from the max of S (A > 0)
            if (last) {
#pragma unroll
              for (int j = 0; j < 64; ++j)
                if (j >= last_valid) x[j] = -INFINITY;     // masked key: p = 2^-inf = 0
            }
            // four independent chains over 16 values each: 7 three-input maxima + 1
            float mq[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              mq[q] = fmaxf(x[16 * q], x[16 * q + 15]);
#pragma unroll
              for (int j = 1; j < 15; j += 2) mq[q] = fmax3(mq[q], x[16 * q + j], x[16 * q + j + 1]);
            }
            const float xmax = fmax3(mq[0], mq[1], fmaxf(mq[2], mq[3]));
#pragma unroll
            for (int j = 0; j < 64; j += 2) {
              const float2 sj = fadd2(make_float2(x[j], x[j + 1]), make_float2(-kSBias, -kSBias));
              x[j] = sj.x;
              x[j + 1] = sj.y;
            }
            const float a = __fmul_rn(__fmul_rn(qs, ks_cur), p.c);
            const float smax = __fmul_rn(__fsub_rn(xmax, kSBias), a);
            mn = fmaxf(m, __fsub_rn(smax, kFp8Offset));
            a2 = make_float2(a, a);
            nb2 = make_float2(-mn, -mn);
          } else {
            // per-token K scales: A_j = (q_scale * k_scale_j) * c; the exponent is
            // fma(S_j, A_j, -mn).  The warp stages the tile's 64 score scales A_j in
            // shared memory (two per lane, from the K scales fetched a tile ago).
            const int nv = last ? last_valid : BN;
            float* kss = ks_stage + (warp - C::SOFTMAX_WARP0) * BN;
            *reinterpret_cast<float2*>(kss + 2 * lane) =
                fmul2(fmul2(make_float2(qs, qs), kraw_pair(kraw)), make_float2(p.c, p.c));
            __syncwarp();
            // (every lane reads the same address: a broadcast, no bank conflict)
#pragma unroll
            for (int j = 0; j < 64; j += 2) {
              const float2 sj = fadd2(make_float2(x[j], x[j + 1]), make_float2(-kSBias, -kSBias));
              x[j] = sj.x;
              x[j + 1] = sj.y;
            }
            float smx = -INFINITY;
            if (!last) {
              smx = kt_tile_max<64>(x, kss);
            } else {
#pragma unroll
              for (int j = 0; j < 64; ++j)
                if (j < nv) smx = fmaxf(smx, __fmul_rn(x[j], kss[j]));
            }
            mn = fmaxf(m, __fsub_rn(smx, kFp8Offset));
            nb2 = make_float2(-mn, -mn);
          }
          const float old = ex2_approx(__fsub_rn(m, mn));
          if constexpr (KMODE == 0) {
            exp_block<0, 64>(x, a2, nb2);
          } else {
            exp_block_kt<0, 64>(x, ks_stage + (warp - C::SOFTMAX_WARP0) * BN, nb2);
            __syncwarp();                                 // kss is rewritten next tile
            if (last) {
#pragma unroll
              for (int j = 0; j < 64; ++j)
                if (j >= last_valid) x[j] = 0.0f;         // masked key: p = 0
            }
          }
          // denominator: unquantized probabilities, four independent pair sums
          float2 acc[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) acc[q] = make_float2(x[2 * q], x[2 * q + 1]);
#pragma unroll
          for (int j = 8; j < 64; j += 8) {
#pragma unroll
            for (int q = 0; q < 4; ++q) acc[q] = fadd2(acc[q], make_float2(x[j + 2 * q], x[j + 2 * q + 1]));
          }
          acc[0] = fadd2(acc[0], acc[1]);
          acc[2] = fadd2(acc[2], acc[3]);
          acc[0] = fadd2(acc[0], acc[2]);
          den = __fadd_rn(__fmul_rn(den, old), __fadd_rn(acc[0].x, acc[0].y));
          uint32_t pk[PV ? 32 : 16];
          if constexpr (PV == 0) {
#pragma unroll
            for (int j = 0; j < 64; j += 4) pk[j / 4] = cvt_e4m3x4(x[j], x[j + 1], x[j + 2], x[j + 3]);
          } else {
#pragma unroll
            for (int j = 0; j < 64; j += 2) pk[j / 2] = cvt_f16x2(x[j], x[j + 1]);
          }
          if (t >= 1) {
            // PV_i(t-1) was issued when this warpgroup finished tile t-1 and has long
            // completed.  Its completion frees P buffer (t & 1), last read by
            // PV_i(t-2), and lets this warp rescale its rows of O_i by old before
            // PV_i(t) accumulates (only if one of its 32 rows' maximum moved).
            ok = __all_sync(0xffffffffu, mbar_wait(pv_done + 2 * wg + ((t - 1) & 1), ((t - 1) >> 1) & 1,
                                                   abort, p.dev_err, kErrTimeoutO));
            if (!ok) break;
            tc_fence_after();
            if (__any_sync(0xffffffffu, old != 1.0f)) rescale_rows<D>(tO, old);
          }
          if constexpr (PV == 0)
            tmem_st16(tP + (t & 1) * (BN / 4), pk);
          else
            tmem_st32(tP, pk);
          tmem_wait_st();                                 // P and any O rescale have landed
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(p_full + 2 * wg + (t & 1));
          m = mn;
        }
        // ---- finalize: O * rcp(d) * v_scale -> BF16, valid rows only ("Finalization")
        if (ok)
          ok = __all_sync(0xffffffffu, mbar_wait(pv_done + 2 * wg + ((nK - 1) & 1), ((nK - 1) >> 1) & 1,
                                                 abort, p.dev_err, kErrTimeoutO));
        if (ok) {
          tc_fence_after();
          const float inv = rcp_approx(den);
          const int n = qt * BM + row;
          const float* vs = PV ? nullptr : p.v_scale + static_cast<int64_t>(bhkv) * D;
          uint16_t* dst = p.out + ((static_cast<int64_t>(b) * p.Nq + n) * p.Hq + h) * D;
#pragma unroll 1
          for (int c0 = 0; c0 < D; c0 += 32) {
            uint32_t o[32];
            tmem_ld32(tO + c0, o);
            tmem_wait_ld();
            if (n < p.Nq) {
              uint32_t w[16];
#pragma unroll
              for (int j = 0; j < 32; j += 2) {
                float2 v = fmul2(make_float2(__uint_as_float(o[j]), __uint_as_float(o[j + 1])),
                                 make_float2(inv, inv));
                if constexpr (PV != 1) v = fmul2(v, make_float2(vs[c0 + j], vs[c0 + j + 1]));
                w[j / 2] = static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(v.x))) |
                           (static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(v.y))) << 16);
              }
              uint4* d4 = reinterpret_cast<uint4*>(dst + c0);
              d4[0] = make_uint4(w[0], w[1], w[2], w[3]);
              d4[1] = make_uint4(w[4], w[5], w[6], w[7]);
              d4[2] = make_uint4(w[8], w[9], w[10], w[11]);
              d4[3] = make_uint4(w[12], w[13], w[14], w[15]);
            }
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// ------------------------------------------------------------------ host side
template <int D, int NQT, int KMODE, bool DUMP, int PV>
cudaError_t launch_fwd_t(const FwdLaunch& L, const ScoreDump& dump, cudaStream_t st,
                         const char** why) {
  using Cf = Cfg<D, NQT, PV>;
  const int nQ = (L.Nq + BM - 1) / BM;
  const int nK = (L.Nkv + BN - 1) / BN;
  const uint64_t BH = static_cast<uint64_t>(L.B) * L.Hkv;
  const CUtensorMapSwizzle swqk =
      (Cf::KCH == 128) ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  CUtensorMap mQ, mK, mV;
  bool ok = make_map(&mQ, L.q8, D, L.Nq, static_cast<uint64_t>(L.B) * L.Hq, Cf::KCH, BM, swqk) &&
            make_map_pitched(&mK, L.k8, D, L.Nkv, BH, D, static_cast<uint64_t>(D) * L.kcap, Cf::KCH,
                             BN, swqk);
  if (PV == 0)   // E4M3 [B,Hkv,D,64*nK]: rows past Nkv hold zeros
    ok = ok && make_map(&mV, L.v, static_cast<uint64_t>(nK) * BN, D, BH, BN, D,
                        CU_TENSOR_MAP_SWIZZLE_64B);
  else if (PV == 2)   // rotated INT8 [B,Hkv,D,64*nK] into the unswizzled staging buffer
    ok = ok && make_map(&mV, L.v, static_cast<uint64_t>(nK) * BN, D, BH, BN, D,
                        CU_TENSOR_MAP_SWIZZLE_NONE);
  else {         // FP16 [B,Hkv,D,vpitch]: keys past Nkv read as zeros (outside the extent)
    const uint64_t vpitch = 8 * ((static_cast<uint64_t>(L.kcap) + 7) / 8);
    ok = ok && make_map_pitched(&mV, L.v, static_cast<uint64_t>(L.Nkv) * 2, D, BH, vpitch * 2,
                                vpitch * 2 * D, BN * 2, D, CU_TENSOR_MAP_SWIZZLE_128B);
  }
  if (!ok) {
    *why = "cuTensorMapEncodeTiled failed (pointer alignment or size)";
    return cudaErrorInvalidValue;
  }
  FwdParams p{};
  p.q8 = L.q8; p.q_scale = L.q_scale; p.k_scale = L.k_scale; p.v_scale = L.v_scale; p.out = L.out;
  p.dev_err = L.dev_err;
  p.B = L.B; p.Nq = L.Nq; p.Nkv = L.Nkv; p.Hq = L.Hq; p.Hkv = L.Hkv;
  p.G = 4 * nQ; p.nK = nK; p.nQ = nQ; p.n_groups = (nQ + NQT - 1) / NQT;
  p.c = L.c;
  p.kcap = L.kcap;
  p.ks_stride = KMODE == 0 ? (L.kcap + 63) / 64 : (KMODE == 1 ? L.kcap : (L.kcap + 31) / 32);
  p.stall_tile = stall_tile();
  p.dump_tiles = reinterpret_cast<const int4*>(dump.tiles);
  p.dump_out = dump.s_out;
  p.n_dump = dump.n_tiles;
  // at least 116 KB so that one CTA (and one 512-column TMEM allocation) owns an SM
  const int smem = (Cf::SMEM_BYTES + 1024 > 116 * 1024) ? Cf::SMEM_BYTES + 1024 : 116 * 1024;
  cudaError_t e = cudaFuncSetAttribute(attn_fwd_kernel<D, NQT, KMODE, DUMP, PV>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const unsigned grid = static_cast<unsigned>(static_cast<int64_t>(L.B) * L.Hq * p.n_groups);
  attn_fwd_kernel<D, NQT, KMODE, DUMP, PV><<<grid, Cf::THREADS, smem, st>>>(mQ, mK, mV, p);
  return cudaGetLastError();
}

template <int D, int NQT, int KMODE>
cudaError_t launch_fwd_k(const FwdLaunch& L, const ScoreDump* dump, cudaStream_t st,
                         const char** why) {
  const ScoreDump none{nullptr, 0, nullptr};
  if (L.pv == 2) {
    if constexpr (D == 256) {
      if (dump != nullptr) {
        *why = "the score copy-out build exists for the FP8 P.V kernel only";
        return cudaErrorInvalidValue;
      }
      return launch_fwd_t<D, NQT, KMODE, false, 2>(L, none, st, why);
    } else {
      *why = "rotated INT8 V needs D = 256";
      return cudaErrorInvalidValue;
    }
  }
  if (L.pv == 1) {
    if (dump != nullptr) {
      *why = "the score copy-out build exists for the FP8 P.V kernel only";
      return cudaErrorInvalidValue;
    }
    return launch_fwd_t<D, NQT, KMODE, false, 1>(L, none, st, why);
  }
  if (dump == nullptr) return launch_fwd_t<D, NQT, KMODE, false, 0>(L, none, st, why);
  return launch_fwd_t<D, NQT, KMODE, true, 0>(L, *dump, st, why);
}

template <int D, int NQT>
cudaError_t launch_fwd_d(const FwdLaunch& L, const ScoreDump* dump, cudaStream_t st,
                         const char** why) {
  switch (L.k_scale_mode) {
    case 0: return launch_fwd_k<D, NQT, 0>(L, dump, st, why);
    case 1: return launch_fwd_k<D, NQT, 1>(L, dump, st, why);
    case 2: return launch_fwd_k<D, NQT, 2>(L, dump, st, why);
    default:
      *why = "k_scale_mode must be 0, 1 or 2";
      return cudaErrorInvalidValue;
  }
}

}  // namespace

void set_stall_tile(int tile) { g_stall_tile.store(tile); }

cudaError_t launch_fwd(const FwdLaunch& L, const ScoreDump* dump, cudaStream_t st,
                       const char** why) {
  switch (L.D) {
    case 64:   // three query tiles: O 192 + S 192 + P 96 of the 512 TMEM columns
      return launch_fwd_d<64, 3>(L, dump, st, why);
    case 128:
      return launch_fwd_d<128, 2>(L, dump, st, why);
    case 256:
      return launch_fwd_d<256, 1>(L, dump, st, why);
    default:
      *why = "head dimension must be 64, 128 or 256";
      return cudaErrorInvalidValue;
  }
}

}  // namespace qattn
