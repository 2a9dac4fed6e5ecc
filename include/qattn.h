/*
 * qattn.h — C ABI of the B200 (sm_100a) quantized attention prefill library.
 *
 * The operation is the SageAttention-style INT8-QK / FP8-PV non-causal
 * attention whose numerics the page "Exact Numerical Contract" fixes:
 *   prep   : per-head Q/K RMSNorm + split-half RoPE        ("Preparation")
 *   quant  : exact K mean subtraction, INT8 Q (32-row groups), INT8 K (64-row
 *            blocks), FP8 E4M3 V with per-channel scales   ("Preparation" step 4,
 *            "Q And K Quantization", "V And PV")
 *   fwd    : INT8 QK^T, base-2 online softmax over 64-key tiles in order, FP8
 *            P.V, BF16 NHD output                          ("INT8 QK And Score
 *            Domain", "Online Softmax", "V And PV", "Finalization And Tails")
 * plus the per-head Walsh-Hadamard rotated int8-K variant of the page
 * "npu plan P7: int8 KV with per-head Hadamard rotation" (design note; PR #1273).
 *
 * Conventions shared by every entry point
 *   - Pointers marked (device) must point to device memory of the current CUDA
 *     device; the caller allocates and owns every buffer.  The library keeps no
 *     state between calls except one thread-local error string.
 *   - Calls are stream-ordered and asynchronous on `stream` (a cudaStream_t;
 *     NULL = legacy default stream).  Argument errors are reported synchronously
 *     and launch nothing.  A failed launch returns QATTN_ERR_CUDA.  A device-side
 *     bounded wait that gave up is reported through the caller's `dev_err` word
 *     (read it with qattn_check after the stream finishes).
 *   - BF16 is passed as uint16_t bit patterns, FP8 E4M3 as uint8_t, FP16 as
 *     uint16_t.  Inputs are finite; NaN/Inf behaviour is not part of the contract.
 *   - No entry point falls back to another implementation: an unsupported case
 *     returns a named refusal (the refusal convention of the "npu plan P7" page).
 */
#ifndef QATTN_H_
#define QATTN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  QATTN_OK = 0,
  QATTN_ERR_NULL = 1,        /* a required pointer is NULL                         */
  QATTN_ERR_SHAPE = 2,       /* a size is <= 0, too large, or inconsistent         */
  QATTN_ERR_STRIDE = 3,      /* last stride != 1, or a row / base not 16-B aligned */
  QATTN_ERR_UNSUPPORTED = 4, /* D not in {64,128,256}, bad rotary_dim, Hq % Hkv,
                                bad k_scale_mode, or a device that is not sm_100   */
  QATTN_ERR_WORKSPACE = 5,   /* workspace NULL or smaller than the query says      */
  QATTN_ERR_CUDA = 6,        /* a CUDA runtime/driver call failed                  */
  QATTN_ERR_TIMEOUT = 7      /* a device-side bounded wait gave up (via dev_err)   */
} qattn_status;

/* A strided BF16 view of logical shape [B, N, H, D].  stride[] are ELEMENT
 * strides of the four logical dims; stride[3] must be 1 and stride[0..2] and the
 * base address must keep every (b, n, h) row 16-byte aligned.  The canonical
 * interleaved QKV buffer of the "Canonical Boundary" section is three such views
 * of one [N, 21504] buffer at element offsets 0 / 7168 / 14336 with strides
 * {813066240, 21504, 128, 1}. */
typedef struct {
  const void* ptr;  /* (device) BF16 data */
  int64_t stride[4];
} qattn_bnhd;

/* ---------------------------------------------------------------- prep
 * Per-head RMSNorm then split-half RoPE on Q [B,N,Hq,D] and K [B,N,Hkv,D]
 * ("Exact Numerical Contract", "Preparation" steps 1-3).
 *   r   = 1/sqrt(mean(x^2) + eps), FP32 with IEEE sqrt/divide; the sum of squares
 *         is taken as D/8 lanes of 8 consecutive dims (left to right) then an XOR
 *         butterfly over lanes (D/16, ..., 2, 1)
 *   n   = bf16_rn(x*r);  y = bf16_rn(n * weight[d])   (weight [D], all heads)
 *   RoPE on dims [0, rotary_dim): pairs (i, i+R/2) with BF16 coefficients
 *         cos/sin(pos * theta^(-2i/R)) computed in FP64 and rounded once to BF16;
 *         y_i' = bf16_rn(y_i c - y_{i+R/2} s), y_{i+R/2}' = bf16_rn(y_{i+R/2} c + y_i s)
 *   pos = pos_offset + n.
 * Arguments
 *   q, k            strided BF16 inputs (device)
 *   q_weight, k_weight  BF16 [D] (device); NULL skips the norm of that tensor
 *   rotary_dim      0 (no RoPE) or a multiple of 16 with rotary_dim <= D
 *   q_out, k_out    contiguous BF16 [B,N,Hq,D] / [B,N,Hkv,D] (device)
 * D in {64,128,256}.  Errors: NULL, SHAPE, STRIDE, UNSUPPORTED, CUDA. */
qattn_status qattn_prep(int B, int N, int Hq, int Hkv, int D,
                        qattn_bnhd q, qattn_bnhd k,
                        const uint16_t* q_weight, const uint16_t* k_weight, float eps,
                        int rotary_dim, double rope_theta, int64_t pos_offset,
                        uint16_t* q_out, uint16_t* k_out, void* stream);

/* ---------------------------------------------------------------- quant
 * Bytes of device workspace qattn_quant / qattn_quant_hadamard need for a KV
 * sequence of Nkv rows: FP64 K column partials per 64-row block, FP32 V column
 * maxima per block and the FP32 V factors.  Returns 0 on invalid sizes. */
size_t qattn_quant_workspace_bytes(int B, int Nkv, int Hkv, int D);

/* Quantize prepared Q/K and raw V ("Preparation" step 4, "Q And K Quantization",
 * "V And PV").
 *   k_mean[b,h,d] = (float)( sum_j sum_{r in block j} k_r / N ), FP64, rows then
 *                   blocks ascending
 *   K: x = (float)k - k_mean (FP32); one scale per 64 rows; Q: one scale per 32
 *   rows inside 128-row tiles, G = 4*ceil(Nq/128) scales per (b,h):
 *       amax = max(1e-7f, max|x|); scale = amax/127.0f; q8 = rni_sat_s8(x*(127.0f/amax))
 *   (tail rows do not count; groups with no row get 1e-7f/127.0f)
 *   V: amax = max(1e-7f, max_n |v|) per (b,h,d); v_scale = amax/2.25f;
 *       v8 = e4m3_rn_satfinite(v * (2.25f/amax)), stored dim-major.
 * Arguments (all device)
 *   qp [B,Nq,Hq,D], kp [B,Nkv,Hkv,D], v [B,Nkv,Hkv,D]  strided BF16 views
 *   q8      int8 [B,Hq,Nq,D]            q_scale FP32 [B,Hq,4*ceil(Nq/128)]
 *   k8      int8 [B,Hkv,Nkv,D]          k_scale FP32 [B,Hkv,ceil(Nkv/64)]
 *   k_mean  FP32 [B,Hkv,D]
 *   v8t     E4M3 [B,Hkv,D,64*ceil(Nkv/64)] (keys contiguous; rows >= Nkv are 0)
 *   v_scale FP32 [B,Hkv,D]
 *   workspace, workspace_bytes: >= qattn_quant_workspace_bytes(B,Nkv,Hkv,D)
 * Hq % Hkv == 0.  Errors: NULL, SHAPE, STRIDE, UNSUPPORTED, WORKSPACE, CUDA. */
qattn_status qattn_quant(int B, int Nq, int Nkv, int Hq, int Hkv, int D,
                         qattn_bnhd qp, qattn_bnhd kp, qattn_bnhd v,
                         int8_t* q8, float* q_scale, int8_t* k8, float* k_scale,
                         float* k_mean, uint8_t* v8t, float* v_scale,
                         void* workspace, size_t workspace_bytes, void* stream);

/* Same as qattn_quant with one K scale per 32-row group instead of per 64-row
 * block: the finer grouping the page "npu plan P7" names for heads whose outliers
 * survive ("per-32-group scales at a small byte cost").  The K arithmetic is that
 * of qattn_quant over 32 rows (x = (float)k - k_mean, amax/127, rni_sat_s8);
 * k_scale is FP32 [B,Hkv,ceil(Nkv/32)].  Use qattn_fwd with k_scale_mode 2.
 * Other arguments, layouts and errors as qattn_quant. */
qattn_status qattn_quant_k32(int B, int Nq, int Nkv, int Hq, int Hkv, int D,
                             qattn_bnhd qp, qattn_bnhd kp, qattn_bnhd v,
                             int8_t* q8, float* q_scale, int8_t* k8, float* k_scale,
                             float* k_mean, uint8_t* v8t, float* v_scale,
                             void* workspace, size_t workspace_bytes, void* stream);

/* V for the FP16 P.V product (page "Fused FP8 PV preparation": FP16 PV is the
 * default, FP8 probabilities the option): v16 = fp16_rn(v) from BF16, no scale
 * (exact wherever |v| lies in FP16's normal range), stored dim-major like the FP8
 * V, keys contiguous: v16t FP16 [B,Hkv,D,capacity] (device), entries past Nkv
 * written as 0.  capacity >= Nkv, a multiple of 8.
 * Errors: NULL, SHAPE, STRIDE, UNSUPPORTED, CUDA. */
qattn_status qattn_quant_v16(int B, int Nkv, int Hkv, int D, qattn_bnhd v, uint16_t* v16t,
                             int capacity, void* stream);

/* ---------------------------------------------------------------- prep + quant, fused
 * qattn_prep followed by qattn_quant on the same self-attention inputs, in two
 * passes over HBM instead of four ("Exact Numerical Contract", "Preparation"
 * steps 1-4, "Q And K Quantization", "V And PV").  Every output is bit for bit
 * what qattn_prep -> qattn_quant give (the prepared BF16 Q and K are the same
 * values; they are only not stored):
 *   pass 1  raw Q, K, V read once: Q prepared and quantized per 32-row group in
 *           registers; K prepared and summed per 64-row block (FP64, rows
 *           ascending); V column maxima per block
 *   finalize  K mean (blocks ascending, FP64, / N, rounded once), V scales
 *   pass 2  raw K, V read again: K prepared again, mean subtracted, quantized per
 *           64-row block; V quantized to E4M3 and stored dim-major
 * The RoPE coefficients (the same FP64 -> BF16 values as qattn_prep, positions
 * pos_offset + n) are tabulated once per call into the workspace.
 * Arguments
 *   q [B,N,Hq,D], k and v [B,N,Hkv,D]   RAW strided BF16 views (device)
 *   q_weight, k_weight, eps, rotary_dim, rope_theta, pos_offset   as qattn_prep
 *   q8, q_scale, k8, k_scale, k_mean, v8t, v_scale   as qattn_quant (Nq = Nkv = N)
 *   workspace   device, 256-byte aligned, >= qattn_prep_quant_workspace_bytes(...)
 * Errors: NULL, SHAPE, STRIDE, UNSUPPORTED, WORKSPACE, CUDA. */
size_t qattn_prep_quant_workspace_bytes(int B, int N, int Hkv, int D, int rotary_dim);
qattn_status qattn_prep_quant(int B, int N, int Hq, int Hkv, int D,
                              qattn_bnhd q, qattn_bnhd k, qattn_bnhd v,
                              const uint16_t* q_weight, const uint16_t* k_weight, float eps,
                              int rotary_dim, double rope_theta, int64_t pos_offset,
                              int8_t* q8, float* q_scale, int8_t* k8, float* k_scale,
                              float* k_mean, uint8_t* v8t, float* v_scale,
                              void* workspace, size_t workspace_bytes, void* stream);

/* Hadamard-rotated variant ("npu plan P7" page: rotate Q and K by the same
 * per-head Walsh-Hadamard H, store K int8 with one FP16 scale per (head, token)).
 *   x' = FWHT(x) / sqrt(D) in FP32 (Sylvester order, no sign vector; stages
 *        h = 1, 2, ..., D/2 mapping (a, b) -> (a+b, a-b)); D in {64, 256}
 *   Q': INT8 per 32-row group as qattn_quant;  no K mean
 *   K': amax = max(1e-7f, max_d |k'|) per token; k_scale_f16 = fp16_rn(amax/127.0f);
 *       k8 = rni_sat_s8(k' * (127.0f/amax))
 *   V : as qattn_quant.
 * k_scale_f16 is FP16 [B,Hkv,Nkv] (device).  Use qattn_fwd with k_scale_mode 1.
 * Errors: as qattn_quant. */
qattn_status qattn_quant_hadamard(int B, int Nq, int Nkv, int Hq, int Hkv, int D,
                                  qattn_bnhd q, qattn_bnhd k, qattn_bnhd v,
                                  int8_t* q8, float* q_scale, int8_t* k8,
                                  uint16_t* k_scale_f16, uint8_t* v8t, float* v_scale,
                                  void* workspace, size_t workspace_bytes, void* stream);

/* Same computation as qattn_quant, for callers that cannot allocate device
 * memory when they quantize: an embedder whose memory manager owns all device
 * memory and hands out only the tensors, or a runtime that must not allocate on
 * its hot path because cudaMalloc / cudaFree can synchronize the device.  The
 * pages have no counterpart: it is an interface choice of this library, not part
 * of the method.
 * The scratch lives in one static device array of QATTN_NOALLOC_SCRATCH_BYTES
 * (16 MiB) compiled into the library; every device on which the library's module
 * is loaded holds it until the process exits.  Problems whose
 * qattn_quant_workspace_bytes exceeds that are refused with QATTN_ERR_WORKSPACE.
 * All calls share the array, so calls that overlap on the GPU (other streams or
 * threads) race: serialize them.  No scratch byte needs clearing between calls
 * (each call writes every byte it reads).  The first call in each CUDA context
 * looks up the array's device address (cudaGetSymbolAddress) and caches it under
 * the context's unique ID; make that first call before any stream capture, and
 * again first after a cudaDeviceReset.
 * Arguments, layouts and errors otherwise as qattn_quant. */
#define QATTN_NOALLOC_SCRATCH_BYTES ((size_t)16 << 20)
qattn_status qattn_quant_noalloc(int B, int Nq, int Nkv, int Hq, int Hkv, int D,
                                 qattn_bnhd qp, qattn_bnhd kp, qattn_bnhd v,
                                 int8_t* q8, float* q_scale, int8_t* k8, float* k_scale,
                                 float* k_mean, uint8_t* v8t, float* v_scale, void* stream);

/* ---------------------------------------------------------------- fwd
 * Fused attention ("INT8 QK And Score Domain", "Online Softmax", "V And PV",
 * "Finalization And Tails").  Per query row, over 64-key tiles t = 0, 1, ... in
 * order, with m = -5e6f, d = 1.0f, O = 0 initially:
 *   S_j  = Q8 K8^T exact in INT32
 *   A_j  = (q_scale * k_scale_j) * c  (FP32), c = (float)(log2(e) * sm_scale)
 *   s_j  = S_j * A_j (FP32); keys >= Nkv are masked (p_j = 0)
 *   mn   = max(m, max_j s_j - 8.807f); old = 2^(m - mn); d *= old; O *= old
 *   p_j  = 2^fma(S_j, A_j, -mn) (the exponent rounded once); d += p_j (FP32,
 *          unquantized); P8 = e4m3_rn_satfinite(p_j)
 *   O   += P8 . V8 (tcgen05 FP8 MMA, FP32 accumulation in tensor memory); m = mn
 *   out  = bf16_rn(O * rcp(d) * v_scale[d]), query rows < Nq only.
 * 2^x is ex2.approx or an FMA-pipe polynomial of equal accuracy; the sums run in
 * FP32 in an order of the kernel's own (within the output tolerance).
 * Arguments (all device except scalars)
 *   q8, q_scale, k8, v8t, v_scale  as produced by qattn_quant / _hadamard
 *   k_scale       k_scale_mode 0: FP32 [B,Hkv,ceil(Nkv/64)];
 *                 k_scale_mode 1: FP16 [B,Hkv,Nkv] (per token);
 *                 k_scale_mode 2: FP32 [B,Hkv,ceil(Nkv/32)] (per 32-row group,
 *                 qattn_quant_k32; A_j takes key j's group scale)
 *   sm_scale      softmax scale; 0 means 1/sqrt(D)
 *   out           contiguous BF16 [B,Nq,Hq,D]
 *   dev_err       one int32 (device), caller-owned; the kernel ORs error bits into
 *                 it (0 = success); read it with qattn_check.
 * D in {64,128,256}; Hq % Hkv == 0; GQA head h reads KV head h / (Hq/Hkv).
 * Errors: NULL, SHAPE, UNSUPPORTED, CUDA (synchronous); TIMEOUT (via dev_err). */
qattn_status qattn_fwd(int B, int Nq, int Nkv, int Hq, int Hkv, int D,
                       const int8_t* q8, const float* q_scale,
                       const int8_t* k8, const void* k_scale, int k_scale_mode,
                       const uint8_t* v8t, const float* v_scale, float sm_scale,
                       uint16_t* out, int* dev_err, void* stream);

/* The FP16 P.V control of the page "Fused FP8 PV preparation": qattn_fwd with
 * the probabilities encoded as FP16 (P16 = fp16_rn(p), same softmax, maximum and
 * unquantized denominator) and V as FP16 from qattn_quant_v16, multiplied by
 * tcgen05 kind::f16 with FP32 accumulation in tensor memory; out = bf16_rn(O *
 * rcp(d)) (no V scale).
 *   k8, k_scale  as qattn_fwd, but the rows (and per-token scales) of one (batch,
 *                KV head) are kv_capacity apart: k8 [B,Hkv,kv_capacity,D],
 *                k_scale mode 0 [B,Hkv,ceil(cap/64)], mode 1 [B,Hkv,cap], mode 2
 *                [B,Hkv,ceil(cap/32)]; only the first Nkv keys are used
 *   v16t         FP16 [B,Hkv,D,vcap], vcap = kv_capacity rounded up to a multiple
 *                of 8 (device; qattn_quant_v16 with capacity vcap)
 *   kv_capacity  >= Nkv: Nkv for a plain problem, the allocated length of a key
 *                cache
 * Errors: as qattn_fwd; SHAPE for kv_capacity. */
qattn_status qattn_fwd_pv16(int B, int Nq, int Nkv, int Hq, int Hkv, int D,
                            const int8_t* q8, const float* q_scale,
                            const int8_t* k8, const void* k_scale, int k_scale_mode,
                            const uint16_t* v16t, int kv_capacity, float sm_scale,
                            uint16_t* out, int* dev_err, void* stream);

/* Rotated INT8 V (page "npu plan P7", P7c: "an int8 V needs an inverse transform
 * on the output that K does not").  qattn_quant_v_rotated:
 *   v' = FWHT(v)/sqrt(D) per token (as qattn_quant_hadamard's K; D in {64, 256});
 *   amax = max(1e-7f, max_n |v'|) per (b, h, channel); v_scale = amax/127.0f;
 *   v8 = rni_sat_s8(v' * (127.0f/amax)), stored dim-major like the FP8 V:
 *   v8t int8 [B,Hkv,D,64*ceil(Nkv/64)] (rows >= Nkv are 0), v_scale FP32 [B,Hkv,D]
 *   workspace as qattn_quant (qattn_quant_workspace_bytes).
 * qattn_fwd_int8v: qattn_fwd_pv16 with this V (D = 256): the INT8 tiles are
 * widened exactly to FP16 on the chip (no FP16 copy of V in HBM), P16 . V8
 * accumulates in FP32, and the output is rotated back:
 *   o' = O * rcp(d) * v_scale (per rotated channel);  out = bf16_rn(FWHT(o')/sqrt(D)).
 * Other arguments as qattn_fwd (k_scale_mode 0, 1 or 2).
 * Errors: as qattn_fwd / qattn_quant; UNSUPPORTED for D. */
qattn_status qattn_quant_v_rotated(int B, int Nkv, int Hkv, int D, qattn_bnhd v, int8_t* v8t,
                                   float* v_scale, void* workspace, size_t workspace_bytes,
                                   void* stream);
qattn_status qattn_fwd_int8v(int B, int Nq, int Nkv, int Hq, int Hkv, int D,
                             const int8_t* q8, const float* q_scale,
                             const int8_t* k8, const void* k_scale, int k_scale_mode,
                             const int8_t* v8t, const float* v_scale, float sm_scale,
                             uint16_t* out, int* dev_err, void* stream);

/* INT32 score tiles S = Q8 K8^T exactly as the attention mainloop computes them
 * ("INT8 QK And Score Domain"), for bit-exact checks of the path qattn_fwd runs.
 * This launches qattn_fwd's own kernel on the whole problem (same operands, same
 * TMA copies, same tcgen05 kind::i8 MMAs with Q read from tensor memory at D 128
 * and 256 and from shared memory at D 64, same score-bias MMA and recovery of the
 * INT32 value), built with one addition: when the softmax
 * warps have recovered the scores of a requested tile from tensor memory, they
 * also copy them out.  `out` receives the attention output as from qattn_fwd.
 *   tiles    int32 [n_tiles][4] = (b, h, q_tile, k_tile) (device, 16-byte
 *            aligned); q_tile indexes 128-row query tiles, k_tile 64-key tiles.
 *            Entries naming no tile of the problem leave their slot untouched.
 *   s_out    int32 [n_tiles][128][64] (device, 16-byte aligned); rows past Nq and
 *            keys past Nkv read as 0 (zero rows of the operands)
 *   n_tiles  1 .. QATTN_SCORES_MAX_TILES
 * Other arguments and errors as qattn_fwd; also NULL (tiles, s_out), SHAPE
 * (n_tiles), STRIDE (alignment).  A debugging aid: slower than qattn_fwd. */
#define QATTN_SCORES_MAX_TILES 65536
qattn_status qattn_scores(int B, int Nq, int Nkv, int Hq, int Hkv, int D,
                          const int8_t* q8, const float* q_scale,
                          const int8_t* k8, const void* k_scale, int k_scale_mode,
                          const uint8_t* v8t, const float* v_scale, float sm_scale,
                          const int32_t* tiles, int n_tiles, int32_t* s_out,
                          uint16_t* out, int* dev_err, void* stream);

/* ---------------------------------------------------------------- key cache
 * Chunked prefill into a persistent rotated int8 key cache (page "npu plan P7:
 * int8 KV with per-head Hadamard rotation": prefill in 1024/2048-token chunks
 * writes the KV in the contract the decode path reads; the design note's first
 * variant keeps K int8, rotated, with a per-token scale sidecar, and V in 16
 * bits; rotating Q by the same H leaves the scores unchanged, so K is never
 * un-rotated).  One (batch, KV head) plane of the cache holds `capacity` keys:
 *   k8_cache      int8 [B,Hkv,capacity,D]
 *   k_scale_cache FP16 [B,Hkv,capacity]     (per-token scales, as qattn_quant_hadamard)
 *   v16_cache     FP16 [B,Hkv,D,capacity]   (dim-major, as qattn_quant_v16)
 * qattn_kcache_append writes the n_new keys of one chunk at positions key0 ..
 * key0+n_new-1: K' = FWHT(k)/sqrt(D) then INT8 with one FP16 scale per token
 * (the arithmetic of qattn_quant_hadamard's K), V as FP16; the V slots up to
 * key0 + n_new rounded up to 8 are written (the padding as 0), nothing else.
 * key0 and capacity are multiples of 8, key0 + n_new rounded up to 8 <= capacity,
 * D in {64, 256}; k and v are the chunk's raw BF16 [B,n_new,Hkv,D] (device).
 * A query chunk then uses qattn_quant_q_hadamard (Q' = FWHT(q)/sqrt(D), INT8 per
 * 32-row group) and qattn_fwd_pv16 with Nkv = key0 + n_new, k_scale_mode 1 and
 * kv_capacity = capacity: attention over every key cached so far.
 * Errors: NULL, SHAPE, STRIDE, UNSUPPORTED, CUDA. */
qattn_status qattn_kcache_append(int B, int Hkv, int D, int n_new, int key0, int capacity,
                                 qattn_bnhd k, qattn_bnhd v, int8_t* k8_cache,
                                 uint16_t* k_scale_cache, uint16_t* v16_cache, void* stream);
qattn_status qattn_quant_q_hadamard(int B, int Nq, int Hq, int D, qattn_bnhd q, int8_t* q8,
                                    float* q_scale, void* stream);

/* ---------------------------------------------------------------- host to host
 * The whole path for inputs and output in HOST memory, overlapping PCIe with
 * compute.  The pages' problem is one call from BF16 Q/K/V to BF16 output; every
 * (batch, KV head) in it is independent (per-head RMSNorm, K mean, scales and
 * softmax), so this entry point cuts the KV heads into chunks of
 * kv_heads_per_chunk (each with its Hq/Hkv query heads) and streams them through
 * two device buffer sets in `workspace`: chunk c's Q/K/V go host -> device on
 * h2d_stream while chunk c-1 computes on its set's stream (qattn_prep_quant ->
 * qattn_fwd, or qattn_quant_hadamard -> qattn_fwd with k_scale_mode 1) and chunk
 * c-2's output goes device -> host on d2h_stream.  The result is the same as
 * those entry points give on the whole problem, bit for bit.  The pages have no
 * counterpart for the chunking: an interface choice of this library.
 * Arguments
 *   q, k, v       BF16 views of HOST memory (pinned, for the copies to overlap):
 *                 q [B,Nq,Hq,D], k and v [B,Nkv,Hkv,D], with stride[3] == 1 and
 *                 stride[2] == D (whole heads back to back in a row; the
 *                 interleaved QKV layout qualifies), rows 16-byte aligned
 *   q_weight, k_weight, eps, rotary_dim, rope_theta   as qattn_prep (device weights;
 *                 positions 0..N-1); unused when hadamard == 1
 *   hadamard      0: prep + qattn_quant (Nq must equal Nkv); 1: qattn_quant_hadamard
 *   sm_scale      as qattn_fwd
 *   out           HOST BF16 [B,Nq,Hq,D], contiguous, 16-byte aligned
 *   kv_heads_per_chunk  >= 1: the chunk size (values above Hkv mean one chunk);
 *                 with Hkv >= 8 * kv_heads_per_chunk the first two chunks are a
 *                 quarter and a half of it (the first copy is then short)
 *   workspace     device, 256-byte aligned, >= qattn_host_workspace_bytes(...)
 *   dev_err       as qattn_fwd (shared by all chunks)
 *   stream        compute stream of buffer set 0; when the call returns, all of
 *                 its work (copies and stream2 included) is ordered before
 *                 anything queued on `stream` later, so qattn_check(dev_err,
 *                 stream) ends it
 *   stream2       compute stream of buffer set 1 (NULL: `stream`): consecutive
 *                 chunks then overlap, the next one's kernels filling the SMs
 *                 the previous one's last wave leaves idle
 *   h2d_stream, d2h_stream   copy streams (NULL: use `stream`, no overlap)
 *                 stream2, h2d_stream and d2h_stream first wait for the work
 *                 already queued on `stream`
 * Ownership: the caller owns every buffer and the streams; the call creates and
 * releases its own CUDA events.  Errors: NULL, SHAPE, STRIDE, UNSUPPORTED,
 * WORKSPACE, CUDA, and those of the entry points it calls.  An error after the
 * first chunk was queued leaves `out` undefined (earlier chunks may still land). */
size_t qattn_host_workspace_bytes(int B, int Nq, int Nkv, int Hq, int Hkv, int D,
                                  int kv_heads_per_chunk);
qattn_status qattn_attention_host(int B, int Nq, int Nkv, int Hq, int Hkv, int D,
                                  qattn_bnhd q, qattn_bnhd k, qattn_bnhd v,
                                  const uint16_t* q_weight, const uint16_t* k_weight, float eps,
                                  int rotary_dim, double rope_theta, int hadamard, float sm_scale,
                                  uint16_t* out, int kv_heads_per_chunk, void* workspace,
                                  size_t workspace_bytes, int* dev_err, void* stream,
                                  void* stream2, void* h2d_stream, void* d2h_stream);

/* ---------------------------------------------------------------- status
 * Synchronize `stream`, read the device error word and map it: 0 -> QATTN_OK,
 * a timed-out wait -> QATTN_ERR_TIMEOUT; a CUDA error -> QATTN_ERR_CUDA. */
qattn_status qattn_check(const int* dev_err, void* stream);

/* ---------------------------------------------------------------- test hook
 * Failure-path test of the bounded waits (the pages have no counterpart).  After
 * this call, every qattn_fwd launch in the process skips the K/V copy of key tile
 * `kv_tile` (0-based, 64 keys each): the tensor-core and softmax waits on that
 * tile give up after about one second, every role drains its in-flight copies and
 * MMAs, the kernel returns, and qattn_check reports QATTN_ERR_TIMEOUT with the
 * error bits set.  The output of such a call is undefined; the CUDA context stays
 * usable.  kv_tile = -1 (the initial state) turns the hook off.  Process-wide and
 * not synchronized with launches in flight: for tests only.
 * Errors: SHAPE if kv_tile < -1. */
qattn_status qattn_debug_stall_kv_tile(int kv_tile);

/* Human-readable reason of the last non-OK status returned on this thread. */
const char* qattn_last_error(void);

/* Library version string. */
const char* qattn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* QATTN_H_ */
