// qattn_api.cu — the extern "C" boundary: argument validation, named refusals,
// workspace carving and kernel launches.  No computation happens on the host.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <string>

#include "qattn_internal.h"

namespace {

thread_local std::string g_last_error;

qattn_status fail(qattn_status s, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
qattn_status fail(qattn_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return s;
}

qattn_status cuda_fail(cudaError_t e, const char* where, const char* why = nullptr) {
  return fail(QATTN_ERR_CUDA, "%s: %s%s%s", where, cudaGetErrorString(e), why ? " — " : "",
              why ? why : "");
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool supported_d(int D) { return D == 64 || D == 128 || D == 256; }

// Refuse devices other than compute capability 10.0 (the sm_100a cubin runs nowhere else).
qattn_status check_device() {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  int major = 0, minor = 0;
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
  if (major != 10 || minor != 0)
    return fail(QATTN_ERR_UNSUPPORTED, "device %d is sm_%d%d; this library is built for sm_100a",
                dev, major, minor);
  return QATTN_OK;
}

qattn_status check_view(const char* name, const qattn_bnhd& v) {
  if (v.ptr == nullptr) return fail(QATTN_ERR_NULL, "%s: null data pointer", name);
  if (v.stride[3] != 1) return fail(QATTN_ERR_STRIDE, "%s: the head-dim stride must be 1", name);
  if (!aligned16(v.ptr)) return fail(QATTN_ERR_STRIDE, "%s: base not 16-byte aligned", name);
  for (int i = 0; i < 3; ++i)
    if (v.stride[i] % 8 != 0)
      return fail(QATTN_ERR_STRIDE, "%s: stride[%d]=%lld keeps rows off 16-byte boundaries", name,
                  i, static_cast<long long>(v.stride[i]));
  return QATTN_OK;
}

qattn_status check_sizes(int B, int Nq, int Nkv, int Hq, int Hkv, int D) {
  if (B <= 0 || Nq <= 0 || Nkv <= 0 || Hq <= 0 || Hkv <= 0 || D <= 0)
    return fail(QATTN_ERR_SHAPE, "sizes must be positive (B=%d Nq=%d Nkv=%d Hq=%d Hkv=%d D=%d)", B,
                Nq, Nkv, Hq, Hkv, D);
  if (!supported_d(D)) return fail(QATTN_ERR_UNSUPPORTED, "head dim %d not in {64,128,256}", D);
  if (Hq % Hkv != 0)
    return fail(QATTN_ERR_UNSUPPORTED, "Hq=%d is not a multiple of Hkv=%d", Hq, Hkv);
  // every kernel indexes with 32-bit grid sizes and 64-bit element offsets
  const long long rows_q = static_cast<long long>(B) * Hq * ((Nq + 127) / 128);
  const long long rows_k = static_cast<long long>(B) * Hkv * ((Nkv + 63) / 64);
  if (rows_q > (1ll << 30) || rows_k > (1ll << 30) || static_cast<long long>(B) * Nkv > (1ll << 31))
    return fail(QATTN_ERR_SHAPE, "problem too large for one call");
  return QATTN_OK;
}

#define QATTN_TRY(x)                  \
  do {                                \
    qattn_status _s = (x);            \
    if (_s != QATTN_OK) return _s;    \
  } while (0)

}  // namespace

void qattn::set_last_error(const char* msg) { g_last_error = msg; }

qattn_status qattn::require_sm100() { return check_device(); }

extern "C" {

const char* qattn_version(void) { return "qattn-b200 0.1.0 (sm_100a)"; }

const char* qattn_last_error(void) { return g_last_error.c_str(); }

qattn_status qattn_prep(int B, int N, int Hq, int Hkv, int D, qattn_bnhd q, qattn_bnhd k,
                        const uint16_t* q_weight, const uint16_t* k_weight, float eps,
                        int rotary_dim, double rope_theta, int64_t pos_offset, uint16_t* q_out,
                        uint16_t* k_out, void* stream) {
  QATTN_TRY(check_sizes(B, N, N, Hq, Hkv, D));
  QATTN_TRY(check_view("q", q));
  QATTN_TRY(check_view("k", k));
  if (q_out == nullptr || k_out == nullptr) return fail(QATTN_ERR_NULL, "prep: null output");
  if (!aligned16(q_out) || !aligned16(k_out) || (q_weight && !aligned16(q_weight)) ||
      (k_weight && !aligned16(k_weight)))
    return fail(QATTN_ERR_STRIDE, "prep: outputs and weights must be 16-byte aligned");
  if (rotary_dim < 0 || rotary_dim > D || rotary_dim % 16 != 0)
    return fail(QATTN_ERR_UNSUPPORTED, "rotary_dim=%d must be a multiple of 16 in [0, D=%d]",
                rotary_dim, D);
  if (rotary_dim > 0 && !(rope_theta > 0.0))
    return fail(QATTN_ERR_UNSUPPORTED, "rope_theta must be positive");
  if (!(eps >= 0.0f)) return fail(QATTN_ERR_UNSUPPORTED, "eps must be >= 0");
  QATTN_TRY(check_device());
  cudaError_t e = qattn::launch_prep(B, N, Hq, Hkv, D, qattn::to_bnhd(q), qattn::to_bnhd(k),
                                     q_weight, k_weight, eps, rotary_dim, rope_theta, pos_offset,
                                     q_out, k_out, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "qattn_prep launch");
  return QATTN_OK;
}

size_t qattn_quant_workspace_bytes(int B, int Nkv, int Hkv, int D) {
  if (B <= 0 || Nkv <= 0 || Hkv <= 0 || !supported_d(D)) return 0;
  return qattn::quant_workspace_bytes(B, Nkv, Hkv, D);
}

static qattn_status check_quant_common(int B, int Nq, int Nkv, int Hq, int Hkv, int D,
                                       int8_t* q8, float* q_scale, int8_t* k8, void* k_scale,
                                       uint8_t* v8t, float* v_scale, void* ws, size_t ws_bytes) {
  QATTN_TRY(check_sizes(B, Nq, Nkv, Hq, Hkv, D));
  if (!q8 || !q_scale || !k8 || !k_scale || !v8t || !v_scale)
    return fail(QATTN_ERR_NULL, "quant: null output pointer");
  if (!aligned16(q8) || !aligned16(k8) || !aligned16(v8t))
    return fail(QATTN_ERR_STRIDE, "quant: q8, k8 and v8t must be 16-byte aligned");
  if (ws == nullptr || !aligned16(ws)) return fail(QATTN_ERR_WORKSPACE, "quant: workspace is null or unaligned");
  const size_t need = qattn::quant_workspace_bytes(B, Nkv, Hkv, D);
  if (ws_bytes < need)
    return fail(QATTN_ERR_WORKSPACE, "quant: workspace of %zu bytes, %zu needed", ws_bytes, need);
  return QATTN_OK;
}

static qattn_status quant_common(int B, int Nq, int Nkv, int Hq, int Hkv, int D, qattn_bnhd qp,
                                 qattn_bnhd kp, qattn_bnhd v, int8_t* q8, float* q_scale,
                                 int8_t* k8, float* k_scale, float* k_mean, uint8_t* v8t,
                                 float* v_scale, void* workspace, size_t workspace_bytes,
                                 void* stream, int k_rows) {
  QATTN_TRY(check_quant_common(B, Nq, Nkv, Hq, Hkv, D, q8, q_scale, k8, k_scale, v8t, v_scale,
                               workspace, workspace_bytes));
  if (k_mean == nullptr) return fail(QATTN_ERR_NULL, "quant: null k_mean");
  QATTN_TRY(check_view("qp", qp));
  QATTN_TRY(check_view("kp", kp));
  QATTN_TRY(check_view("v", v));
  QATTN_TRY(check_device());
  auto st = static_cast<cudaStream_t>(stream);
  qattn::QuantWorkspace w = qattn::carve_workspace(workspace, B, Nkv, Hkv, D);
  const qattn::BNHD kv = qattn::to_bnhd(kp);
  cudaError_t e = qattn::launch_kv_stats(B, Nkv, Hkv, D, &kv, qattn::to_bnhd(v), w, k_mean,
                                         v_scale, st);
  if (e != cudaSuccess) return cuda_fail(e, "qattn_quant stats launch");
  e = qattn::launch_quant(B, Nq, Nkv, Hq, Hkv, D, qattn::to_bnhd(qp), kv, qattn::to_bnhd(v),
                          k_mean, w.vfac, q8, q_scale, k8, k_scale, v8t, st, k_rows);
  if (e != cudaSuccess) return cuda_fail(e, "qattn_quant launch");
  return QATTN_OK;
}

size_t qattn_prep_quant_workspace_bytes(int B, int N, int Hkv, int D, int rotary_dim) {
  if (B <= 0 || N <= 0 || Hkv <= 0 || !supported_d(D) || rotary_dim < 0 || rotary_dim > D ||
      rotary_dim % 16 != 0)
    return 0;
  return qattn::quant_workspace_bytes(B, N, Hkv, D) + qattn::prep_quant_table_bytes(N, rotary_dim);
}

qattn_status qattn_prep_quant(int B, int N, int Hq, int Hkv, int D, qattn_bnhd q, qattn_bnhd k,
                              qattn_bnhd v, const uint16_t* q_weight, const uint16_t* k_weight,
                              float eps, int rotary_dim, double rope_theta, int64_t pos_offset,
                              int8_t* q8, float* q_scale, int8_t* k8, float* k_scale,
                              float* k_mean, uint8_t* v8t, float* v_scale, void* workspace,
                              size_t workspace_bytes, void* stream) {
  QATTN_TRY(check_sizes(B, N, N, Hq, Hkv, D));
  QATTN_TRY(check_view("q", q));
  QATTN_TRY(check_view("k", k));
  QATTN_TRY(check_view("v", v));
  if (!q8 || !q_scale || !k8 || !k_scale || !k_mean || !v8t || !v_scale)
    return fail(QATTN_ERR_NULL, "prep_quant: null output pointer");
  if (!aligned16(q8) || !aligned16(k8) || !aligned16(v8t) || (q_weight && !aligned16(q_weight)) ||
      (k_weight && !aligned16(k_weight)))
    return fail(QATTN_ERR_STRIDE, "prep_quant: q8, k8, v8t and the weights must be 16-byte aligned");
  if (rotary_dim < 0 || rotary_dim > D || rotary_dim % 16 != 0)
    return fail(QATTN_ERR_UNSUPPORTED, "rotary_dim=%d must be a multiple of 16 in [0, D=%d]",
                rotary_dim, D);
  if (rotary_dim > 0 && !(rope_theta > 0.0))
    return fail(QATTN_ERR_UNSUPPORTED, "rope_theta must be positive");
  if (!(eps >= 0.0f)) return fail(QATTN_ERR_UNSUPPORTED, "eps must be >= 0");
  const size_t need = qattn_prep_quant_workspace_bytes(B, N, Hkv, D, rotary_dim);
  if (workspace == nullptr || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return fail(QATTN_ERR_WORKSPACE, "prep_quant: workspace is null or not 256-byte aligned");
  if (workspace_bytes < need)
    return fail(QATTN_ERR_WORKSPACE, "prep_quant: workspace of %zu bytes, %zu needed",
                workspace_bytes, need);
  QATTN_TRY(check_device());
  cudaError_t e = qattn::launch_prep_quant(B, N, Hq, Hkv, D, qattn::to_bnhd(q), qattn::to_bnhd(k),
                                           qattn::to_bnhd(v), q_weight, k_weight, eps, rotary_dim,
                                           rope_theta, pos_offset, q8, q_scale, k8, k_scale,
                                           k_mean, v8t, v_scale, workspace,
                                           static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "qattn_prep_quant launch");
  return QATTN_OK;
}

qattn_status qattn_quant(int B, int Nq, int Nkv, int Hq, int Hkv, int D, qattn_bnhd qp,
                         qattn_bnhd kp, qattn_bnhd v, int8_t* q8, float* q_scale, int8_t* k8,
                         float* k_scale, float* k_mean, uint8_t* v8t, float* v_scale,
                         void* workspace, size_t workspace_bytes, void* stream) {
  return quant_common(B, Nq, Nkv, Hq, Hkv, D, qp, kp, v, q8, q_scale, k8, k_scale, k_mean, v8t,
                      v_scale, workspace, workspace_bytes, stream, 64);
}

qattn_status qattn_quant_k32(int B, int Nq, int Nkv, int Hq, int Hkv, int D, qattn_bnhd qp,
                             qattn_bnhd kp, qattn_bnhd v, int8_t* q8, float* q_scale, int8_t* k8,
                             float* k_scale, float* k_mean, uint8_t* v8t, float* v_scale,
                             void* workspace, size_t workspace_bytes, void* stream) {
  return quant_common(B, Nq, Nkv, Hq, Hkv, D, qp, kp, v, q8, q_scale, k8, k_scale, k_mean, v8t,
                      v_scale, workspace, workspace_bytes, stream, 32);
}

qattn_status qattn_quant_hadamard(int B, int Nq, int Nkv, int Hq, int Hkv, int D, qattn_bnhd q,
                                  qattn_bnhd k, qattn_bnhd v, int8_t* q8, float* q_scale,
                                  int8_t* k8, uint16_t* k_scale_f16, uint8_t* v8t,
                                  float* v_scale, void* workspace, size_t workspace_bytes,
                                  void* stream) {
  QATTN_TRY(check_quant_common(B, Nq, Nkv, Hq, Hkv, D, q8, q_scale, k8, k_scale_f16, v8t,
                               v_scale, workspace, workspace_bytes));
  if (D != 64 && D != 256)
    return fail(QATTN_ERR_UNSUPPORTED,
                "Hadamard variant needs D in {64, 256} (1/sqrt(D) a power of two), got %d", D);
  QATTN_TRY(check_view("q", q));
  QATTN_TRY(check_view("k", k));
  QATTN_TRY(check_view("v", v));
  QATTN_TRY(check_device());
  auto st = static_cast<cudaStream_t>(stream);
  qattn::QuantWorkspace w = qattn::carve_workspace(workspace, B, Nkv, Hkv, D);
  cudaError_t e = qattn::launch_kv_stats(B, Nkv, Hkv, D, nullptr, qattn::to_bnhd(v), w, nullptr,
                                         v_scale, st);
  if (e != cudaSuccess) return cuda_fail(e, "qattn_quant_hadamard stats launch");
  e = qattn::launch_quant_hadamard(B, Nq, Nkv, Hq, Hkv, D, qattn::to_bnhd(q), qattn::to_bnhd(k),
                                   qattn::to_bnhd(v), w.vfac, q8, q_scale, k8, k_scale_f16, v8t,
                                   st);
  if (e != cudaSuccess) return cuda_fail(e, "qattn_quant_hadamard launch");
  return QATTN_OK;
}

static qattn_status fwd_common(int B, int Nq, int Nkv, int Hq, int Hkv, int D, const int8_t* q8,
                               const float* q_scale, const int8_t* k8, const void* k_scale,
                               int k_scale_mode, const void* v, const float* v_scale, int pv,
                               int kcap, float sm_scale, uint16_t* out, int* dev_err,
                               const qattn::ScoreDump* dump, void* stream, const char* what) {
  QATTN_TRY(check_sizes(B, Nq, Nkv, Hq, Hkv, D));
  if (!q8 || !q_scale || !k8 || !k_scale || !v || (pv == 0 && !v_scale) || !out || !dev_err)
    return fail(QATTN_ERR_NULL, "%s: null pointer argument", what);
  if (!aligned16(q8) || !aligned16(k8) || !aligned16(v) || !aligned16(out))
    return fail(QATTN_ERR_STRIDE, "%s: q8, k8, the V operand and out must be 16-byte aligned", what);
  if (k_scale_mode < 0 || k_scale_mode > 2)
    return fail(QATTN_ERR_UNSUPPORTED,
                "k_scale_mode %d (0: per 64 rows, 1: per token FP16, 2: per 32 rows)", k_scale_mode);
  if (kcap < Nkv)
    return fail(QATTN_ERR_SHAPE, "%s: kv_capacity %d must be >= Nkv=%d", what, kcap, Nkv);
  if (!(sm_scale >= 0.0f) || std::isinf(sm_scale))
    return fail(QATTN_ERR_UNSUPPORTED, "sm_scale must be finite and >= 0");
  QATTN_TRY(check_device());
  const double sc = (sm_scale == 0.0f) ? 1.0 / std::sqrt(static_cast<double>(D))
                                       : static_cast<double>(sm_scale);
  qattn::FwdLaunch L{};
  L.B = B; L.Nq = Nq; L.Nkv = Nkv; L.Hq = Hq; L.Hkv = Hkv; L.D = D;
  L.q8 = q8; L.q_scale = q_scale; L.k8 = k8; L.k_scale = k_scale; L.k_scale_mode = k_scale_mode;
  L.v = v; L.v_scale = v_scale; L.pv = pv; L.kcap = kcap;
  L.c = static_cast<float>(1.4426950408889634 * sc);   // log2(e) * scale
  L.out = out; L.dev_err = dev_err;
  const char* why = nullptr;
  cudaError_t e = qattn::launch_fwd(L, dump, static_cast<cudaStream_t>(stream), &why);
  if (e != cudaSuccess) return cuda_fail(e, what, why);
  return QATTN_OK;
}

qattn_status qattn_quant_q_hadamard(int B, int Nq, int Hq, int D, qattn_bnhd q, int8_t* q8,
                                    float* q_scale, void* stream) {
  QATTN_TRY(check_sizes(B, Nq, Nq, Hq, Hq, D));
  if (D != 64 && D != 256)
    return fail(QATTN_ERR_UNSUPPORTED,
                "Hadamard variant needs D in {64, 256} (1/sqrt(D) a power of two), got %d", D);
  QATTN_TRY(check_view("q", q));
  if (!q8 || !q_scale) return fail(QATTN_ERR_NULL, "quant_q_hadamard: null output");
  if (!aligned16(q8)) return fail(QATTN_ERR_STRIDE, "quant_q_hadamard: q8 must be 16-byte aligned");
  QATTN_TRY(check_device());
  cudaError_t e = qattn::launch_hadamard_part(B, Nq, Hq, D, qattn::to_bnhd(q), true, q8, q_scale, 0,
                                              0, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "qattn_quant_q_hadamard launch");
  return QATTN_OK;
}

qattn_status qattn_kcache_append(int B, int Hkv, int D, int n_new, int key0, int capacity,
                                 qattn_bnhd k, qattn_bnhd v, int8_t* k8_cache,
                                 uint16_t* k_scale_cache, uint16_t* v16_cache, void* stream) {
  QATTN_TRY(check_sizes(B, n_new, n_new, Hkv, Hkv, D));
  if (D != 64 && D != 256)
    return fail(QATTN_ERR_UNSUPPORTED,
                "Hadamard variant needs D in {64, 256} (1/sqrt(D) a power of two), got %d", D);
  QATTN_TRY(check_view("k", k));
  QATTN_TRY(check_view("v", v));
  if (!k8_cache || !k_scale_cache || !v16_cache)
    return fail(QATTN_ERR_NULL, "kcache_append: null cache pointer");
  if (!aligned16(k8_cache) || !aligned16(v16_cache))
    return fail(QATTN_ERR_STRIDE, "kcache_append: k8_cache and v16_cache must be 16-byte aligned");
  const long long n_write = 8ll * ((n_new + 7) / 8);
  if (key0 < 0 || key0 % 8 != 0 || capacity % 8 != 0 || key0 + n_write > capacity)
    return fail(QATTN_ERR_SHAPE,
                "kcache_append: key0=%d must be a multiple of 8 and key0 + %lld (n_new rounded up "
                "to 8) <= capacity=%d (a multiple of 8)", key0, n_write, capacity);
  QATTN_TRY(check_device());
  auto st = static_cast<cudaStream_t>(stream);
  cudaError_t e = qattn::launch_hadamard_part(B, n_new, Hkv, D, qattn::to_bnhd(k), false, k8_cache,
                                              k_scale_cache, capacity, key0, st);
  if (e != cudaSuccess) return cuda_fail(e, "qattn_kcache_append K launch");
  e = qattn::launch_quant_v16(B, n_new, Hkv, D, qattn::to_bnhd(v), capacity, key0,
                              static_cast<int>(n_write), v16_cache, st);
  if (e != cudaSuccess) return cuda_fail(e, "qattn_kcache_append V launch");
  return QATTN_OK;
}

qattn_status qattn_fwd(int B, int Nq, int Nkv, int Hq, int Hkv, int D, const int8_t* q8,
                       const float* q_scale, const int8_t* k8, const void* k_scale,
                       int k_scale_mode, const uint8_t* v8t, const float* v_scale,
                       float sm_scale, uint16_t* out, int* dev_err, void* stream) {
  return fwd_common(B, Nq, Nkv, Hq, Hkv, D, q8, q_scale, k8, k_scale, k_scale_mode, v8t, v_scale,
                    0, Nkv, sm_scale, out, dev_err, nullptr, stream, "qattn_fwd");
}

qattn_status qattn_fwd_pv16(int B, int Nq, int Nkv, int Hq, int Hkv, int D, const int8_t* q8,
                            const float* q_scale, const int8_t* k8, const void* k_scale,
                            int k_scale_mode, const uint16_t* v16t, int kv_capacity,
                            float sm_scale, uint16_t* out, int* dev_err, void* stream) {
  return fwd_common(B, Nq, Nkv, Hq, Hkv, D, q8, q_scale, k8, k_scale, k_scale_mode, v16t, nullptr,
                    1, kv_capacity, sm_scale, out, dev_err, nullptr, stream, "qattn_fwd_pv16");
}

qattn_status qattn_fwd_int8v(int B, int Nq, int Nkv, int Hq, int Hkv, int D, const int8_t* q8,
                             const float* q_scale, const int8_t* k8, const void* k_scale,
                             int k_scale_mode, const int8_t* v8t, const float* v_scale,
                             float sm_scale, uint16_t* out, int* dev_err, void* stream) {
  if (D != 256)
    return fail(QATTN_ERR_UNSUPPORTED, "qattn_fwd_int8v: rotated INT8 V needs D = 256, got %d", D);
  return fwd_common(B, Nq, Nkv, Hq, Hkv, D, q8, q_scale, k8, k_scale, k_scale_mode, v8t, v_scale,
                    2, Nkv, sm_scale, out, dev_err, nullptr, stream, "qattn_fwd_int8v");
}

qattn_status qattn_quant_v_rotated(int B, int Nkv, int Hkv, int D, qattn_bnhd v, int8_t* v8t,
                                   float* v_scale, void* workspace, size_t workspace_bytes,
                                   void* stream) {
  QATTN_TRY(check_sizes(B, Nkv, Nkv, Hkv, Hkv, D));
  if (D != 64 && D != 256)
    return fail(QATTN_ERR_UNSUPPORTED,
                "Hadamard variant needs D in {64, 256} (1/sqrt(D) a power of two), got %d", D);
  QATTN_TRY(check_view("v", v));
  if (!v8t || !v_scale) return fail(QATTN_ERR_NULL, "quant_v_rotated: null output");
  if (!aligned16(v8t)) return fail(QATTN_ERR_STRIDE, "quant_v_rotated: v8t must be 16-byte aligned");
  if (workspace == nullptr || !aligned16(workspace))
    return fail(QATTN_ERR_WORKSPACE, "quant_v_rotated: workspace is null or unaligned");
  const size_t need = qattn::quant_workspace_bytes(B, Nkv, Hkv, D);
  if (workspace_bytes < need)
    return fail(QATTN_ERR_WORKSPACE, "quant_v_rotated: workspace of %zu bytes, %zu needed",
                workspace_bytes, need);
  QATTN_TRY(check_device());
  qattn::QuantWorkspace w = qattn::carve_workspace(workspace, B, Nkv, Hkv, D);
  cudaError_t e = qattn::launch_quant_v_rotated(B, Nkv, Hkv, D, qattn::to_bnhd(v), w, v8t, v_scale,
                                                static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "qattn_quant_v_rotated launch");
  return QATTN_OK;
}

qattn_status qattn_quant_v16(int B, int Nkv, int Hkv, int D, qattn_bnhd v, uint16_t* v16t,
                             int capacity, void* stream) {
  QATTN_TRY(check_sizes(B, Nkv, Nkv, Hkv, Hkv, D));
  QATTN_TRY(check_view("v", v));
  if (v16t == nullptr) return fail(QATTN_ERR_NULL, "quant_v16: null v16t");
  if (!aligned16(v16t)) return fail(QATTN_ERR_STRIDE, "quant_v16: v16t must be 16-byte aligned");
  if (capacity < Nkv || capacity % 8 != 0)
    return fail(QATTN_ERR_SHAPE, "quant_v16: capacity %d must be >= Nkv=%d and a multiple of 8",
                capacity, Nkv);
  QATTN_TRY(check_device());
  cudaError_t e = qattn::launch_quant_v16(B, Nkv, Hkv, D, qattn::to_bnhd(v), capacity, 0, capacity,
                                          v16t, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "qattn_quant_v16 launch");
  return QATTN_OK;
}

qattn_status qattn_scores(int B, int Nq, int Nkv, int Hq, int Hkv, int D, const int8_t* q8,
                          const float* q_scale, const int8_t* k8, const void* k_scale,
                          int k_scale_mode, const uint8_t* v8t, const float* v_scale,
                          float sm_scale, const int32_t* tiles, int n_tiles, int32_t* s_out,
                          uint16_t* out, int* dev_err, void* stream) {
  if (!tiles || !s_out) return fail(QATTN_ERR_NULL, "qattn_scores: null tiles or s_out");
  if (n_tiles <= 0 || n_tiles > QATTN_SCORES_MAX_TILES)
    return fail(QATTN_ERR_SHAPE, "qattn_scores: n_tiles=%d must be in [1, %d]", n_tiles,
                QATTN_SCORES_MAX_TILES);
  if (!aligned16(tiles) || !aligned16(s_out))
    return fail(QATTN_ERR_STRIDE, "qattn_scores: tiles and s_out must be 16-byte aligned");
  const qattn::ScoreDump dump{tiles, n_tiles, s_out};
  return fwd_common(B, Nq, Nkv, Hq, Hkv, D, q8, q_scale, k8, k_scale, k_scale_mode, v8t, v_scale,
                    0, Nkv, sm_scale, out, dev_err, &dump, stream, "qattn_scores");
}

qattn_status qattn_tc_probe(int kind, int iters, int n_ctas, unsigned long long* cycles,
                            int* dev_err, void* stream) {
  if (kind != 0 && kind != 1) return fail(QATTN_ERR_SHAPE, "tc_probe: kind %d (0: i8, 1: e4m3)", kind);
  if (iters < 1 || iters > (1 << 20)) return fail(QATTN_ERR_SHAPE, "tc_probe: iters must be in [1, 2^20]");
  if (n_ctas < 1 || n_ctas > (1 << 16)) return fail(QATTN_ERR_SHAPE, "tc_probe: n_ctas must be in [1, 2^16]");
  if (!cycles || !dev_err) return fail(QATTN_ERR_NULL, "tc_probe: null cycles or dev_err");
  QATTN_TRY(check_device());
  cudaError_t e = qattn::launch_tc_probe(kind, iters, n_ctas, cycles, dev_err,
                                         static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "qattn_tc_probe launch");
  return QATTN_OK;
}

qattn_status qattn_debug_stall_kv_tile(int kv_tile) {
  if (kv_tile < -1) return fail(QATTN_ERR_SHAPE, "debug_stall_kv_tile: tile must be >= -1");
  qattn::set_stall_tile(kv_tile);
  return QATTN_OK;
}

qattn_status qattn_check(const int* dev_err, void* stream) {
  if (dev_err == nullptr) return fail(QATTN_ERR_NULL, "check: null dev_err");
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  int h = 0;
  e = cudaMemcpy(&h, dev_err, sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "reading dev_err");
  if (h != 0) return fail(QATTN_ERR_TIMEOUT, "device wait timed out (error bits 0x%x)", h);
  return QATTN_OK;
}

}  // extern "C"
