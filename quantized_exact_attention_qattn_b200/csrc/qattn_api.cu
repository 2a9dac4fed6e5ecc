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

qattn_status qattn_quant(int B, int Nq, int Nkv, int Hq, int Hkv, int D, qattn_bnhd qp,
                         qattn_bnhd kp, qattn_bnhd v, int8_t* q8, float* q_scale, int8_t* k8,
                         float* k_scale, float* k_mean, uint8_t* v8t, float* v_scale,
                         void* workspace, size_t workspace_bytes, void* stream) {
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
                          k_mean, w.vfac, q8, q_scale, k8, k_scale, v8t, st);
  if (e != cudaSuccess) return cuda_fail(e, "qattn_quant launch");
  return QATTN_OK;
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

qattn_status qattn_fwd(int B, int Nq, int Nkv, int Hq, int Hkv, int D, const int8_t* q8,
                       const float* q_scale, const int8_t* k8, const void* k_scale,
                       int k_scale_mode, const uint8_t* v8t, const float* v_scale,
                       float sm_scale, uint16_t* out, int* dev_err, void* stream) {
  QATTN_TRY(check_sizes(B, Nq, Nkv, Hq, Hkv, D));
  if (!q8 || !q_scale || !k8 || !k_scale || !v8t || !v_scale || !out || !dev_err)
    return fail(QATTN_ERR_NULL, "fwd: null pointer argument");
  if (!aligned16(q8) || !aligned16(k8) || !aligned16(v8t) || !aligned16(out))
    return fail(QATTN_ERR_STRIDE, "fwd: q8, k8, v8t and out must be 16-byte aligned");
  if (k_scale_mode != 0 && k_scale_mode != 1)
    return fail(QATTN_ERR_UNSUPPORTED, "k_scale_mode %d (0: per 64 rows, 1: per token)", k_scale_mode);
  if (!(sm_scale >= 0.0f) || std::isinf(sm_scale))
    return fail(QATTN_ERR_UNSUPPORTED, "sm_scale must be finite and >= 0");
  QATTN_TRY(check_device());
  const double sc = (sm_scale == 0.0f) ? 1.0 / std::sqrt(static_cast<double>(D))
                                       : static_cast<double>(sm_scale);
  const float c = static_cast<float>(1.4426950408889634 * sc);   // log2(e) * scale
  const char* why = nullptr;
  cudaError_t e = qattn::launch_fwd(B, Nq, Nkv, Hq, Hkv, D, q8, q_scale, k8, k_scale,
                                    k_scale_mode, v8t, v_scale, c, out, dev_err,
                                    static_cast<cudaStream_t>(stream), &why);
  if (e != cudaSuccess) return cuda_fail(e, "qattn_fwd launch", why);
  return QATTN_OK;
}

qattn_status qattn_scores(int B, int Nq, int Nkv, int Hq, int Hkv, int D, const int8_t* q8,
                          const int8_t* k8, const int32_t* tiles, int n_tiles, int32_t* s_out,
                          int* dev_err, void* stream) {
  QATTN_TRY(check_sizes(B, Nq, Nkv, Hq, Hkv, D));
  if (!q8 || !k8 || !tiles || !s_out || !dev_err)
    return fail(QATTN_ERR_NULL, "scores: null pointer argument");
  if (n_tiles <= 0) return fail(QATTN_ERR_SHAPE, "scores: n_tiles must be positive");
  if (!aligned16(q8) || !aligned16(k8) || !aligned16(s_out))
    return fail(QATTN_ERR_STRIDE, "scores: q8, k8 and s_out must be 16-byte aligned");
  QATTN_TRY(check_device());
  const char* why = nullptr;
  cudaError_t e = qattn::launch_scores(B, Nq, Nkv, Hq, Hkv, D, q8, k8, tiles, n_tiles, s_out,
                                       dev_err, static_cast<cudaStream_t>(stream), &why);
  if (e != cudaSuccess) return cuda_fail(e, "qattn_scores launch", why);
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
