// qattn_internal.h — launchers shared between the C-ABI layer and the kernel files.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/qattn.h"

namespace qattn {

struct BNHD {               // device-side strided BF16 view [B, N, H, D]
  const uint16_t* ptr;
  int64_t sb, sn, sh;       // element strides of B, N, H (D stride is 1)
};

inline BNHD to_bnhd(const qattn_bnhd& v) {
  return BNHD{static_cast<const uint16_t*>(v.ptr), v.stride[0], v.stride[1], v.stride[2]};
}

// qattn_api.cu: record the thread-local message returned by qattn_last_error()
void set_last_error(const char* msg);

// prep.cu
cudaError_t launch_prep(int B, int N, int Hq, int Hkv, int D, BNHD q, BNHD k,
                        const uint16_t* qw, const uint16_t* kw, float eps, int rotary_dim,
                        double theta, int64_t pos_offset, uint16_t* q_out, uint16_t* k_out,
                        cudaStream_t st);

// quant.cu
struct QuantWorkspace {
  double* ksum;     // [B, nK, Hkv*D] FP64 per-block column sums (may be null: no K mean)
  float* vmax;      // [B, nK, Hkv*D] FP32 per-block column |v| maxima
  float* vfac;      // [B, Hkv*D] FP32 V factor 2.25f/amax
};
size_t quant_workspace_bytes(int B, int Nkv, int Hkv, int D);
QuantWorkspace carve_workspace(void* ws, int B, int Nkv, int Hkv, int D);

cudaError_t launch_kv_stats(int B, int Nkv, int Hkv, int D, const BNHD* kp, BNHD v,
                            QuantWorkspace ws, float* k_mean, float* v_scale, cudaStream_t st);
cudaError_t launch_quant(int B, int Nq, int Nkv, int Hq, int Hkv, int D, BNHD qp, BNHD kp,
                         BNHD v, const float* k_mean, const float* vfac, int8_t* q8,
                         float* q_scale, int8_t* k8, float* k_scale, uint8_t* v8t,
                         cudaStream_t st);
cudaError_t launch_quant_hadamard(int B, int Nq, int Nkv, int Hq, int Hkv, int D, BNHD q,
                                  BNHD k, BNHD v, const float* vfac, int8_t* q8,
                                  float* q_scale, int8_t* k8, uint16_t* k_scale16,
                                  uint8_t* v8t, cudaStream_t st);

// attn_fwd.cu
// Test hook: K/V tile whose copy later attention launches skip (-1: none).
void set_stall_tile(int tile);
int stall_tile();

cudaError_t launch_fwd(int B, int Nq, int Nkv, int Hq, int Hkv, int D, const int8_t* q8,
                       const float* q_scale, const int8_t* k8, const void* k_scale,
                       int k_scale_mode, const uint8_t* v8t, const float* v_scale,
                       float score_c, uint16_t* out, int* dev_err, cudaStream_t st,
                       const char** why);
cudaError_t launch_scores(int B, int Nq, int Nkv, int Hq, int Hkv, int D, const int8_t* q8,
                          const int8_t* k8, const int32_t* tiles, int n_tiles, int32_t* s_out,
                          int* dev_err, cudaStream_t st, const char** why);

}  // namespace qattn
