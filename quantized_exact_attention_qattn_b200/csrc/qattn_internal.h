// qattn_internal.h — launchers shared between the C-ABI layer and the kernel files.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/qattn.h"
#include "../../include/qattn_probe.h"

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
// qattn_api.cu: QATTN_OK on a compute capability 10.0 device, else a named refusal
qattn_status require_sm100();

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
                         cudaStream_t st, int k_rows = 64);
// Rotated INT8 V (V H/sqrt(D), per-channel scale amax/127), dim-major
// [B, Hkv, D, 64*ceil(Nkv/64)]; uses ws.vmax / ws.vfac.
cudaError_t launch_quant_v_rotated(int B, int Nkv, int Hkv, int D, BNHD v, QuantWorkspace ws,
                                   int8_t* v8t, float* v_scale, cudaStream_t st);
cudaError_t launch_hadamard_part(int B, int N, int H, int D, BNHD x, bool is_q, int8_t* x8,
                                 void* scale, int kcap, int key0, cudaStream_t st);
// FP16 V, dim-major [B, Hkv, D, cap]: source rows -> keys key0 .. key0 + n_write
cudaError_t launch_quant_v16(int B, int n_src, int Hkv, int D, BNHD v, int cap, int key0,
                             int n_write, uint16_t* v16t, cudaStream_t st);
// fused path: workspace = quant workspace, then BF16 cos / sin tables [N][R/2]
size_t prep_quant_table_bytes(int N, int rotary_dim);
cudaError_t launch_prep_quant(int B, int N, int Hq, int Hkv, int D, BNHD q, BNHD k, BNHD v,
                              const uint16_t* qw, const uint16_t* kw, float eps, int rotary_dim,
                              double theta, int64_t pos_offset, int8_t* q8, float* q_scale,
                              int8_t* k8, float* k_scale, float* k_mean, uint8_t* v8t,
                              float* v_scale, void* ws, cudaStream_t st);
cudaError_t launch_quant_hadamard(int B, int Nq, int Nkv, int Hq, int Hkv, int D, BNHD q,
                                  BNHD k, BNHD v, const float* vfac, int8_t* q8,
                                  float* q_scale, int8_t* k8, uint16_t* k_scale16,
                                  uint8_t* v8t, cudaStream_t st);

// attn_fwd.cu
// Test hook: K/V tile whose copy later attention launches skip (-1: none).
void set_stall_tile(int tile);
int stall_tile();

// Score copy-out requested by qattn_scores: n_tiles (b, h, q_tile, k_tile) quads
// (device, 16-byte aligned) and an INT32 [n_tiles][128][64] destination.
struct ScoreDump {
  const int32_t* tiles;
  int n_tiles;
  int32_t* s_out;
};

// One attention launch.  k8 rows and k_scale entries per (batch, KV head) are
// spaced kcap (>= Nkv) apart: kcap = Nkv for a plain problem, the allocated length
// for a cache of which the first Nkv keys are used.  pv 0: v = E4M3
// [B,Hkv,D,64*ceil(Nkv/64)] with v_scale; pv 1: v = FP16 [B,Hkv,D,kcap rounded up
// to 8], no scale.
// k_scale_mode 0: FP32 per 64 rows, 1: FP16 per token, 2: FP32 per 32 rows.
struct FwdLaunch {
  int B, Nq, Nkv, Hq, Hkv, D;
  const int8_t* q8;
  const float* q_scale;
  const int8_t* k8;
  const void* k_scale;
  int k_scale_mode;
  const void* v;
  const float* v_scale;
  int pv;
  int kcap;
  float c;             // log2(e) * softmax scale
  uint16_t* out;
  int* dev_err;
};

// dump == nullptr: the production kernel; otherwise its debug build that also
// copies the requested score tiles out.
cudaError_t launch_fwd(const FwdLaunch& L, const ScoreDump* dump, cudaStream_t st,
                       const char** why);

// tc_probe.cu
cudaError_t launch_tc_probe(int kind, int iters, int n_ctas, unsigned long long* cycles,
                            int* dev_err, cudaStream_t st);

}  // namespace qattn
