// quant_noalloc.cu — qattn_quant without a caller-provided workspace.
//
// Some callers cannot allocate device memory at the point where they quantize:
// code running inside a CUDA-graph capture (cudaMalloc is not capturable),
// allocators that forbid allocation on a hot path, or embedders whose memory
// manager owns every byte and only hands out the tensors themselves.  For them
// this entry point takes its reduction scratch (FP64 per-block K column sums,
// FP32 per-block V column maxima, FP32 V factors) from one statically sized
// device array compiled into this library instead of from a workspace argument.
//
// Properties:
//   * kNoallocScratchBytes (QATTN_NOALLOC_SCRATCH_BYTES, 16 MiB) is the limit;
//     problems needing more are refused with QATTN_ERR_WORKSPACE.
//   * Every device that uses it keeps the array resident until the process exits.
//   * All calls share the one array: calls whose kernels overlap on the GPU (two
//     streams, two threads) race on it.  Serialize them on one stream.
//   * Nothing in the scratch needs to start at zero: each byte a call reads was
//     written earlier in the same call, so the previous call's leftovers are
//     harmless and no clearing pass is needed.
//   * The first call on each device looks the array's device address up
//     (cudaGetSymbolAddress) and caches it; make that first call before any
//     stream capture begins.
#include <cuda_runtime.h>

#include <cstdio>
#include <mutex>
#include <string>

#include "qattn_internal.h"

namespace qattn {
namespace {

constexpr size_t kNoallocScratchBytes = QATTN_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of the static scratch on the current device (cached per device).
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    // host code must not use g_noalloc_scratch's name as an address: it is a
    // host-side shadow; the runtime maps it to this device's copy
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return cudaSuccess;
}

}  // namespace
}  // namespace qattn

extern "C" qattn_status qattn_quant_noalloc(int B, int Nq, int Nkv, int Hq, int Hkv, int D,
                                            qattn_bnhd qp, qattn_bnhd kp, qattn_bnhd v, int8_t* q8,
                                            float* q_scale, int8_t* k8, float* k_scale,
                                            float* k_mean, uint8_t* v8t, float* v_scale,
                                            void* stream) {
  // Size check first: it needs no device and reports the limit plainly.
  const size_t need = qattn_quant_workspace_bytes(B, Nkv, Hkv, D);
  if (need == 0) return qattn_quant(B, Nq, Nkv, Hq, Hkv, D, qp, kp, v, q8, q_scale, k8, k_scale,
                                    k_mean, v8t, v_scale, nullptr, 0, stream);  // names the bad size
  if (need > qattn::kNoallocScratchBytes) {
    char msg[256];
    snprintf(msg, sizeof(msg),
             "quant_noalloc: this problem needs %zu bytes of scratch, more than the %zu-byte "
             "static array; use qattn_quant with a workspace",
             need, qattn::kNoallocScratchBytes);
    qattn::set_last_error(msg);
    return QATTN_ERR_WORKSPACE;
  }
  void* scratch = nullptr;
  const cudaError_t e = qattn::scratch_address(&scratch);
  if (e != cudaSuccess) {
    char msg[256];
    snprintf(msg, sizeof(msg), "quant_noalloc: cudaGetSymbolAddress failed: %s",
             cudaGetErrorString(e));
    qattn::set_last_error(msg);
    return QATTN_ERR_CUDA;
  }
  // Same validation, kernels and launch order as qattn_quant, on the static scratch.
  return qattn_quant(B, Nq, Nkv, Hq, Hkv, D, qp, kp, v, q8, q_scale, k8, k_scale, k_mean, v8t,
                     v_scale, scratch, qattn::kNoallocScratchBytes, stream);
}
