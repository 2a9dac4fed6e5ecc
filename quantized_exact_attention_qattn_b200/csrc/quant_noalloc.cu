// quant_noalloc.cu — qattn_quant without a caller-provided workspace.
//
// Some callers cannot allocate device memory at the point where they quantize:
// an embedder whose memory manager owns all device memory and hands out only the
// tensors themselves, or a runtime that must not allocate on its hot path because
// cudaMalloc and cudaFree can synchronize the device and stall every stream.  For
// them this entry point takes its reduction scratch (FP64 per-block K column
// sums, FP32 per-block V column maxima, FP32 V factors) from one statically sized
// device array compiled into this library instead of from a workspace argument.
//
// Properties:
//   * kNoallocScratchBytes (QATTN_NOALLOC_SCRATCH_BYTES, 16 MiB) is the limit;
//     problems needing more are refused with QATTN_ERR_WORKSPACE.
//   * The array is part of this library's device code: every device on which the
//     library's module gets loaded holds it until the process exits.
//   * All calls share the one array: calls whose kernels overlap on the GPU (two
//     streams, two threads) race on it.  Serialize them on one stream.
//   * Nothing in the scratch needs to start at zero: each byte a call reads was
//     written earlier in the same call, so the previous call's leftovers are
//     harmless and no clearing pass is needed.
//   * Host code cannot use the array's name as a device address (it names a
//     host-side stand-in).  The first call in each CUDA context looks the device
//     address up with cudaGetSymbolAddress (with the context's device current)
//     and caches it under the context's unique ID; make that first call before any
//     stream capture begins.  A context created later (after cudaDeviceReset, or
//     another context made current on the device) gets its own lookup on its
//     first call.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdio>
#include <mutex>

#include "qattn_internal.h"

namespace qattn {
namespace {

constexpr size_t kNoallocScratchBytes = QATTN_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

struct DriverFns {
  CtxGetCurrentFn get_current = nullptr;
  CtxGetIdFn get_id = nullptr;
};

DriverFns driver_fns() {
  static DriverFns fns;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fns.get_current = reinterpret_cast<CtxGetCurrentFn>(p);
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fns.get_id = reinterpret_cast<CtxGetIdFn>(p);
  });
  return fns;
}

// (context ID, scratch address) pairs; IDs are unique for the life of the process.
constexpr int kMaxContexts = 64;
std::mutex g_mu;
unsigned long long g_ctx_id[kMaxContexts] = {};
void* g_ctx_addr[kMaxContexts] = {};
int g_n_ctx = 0;

// Unique ID of the current context, or 0 when it cannot be read (no context yet,
// or a driver without the query): the caller then looks the address up afresh.
unsigned long long current_context_id() {
  const DriverFns f = driver_fns();
  if (!f.get_current || !f.get_id) return 0;
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (f.get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return 0;
  if (f.get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

// Device address of the static scratch in the current context.
cudaError_t scratch_address(void** out) {
  const unsigned long long id = current_context_id();
  std::lock_guard<std::mutex> lock(g_mu);
  if (id != 0) {
    for (int i = 0; i < g_n_ctx; ++i)
      if (g_ctx_id[i] == id) {
        *out = g_ctx_addr[i];
        return cudaSuccess;
      }
  }
  void* p = nullptr;
  // the runtime maps the symbol to this context's copy of the array (loading the
  // module here if it has not been loaded yet)
  const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
  if (e != cudaSuccess) return e;
  const unsigned long long id_now = id != 0 ? id : current_context_id();
  if (id_now != 0 && g_n_ctx < kMaxContexts) {
    g_ctx_id[g_n_ctx] = id_now;
    g_ctx_addr[g_n_ctx] = p;
    ++g_n_ctx;
  }
  *out = p;
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
  // the device check before the symbol lookup, so another device gets its refusal
  if (qattn_status s = qattn::require_sm100(); s != QATTN_OK) return s;
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
