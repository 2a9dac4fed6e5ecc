// tc_probe.cu — tensor-core throughput probe: the INT8 / FP8 peak that the
// attention mainloop's roofline fraction is reported against.
//
// One CTA per SM; one thread issues `iters` back-to-back tcgen05.mma of shape
// M128 N256 K32 (kind::i8: s8 x s8 -> s32, or kind::f8f6f4: e4m3 x e4m3 -> f32),
// both operands K-major in shared memory (128-byte swizzle), accumulating into 256
// tensor-memory columns, then waits for their completion.  Each MMA is 128 x 256
// x 32 multiply-adds, so a launch does n_ctas * iters * 2 * 128 * 256 * 32
// operations.  The operands hold fixed pseudo-random bytes (finite E4M3 codes for
// the FP8 kind).  The issuing thread also counts the SM cycles from its first
// issue to the completion it observes; the largest count over the CTAs is stored.
#include <cuda_runtime.h>

#include "qattn_device.cuh"
#include "qattn_internal.h"

namespace qattn {
namespace {

constexpr int kProbeM = 128, kProbeN = 256;
constexpr int kProbeA = kProbeM * 128;   // bytes: 128 rows x one 128-byte swizzle row
constexpr int kProbeB = kProbeN * 128;

template <int KIND>
__global__ void __launch_bounds__(128, 1)
tc_probe_kernel(int iters, unsigned long long* cycles, int* dev_err) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  __shared__ uint64_t bar;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_flag;
  const int warp = threadIdx.x >> 5;
  uint32_t* w = reinterpret_cast<uint32_t*>(smem);
  for (int i = threadIdx.x; i < (kProbeA + kProbeB) / 4; i += blockDim.x) {
    uint32_t x = static_cast<uint32_t>(i) * 2654435761u + 0x9E3779B9u;
    x ^= x >> 15;
    x *= 2246822519u;
    x ^= x >> 13;
    w[i] = KIND == 1 ? (x & 0x77777777u) : x;   // E4M3: exponent field <= 14, never NaN
  }
  fence_proxy_async_smem();
  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(&bar, 1);
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(&tmem_base_sh, kProbeN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  if (threadIdx.x == 32) {
    const uint64_t ad = smem_desc(smem_u32(smem), 8 * 128, 2u);
    const uint64_t bd = smem_desc(smem_u32(smem + kProbeA), 8 * 128, 2u);
    constexpr uint32_t idesc = KIND == 0 ? instr_desc(2, 1, kProbeM, kProbeN)
                                         : instr_desc(1, 0, kProbeM, kProbeN);
    const long long t0 = clock64();
    for (int it = 0; it < iters; ++it) {
      if constexpr (KIND == 0)
        mma_i8_ss(tmem, ad, bd, idesc, it > 0 ? 1u : 0u);
      else
        mma_f8_ss(tmem, ad, bd, idesc, it > 0 ? 1u : 0u);
    }
    tc_commit(&bar);
    // bounded: the MMAs take about iters * 128 cycles, far below the bound
    if (mbar_wait(&bar, 0, &abort_flag, dev_err, kErrTimeoutDrain))
      atomicMax(cycles, static_cast<unsigned long long>(clock64() - t0));
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kProbeN);
  }
}

}  // namespace

cudaError_t launch_tc_probe(int kind, int iters, int n_ctas, unsigned long long* cycles,
                            int* dev_err, cudaStream_t st) {
  const int smem = kProbeA + kProbeB + 1024;
  // at least 116 KB of shared memory: one CTA per SM
  const int smem_req = smem > 116 * 1024 ? smem : 116 * 1024;
  cudaError_t e = cudaMemsetAsync(cycles, 0, sizeof(unsigned long long), st);
  if (e != cudaSuccess) return e;
  if (kind == 0) {
    e = cudaFuncSetAttribute(tc_probe_kernel<0>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_req);
    if (e != cudaSuccess) return e;
    tc_probe_kernel<0><<<n_ctas, 128, smem_req, st>>>(iters, cycles, dev_err);
  } else {
    e = cudaFuncSetAttribute(tc_probe_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_req);
    if (e != cudaSuccess) return e;
    tc_probe_kernel<1><<<n_ctas, 128, smem_req, st>>>(iters, cycles, dev_err);
  }
  return cudaGetLastError();
}

}  // namespace qattn
