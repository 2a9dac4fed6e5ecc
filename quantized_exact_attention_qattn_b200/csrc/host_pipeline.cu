// host_pipeline.cu — the whole path (fused prep + quant -> fwd, or the Hadamard
// quant -> fwd) for inputs and output in host memory.  Every (batch, KV head) is
// an independent problem (per-head norms, means, scales and softmax), so the KV
// heads are cut into chunks that stream through two device buffer sets: while one
// chunk computes, the next one's Q/K/V cross PCIe on the host-to-device stream
// and the previous one's output on the device-to-host stream.  No arithmetic
// here: copies, events and the library's own entry points.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdarg>
#include <cstdio>

#include "qattn_internal.h"

namespace {

qattn_status hfail(qattn_status s, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
qattn_status hfail(qattn_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  qattn::set_last_error(buf);
  return s;
}

qattn_status hcuda(cudaError_t e, const char* where) {
  return hfail(QATTN_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

constexpr size_t kAlign = 256;
size_t up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

// Byte offsets of one buffer set, sized for `ck` KV heads (ck * G query heads).
struct SetLayout {
  size_t q_in, k_in, v_in, q8, q_scale, k8, k_scale, k_mean, v8t, v_scale, qws, out;
  size_t qws_bytes, bytes;
};

SetLayout set_layout(int B, int Nq, int Nkv, int G, int ck, int D) {
  const size_t cq = static_cast<size_t>(ck) * G;
  const size_t nK = (Nkv + 63) / 64, nQ = (Nq + 127) / 128;
  const size_t rq = static_cast<size_t>(B) * Nq, rk = static_cast<size_t>(B) * Nkv;
  SetLayout L{};
  size_t o = 0;
  auto take = [&](size_t bytes) {
    const size_t at = o;
    o += up(bytes);
    return at;
  };
  L.q_in = take(rq * cq * D * 2);
  L.k_in = take(rk * ck * D * 2);
  L.v_in = take(rk * ck * D * 2);
  L.q8 = take(rq * cq * D);
  L.q_scale = take(static_cast<size_t>(B) * cq * 4 * nQ * 4);
  L.k8 = take(rk * ck * D);
  // FP32 per 64-key block, or (Hadamard) FP16 per token
  L.k_scale = take(static_cast<size_t>(B) * ck * std::max(nK * 4, static_cast<size_t>(Nkv) * 2));
  L.k_mean = take(static_cast<size_t>(B) * ck * D * 4);
  L.v8t = take(static_cast<size_t>(B) * ck * D * 64 * nK);
  L.v_scale = take(static_cast<size_t>(B) * ck * D * 4);
  // the fused quantizer's scratch (its RoPE tables sized for rotary_dim = D, the
  // largest); the Hadamard quantizer needs less
  L.qws_bytes = qattn_prep_quant_workspace_bytes(B, Nkv, ck, D, D);
  L.qws = take(L.qws_bytes);
  L.out = take(rq * cq * D * 2);
  L.bytes = o;
  return L;
}

bool sizes_ok(int B, int Nq, int Nkv, int Hq, int Hkv, int D, int chunk) {
  return B > 0 && Nq > 0 && Nkv > 0 && Hq > 0 && Hkv > 0 && Hq % Hkv == 0 &&
         (D == 64 || D == 128 || D == 256) && chunk > 0;
}

// A host view must hold whole head rows back to back: stride[3] == 1 and
// stride[2] == D, so the heads of one chunk are one contiguous span per (b, n).
qattn_status check_host_view(const char* name, const qattn_bnhd& v, int D) {
  if (v.ptr == nullptr) return hfail(QATTN_ERR_NULL, "attention_host: %s is null", name);
  if (v.stride[3] != 1 || v.stride[2] != D)
    return hfail(QATTN_ERR_STRIDE, "attention_host: %s needs stride[3] == 1 and stride[2] == D", name);
  if ((reinterpret_cast<uintptr_t>(v.ptr) & 15u) != 0 || v.stride[1] % 8 != 0 || v.stride[0] % 8 != 0)
    return hfail(QATTN_ERR_STRIDE, "attention_host: %s rows must be 16-byte aligned", name);
  return QATTN_OK;
}

// Heads [h0, h0+hc) of every row (b, n): host view -> a contiguous device block
// [B, N, hc, D].  One 2D copy when the batch entries' rows are equally spaced
// (stride[0] == N * stride[1]), else one per batch entry.
cudaError_t copy_in(uint8_t* dst, const qattn_bnhd& v, int B, int N, int h0, int hc, int D,
                    cudaStream_t st) {
  const size_t width = static_cast<size_t>(hc) * D * 2;
  const size_t pitch = static_cast<size_t>(v.stride[1]) * 2;
  const bool merged = (v.stride[0] == static_cast<int64_t>(N) * v.stride[1]);
  for (int b = 0; b < (merged ? 1 : B); ++b) {
    const uint8_t* src = static_cast<const uint8_t*>(v.ptr) +
                         (static_cast<int64_t>(b) * v.stride[0] + static_cast<int64_t>(h0) * D) * 2;
    cudaError_t e = cudaMemcpy2DAsync(dst + static_cast<size_t>(b) * N * width, width, src, pitch,
                                      width, merged ? static_cast<size_t>(B) * N : N,
                                      cudaMemcpyHostToDevice, st);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace

extern "C" {

size_t qattn_host_workspace_bytes(int B, int Nq, int Nkv, int Hq, int Hkv, int D,
                                  int kv_heads_per_chunk) {
  if (!sizes_ok(B, Nq, Nkv, Hq, Hkv, D, kv_heads_per_chunk)) return 0;
  const int ck = std::min(kv_heads_per_chunk, Hkv);
  return 2 * set_layout(B, Nq, Nkv, Hq / Hkv, ck, D).bytes;
}

qattn_status qattn_attention_host(int B, int Nq, int Nkv, int Hq, int Hkv, int D,
                                  qattn_bnhd q, qattn_bnhd k, qattn_bnhd v,
                                  const uint16_t* q_weight, const uint16_t* k_weight, float eps,
                                  int rotary_dim, double rope_theta, int hadamard, float sm_scale,
                                  uint16_t* out, int kv_heads_per_chunk, void* workspace,
                                  size_t workspace_bytes, int* dev_err, void* stream,
                                  void* stream2, void* h2d_stream, void* d2h_stream) {
  if (!sizes_ok(B, Nq, Nkv, Hq, Hkv, D, kv_heads_per_chunk))
    return hfail(QATTN_ERR_SHAPE,
                 "attention_host: sizes must be positive, Hq %% Hkv == 0, D in {64,128,256} and "
                 "kv_heads_per_chunk >= 1");
  if (hadamard != 0 && hadamard != 1)
    return hfail(QATTN_ERR_UNSUPPORTED, "attention_host: hadamard must be 0 or 1");
  if (!hadamard && Nq != Nkv)
    return hfail(QATTN_ERR_UNSUPPORTED, "attention_host: prep needs Nq == Nkv (self-attention)");
  if (qattn_status s = check_host_view("q", q, D); s != QATTN_OK) return s;
  if (qattn_status s = check_host_view("k", k, D); s != QATTN_OK) return s;
  if (qattn_status s = check_host_view("v", v, D); s != QATTN_OK) return s;
  if (out == nullptr || dev_err == nullptr)
    return hfail(QATTN_ERR_NULL, "attention_host: out and dev_err must not be null");
  if ((reinterpret_cast<uintptr_t>(out) & 15u) != 0)
    return hfail(QATTN_ERR_STRIDE, "attention_host: out must be 16-byte aligned");
  const int G = Hq / Hkv;
  const int ck = std::min(kv_heads_per_chunk, Hkv);
  const SetLayout L = set_layout(B, Nq, Nkv, G, ck, D);
  if (workspace == nullptr || (reinterpret_cast<uintptr_t>(workspace) & (kAlign - 1)) != 0 ||
      workspace_bytes < 2 * L.bytes)
    return hfail(QATTN_ERR_WORKSPACE,
                 "attention_host: workspace null, not 256-byte aligned, or under %zu bytes",
                 2 * L.bytes);

  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  // buffer set s computes on compute[s]: chunks of one set stay in order, and the
  // next chunk's kernels fill the SMs that the previous chunk's last wave leaves
  cudaStream_t compute[2] = {cs, stream2 ? static_cast<cudaStream_t>(stream2) : cs};
  cudaStream_t hs = h2d_stream ? static_cast<cudaStream_t>(h2d_stream) : cs;
  cudaStream_t ds = d2h_stream ? static_cast<cudaStream_t>(d2h_stream) : cs;
  cudaEvent_t ev[8];   // start, h2d[2], comp[2], d2h[2], join
  for (int i = 0; i < 8; ++i) {
    cudaError_t e = cudaEventCreateWithFlags(&ev[i], cudaEventDisableTiming);
    if (e != cudaSuccess) {
      for (int j = 0; j < i; ++j) cudaEventDestroy(ev[j]);
      return hcuda(e, "cudaEventCreateWithFlags");
    }
  }
  cudaEvent_t e_start = ev[0], *e_h2d = ev + 1, *e_comp = ev + 3, *e_d2h = ev + 5, e_join = ev[7];
  qattn_status st = QATTN_OK;
  auto cu = [&](cudaError_t e, const char* where) {
    if (e != cudaSuccess && st == QATTN_OK) st = hcuda(e, where);
    return st == QATTN_OK;
  };
  // the copy streams start after everything already queued on `stream` (the
  // previous call's use of the workspace included)
  cu(cudaEventRecord(e_start, cs), "cudaEventRecord") &&
      cu(cudaStreamWaitEvent(hs, e_start, 0), "cudaStreamWaitEvent") &&
      cu(cudaStreamWaitEvent(ds, e_start, 0), "cudaStreamWaitEvent") &&
      cu(cudaStreamWaitEvent(compute[1], e_start, 0), "cudaStreamWaitEvent");

  // With eight or more chunks the sizes ramp up (a quarter, a half, then the full
  // chunk): nothing computes before the first chunk has crossed PCIe, so it is
  // made short.  Fewer, smaller problems keep equal chunks (narrow copy rows move
  // slowly).
  const bool ramp = Hkv >= 8 * ck;
  auto chunk_heads = [&](int c) {
    if (!ramp) return ck;
    return c == 0 ? std::max(1, ck / 4) : (c == 1 ? std::max(1, ck / 2) : ck);
  };
  int n_chunks = 0;
  for (int h = 0; h < Hkv; h += chunk_heads(n_chunks++)) {
  }
  uint8_t* const ws = static_cast<uint8_t*>(workspace);
  int k0 = 0;
  for (int c = 0; st == QATTN_OK && c < n_chunks; k0 += chunk_heads(c), ++c) {
    const int s = c & 1;
    const int kc = std::min(chunk_heads(c), Hkv - k0), q0 = k0 * G, qc = kc * G;
    uint8_t* const base = ws + s * L.bytes;
    // ---- host -> device: this set's inputs were last read by chunk c-2
    if (c >= 2 && !cu(cudaStreamWaitEvent(hs, e_comp[s], 0), "cudaStreamWaitEvent")) break;
    cu(copy_in(base + L.q_in, q, B, Nq, q0, qc, D, hs), "cudaMemcpy2DAsync (q)") &&
        cu(copy_in(base + L.k_in, k, B, Nkv, k0, kc, D, hs), "cudaMemcpy2DAsync (k)") &&
        cu(copy_in(base + L.v_in, v, B, Nkv, k0, kc, D, hs), "cudaMemcpy2DAsync (v)");
    if (!cu(cudaEventRecord(e_h2d[s], hs), "cudaEventRecord")) break;
    // ---- compute: inputs landed, and this set's output was copied out (chunk c-2)
    cudaStream_t xs = compute[s];
    if (!cu(cudaStreamWaitEvent(xs, e_h2d[s], 0), "cudaStreamWaitEvent")) break;
    if (c >= 2 && !cu(cudaStreamWaitEvent(xs, e_d2h[s], 0), "cudaStreamWaitEvent")) break;
    const int64_t sq[4] = {static_cast<int64_t>(Nq) * qc * D, static_cast<int64_t>(qc) * D, D, 1};
    const int64_t sk[4] = {static_cast<int64_t>(Nkv) * kc * D, static_cast<int64_t>(kc) * D, D, 1};
    const qattn_bnhd qv{base + L.q_in, {sq[0], sq[1], sq[2], sq[3]}};
    const qattn_bnhd kv{base + L.k_in, {sk[0], sk[1], sk[2], sk[3]}};
    const qattn_bnhd vv{base + L.v_in, {sk[0], sk[1], sk[2], sk[3]}};
    int8_t* q8 = reinterpret_cast<int8_t*>(base + L.q8);
    float* q_scale = reinterpret_cast<float*>(base + L.q_scale);
    int8_t* k8 = reinterpret_cast<int8_t*>(base + L.k8);
    uint8_t* v8t = base + L.v8t;
    float* v_scale = reinterpret_cast<float*>(base + L.v_scale);
    uint16_t* out_c = reinterpret_cast<uint16_t*>(base + L.out);
    if (hadamard) {
      st = qattn_quant_hadamard(B, Nq, Nkv, qc, kc, D, qv, kv, vv, q8, q_scale, k8,
                                reinterpret_cast<uint16_t*>(base + L.k_scale), v8t, v_scale,
                                base + L.qws, L.qws_bytes, xs);
    } else {
      st = qattn_prep_quant(B, Nq, qc, kc, D, qv, kv, vv, q_weight, k_weight, eps, rotary_dim,
                            rope_theta, 0, q8, q_scale, k8, reinterpret_cast<float*>(base + L.k_scale),
                            reinterpret_cast<float*>(base + L.k_mean), v8t, v_scale, base + L.qws,
                            L.qws_bytes, xs);
    }
    if (st == QATTN_OK)
      st = qattn_fwd(B, Nq, Nkv, qc, kc, D, q8, q_scale, k8, base + L.k_scale, hadamard ? 1 : 0,
                     v8t, v_scale, sm_scale, out_c, dev_err, xs);
    if (st != QATTN_OK || !cu(cudaEventRecord(e_comp[s], xs), "cudaEventRecord")) break;
    // ---- device -> host: heads [q0, q0+qc) of every output row (b, n), one 2D copy
    if (!cu(cudaStreamWaitEvent(ds, e_comp[s], 0), "cudaStreamWaitEvent")) break;
    {
      const size_t width = static_cast<size_t>(qc) * D * 2;
      cu(cudaMemcpy2DAsync(reinterpret_cast<uint8_t*>(out) + static_cast<size_t>(q0) * D * 2,
                           static_cast<size_t>(Hq) * D * 2, base + L.out, width, width,
                           static_cast<size_t>(B) * Nq, cudaMemcpyDeviceToHost, ds),
         "cudaMemcpy2DAsync (out)");
    }
    cu(cudaEventRecord(e_d2h[s], ds), "cudaEventRecord");
  }
  // `stream` ends after everything this call queued on the other streams, on
  // success and after an error alike (a chunk may fail after its copies were
  // queued): synchronizing it (or qattn_check on it) covers the whole call, so the
  // caller may then reuse the workspace and the host buffers
  const cudaStream_t others[3] = {hs, ds, compute[1]};
  for (cudaStream_t o : others) {
    if (o == cs) continue;
    if (cudaEventRecord(e_join, o) == cudaSuccess) cudaStreamWaitEvent(cs, e_join, 0);
  }
  for (int i = 0; i < 8; ++i) cudaEventDestroy(ev[i]);   // released once their work completes
  return st;
}

}  // extern "C"
