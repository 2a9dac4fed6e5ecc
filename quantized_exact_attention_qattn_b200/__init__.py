"""B200-native quantized attention prefill (INT8 QK^T, FP8 P.V).

The compute lives in ``libqattn.so`` (hand-written sm_100a CUDA, C ABI in
``include/qattn.h``); this package only marshals arguments to it and uses
PyTorch for device memory and streams.  ``synth`` holds the seeded synthetic
workloads and imports nothing from here.
"""
from __future__ import annotations

import math

from ._lib import (EXPORTED, QAttnError, bnhd, load, qattn_attention_host,  # noqa: F401
                   qattn_check, qattn_debug_stall_kv_tile, qattn_fwd, qattn_host_workspace_bytes,
                   qattn_prep, qattn_prep_quant, qattn_prep_quant_workspace_bytes, qattn_quant,
                   qattn_quant_hadamard, qattn_quant_noalloc, qattn_quant_workspace_bytes,
                   qattn_quant_k32, qattn_quant_v16, qattn_fwd_pv16, qattn_kcache_append,
                   qattn_quant_q_hadamard, qattn_quant_v_rotated, qattn_fwd_int8v,
                   qattn_scores, qattn_tc_probe, qattn_version)

__all__ = ["Pipeline", "HostRunner", "default_kv_heads_per_chunk", "QAttnError", "qattn_prep",
           "qattn_prep_quant", "qattn_prep_quant_workspace_bytes", "qattn_tc_probe", "qattn_quant",
           "qattn_quant_k32", "qattn_quant_v16", "qattn_fwd_pv16", "qattn_kcache_append",
           "qattn_quant_q_hadamard", "qattn_quant_v_rotated", "qattn_fwd_int8v", "KCache",
           "qattn_quant_noalloc", "qattn_quant_hadamard",
           "qattn_fwd", "qattn_scores", "qattn_check", "qattn_quant_workspace_bytes",
           "qattn_host_workspace_bytes", "qattn_attention_host",
           "qattn_debug_stall_kv_tile", "qattn_version", "load"]


def _cdiv(a, b):
    return -(-a // b)


class Pipeline:
    """Device buffers for one problem size plus the call sequence
    prep -> quant -> fwd (or quant_hadamard -> fwd) through the C ABI; with
    ``fused=True`` the first two are one qattn_prep_quant call (same outputs bit
    for bit, no prepared BF16 Q/K stored, rotary_dim fixed at construction).

    Buffers are allocated once (PyTorch caching allocator) and reused by every
    ``run``; nothing is computed outside the library's kernels.
    """

    def __init__(self, B, Nq, Nkv, Hq, Hkv, D, *, hadamard=False, prep=True, fused=False,
                 rotary_dim=0, device="cuda"):
        import torch
        self.B, self.Nq, self.Nkv, self.Hq, self.Hkv, self.D = B, Nq, Nkv, Hq, Hkv, D
        self.hadamard, self.prep = hadamard, prep and not hadamard
        self.fused = fused and self.prep
        if self.fused and Nq != Nkv:
            raise ValueError("the fused prep + quant path works on self-attention inputs")
        nq, nk = _cdiv(Nq, 128), _cdiv(Nkv, 64)
        e = dict(device=device)
        if self.prep and not self.fused:
            self.qp = torch.empty((B, Nq, Hq, D), dtype=torch.bfloat16, **e)
            self.kp = torch.empty((B, Nkv, Hkv, D), dtype=torch.bfloat16, **e)
        self.q8 = torch.empty((B, Hq, Nq, D), dtype=torch.int8, **e)
        self.q_scale = torch.empty((B, Hq, 4 * nq), dtype=torch.float32, **e)
        self.k8 = torch.empty((B, Hkv, Nkv, D), dtype=torch.int8, **e)
        if hadamard:
            self.k_scale = torch.empty((B, Hkv, Nkv), dtype=torch.float16, **e)
        else:
            self.k_scale = torch.empty((B, Hkv, nk), dtype=torch.float32, **e)
        self.k_mean = torch.empty((B, Hkv, D), dtype=torch.float32, **e)
        self.v8t = torch.empty((B, Hkv, D, 64 * nk), dtype=torch.uint8, **e)
        self.v_scale = torch.empty((B, Hkv, D), dtype=torch.float32, **e)
        self.out = torch.empty((B, Nq, Hq, D), dtype=torch.bfloat16, **e)
        ws = qattn_quant_workspace_bytes(B, Nkv, Hkv, D)
        if self.fused:
            self.rotary_dim = rotary_dim
            ws = qattn_prep_quant_workspace_bytes(B, Nkv, Hkv, D, rotary_dim)
        self.ws = torch.empty(ws, dtype=torch.uint8, **e)
        self.dev_err = torch.zeros(1, dtype=torch.int32, **e)

    # --------------------------------------------------------------- steps
    def run_prep(self, q, k, q_weight, k_weight, eps, rotary_dim, theta=10000.0, pos_offset=0,
                 stream=None):
        assert self.Nq == self.Nkv, "prep works on self-attention inputs"
        qattn_prep(self.B, self.Nq, self.Hq, self.Hkv, self.D, q, k, q_weight, k_weight, eps,
                   rotary_dim, theta, pos_offset, self.qp, self.kp, stream)

    def run_prep_quant(self, q, k, v, q_weight, k_weight, eps, theta=10000.0, pos_offset=0,
                       stream=None):
        qattn_prep_quant(self.B, self.Nq, self.Hq, self.Hkv, self.D, q, k, v, q_weight, k_weight,
                         eps, self.rotary_dim, theta, pos_offset, self.q8, self.q_scale, self.k8,
                         self.k_scale, self.k_mean, self.v8t, self.v_scale, self.ws, stream=stream)

    def run_quant(self, qp, kp, v, stream=None):
        qattn_quant(self.B, self.Nq, self.Nkv, self.Hq, self.Hkv, self.D, qp, kp, v, self.q8,
                    self.q_scale, self.k8, self.k_scale, self.k_mean, self.v8t, self.v_scale,
                    self.ws, stream=stream)

    def run_quant_hadamard(self, q, k, v, stream=None):
        qattn_quant_hadamard(self.B, self.Nq, self.Nkv, self.Hq, self.Hkv, self.D, q, k, v,
                             self.q8, self.q_scale, self.k8, self.k_scale, self.v8t,
                             self.v_scale, self.ws, stream=stream)

    def run_fwd(self, sm_scale=0.0, stream=None):
        qattn_fwd(self.B, self.Nq, self.Nkv, self.Hq, self.Hkv, self.D, self.q8, self.q_scale,
                  self.k8, self.k_scale, 1 if self.hadamard else 0, self.v8t, self.v_scale,
                  sm_scale, self.out, self.dev_err, stream)

    def run(self, q, k, v, q_weight=None, k_weight=None, eps=1e-5, rotary_dim=0,
            theta=10000.0, pos_offset=0, stream=None):
        """The whole hot path on strided BF16 [B, N, H, D] views q, k, v."""
        if self.hadamard:
            self.run_quant_hadamard(q, k, v, stream)
        elif self.fused:
            if rotary_dim != self.rotary_dim:
                raise ValueError("rotary_dim differs from the one the workspace was sized for")
            self.run_prep_quant(q, k, v, q_weight, k_weight, eps, theta, pos_offset, stream)
        elif self.prep:
            self.run_prep(q, k, q_weight, k_weight, eps, rotary_dim, theta, pos_offset, stream)
            self.run_quant(self.qp, self.kp, v, stream)
        else:
            self.run_quant(q, k, v, stream)
        self.run_fwd(stream=stream)
        return self.out

    def check(self, stream=None):
        qattn_check(self.dev_err, stream)

    @property
    def attn_ops(self) -> float:
        return 4.0 * self.B * self.Hq * self.Nq * self.Nkv * self.D


class KCache:
    """A persistent rotated int8 key cache for chunked prefill (page "npu plan
    P7"): int8 K' = FWHT(k)/sqrt(D) with one FP16 scale per token, FP16 V, room
    for ``capacity`` keys per (batch, KV head).  ``append`` writes one chunk's
    keys after those already cached; ``attend`` runs a query chunk against every
    key cached so far.  All arithmetic is in the library's kernels."""

    def __init__(self, B, Hkv, D, capacity, device="cuda"):
        import torch
        if capacity % 8:
            raise ValueError("capacity must be a multiple of 8")
        self.B, self.Hkv, self.D, self.capacity = B, Hkv, D, capacity
        e = dict(device=device)
        self.k8 = torch.zeros((B, Hkv, capacity, D), dtype=torch.int8, **e)
        self.k_scale = torch.zeros((B, Hkv, capacity), dtype=torch.float16, **e)
        self.v16 = torch.zeros((B, Hkv, D, capacity), dtype=torch.float16, **e)
        self.dev_err = torch.zeros(1, dtype=torch.int32, **e)
        self.n = 0

    def append(self, k, v, stream=None):
        """k, v: raw BF16 [B, n_new, Hkv, D] views of the next chunk's keys.  The
        cache grows by n_new rounded up to a multiple of 8 (padding keys are never
        attended: only the first ``n`` keys are)."""
        n_new = k.shape[1]
        if self.n % 8:
            raise ValueError("only the last chunk may have a length that is not a multiple of 8")
        qattn_kcache_append(self.B, self.Hkv, self.D, n_new, self.n, self.capacity, k, v, self.k8,
                            self.k_scale, self.v16, stream)
        self.n += n_new

    def attend(self, q, out=None, sm_scale=0.0, stream=None):
        """q: raw BF16 [B, Nq, Hq, D] query chunk (rotated and quantized here);
        returns BF16 [B, Nq, Hq, D] attention over the cached keys."""
        import torch
        B, Nq, Hq, D = q.shape
        e = dict(device=self.k8.device)
        q8 = torch.empty((B, Hq, Nq, D), dtype=torch.int8, **e)
        qs = torch.empty((B, Hq, 4 * _cdiv(Nq, 128)), dtype=torch.float32, **e)
        qattn_quant_q_hadamard(B, Nq, Hq, D, q, q8, qs, stream)
        if out is None:
            out = torch.empty((B, Nq, Hq, D), dtype=torch.bfloat16, **e)
        qattn_fwd_pv16(B, Nq, self.n, Hq, self.Hkv, D, q8, qs, self.k8, self.k_scale, 1, self.v16,
                       self.capacity, sm_scale, out, self.dev_err, stream)
        return out

    def check(self, stream=None):
        qattn_check(self.dev_err, stream)


def default_kv_heads_per_chunk(B, Nq, Nkv, Hq, Hkv, D) -> int:
    """KV heads per chunk for ``qattn_attention_host`` (measured on one B200):
    inputs of 512 MB or more in about fourteen chunks (4 KV heads at N37810 H56
    D128: 40.9 ms end to end against 41.9 with 7 and 46.0 with 14), smaller ones
    in about four chunks of at least two KV heads (encoder B32 N729 H16 D64: 3.21
    ms against 3.76 in one chunk; GQA Nq1024 Nkv32768 Hkv4 D256: 3.53 ms with two
    heads, 3.68 in one chunk, 3.88 with one head per chunk)."""
    in_bytes = 2 * B * D * (Nq * Hq + 2 * Nkv * Hkv)
    if in_bytes >= (512 << 20):
        return -(-Hkv // 14)
    return min(Hkv, max(-(-Hkv // 4), 2 if Hkv >= 4 else 1))


class HostRunner:
    """``qattn_attention_host`` with its device workspace, error word and two
    copy streams: host Q/K/V in, host output back, chunks of KV heads overlapping
    PCIe with compute; the default chunk is ``default_kv_heads_per_chunk``."""

    def __init__(self, B, Nq, Nkv, Hq, Hkv, D, *, hadamard=False, kv_heads_per_chunk=None,
                 device="cuda"):
        import torch
        self.B, self.Nq, self.Nkv, self.Hq, self.Hkv, self.D = B, Nq, Nkv, Hq, Hkv, D
        self.hadamard = hadamard
        self.chunk = kv_heads_per_chunk or default_kv_heads_per_chunk(B, Nq, Nkv, Hq, Hkv, D)
        nbytes = qattn_host_workspace_bytes(B, Nq, Nkv, Hq, Hkv, D, self.chunk)
        if nbytes == 0:
            raise ValueError("invalid sizes for qattn_host_workspace_bytes")
        self.ws = torch.empty(nbytes, dtype=torch.uint8, device=device)
        self.dev_err = torch.zeros(1, dtype=torch.int32, device=device)
        self.compute2 = torch.cuda.Stream(device=device)
        self.h2d = torch.cuda.Stream(device=device)
        self.d2h = torch.cuda.Stream(device=device)

    def run(self, q, k, v, out, q_weight=None, k_weight=None, eps=1e-5, rotary_dim=0,
            theta=10000.0, sm_scale=0.0, stream=None):
        """q, k, v: host BF16 [B, N, H, D] views (pinned); out: host BF16 [B, Nq, Hq, D]."""
        qattn_attention_host(self.B, self.Nq, self.Nkv, self.Hq, self.Hkv, self.D, q, k, v,
                             q_weight, k_weight, eps, rotary_dim, theta, self.hadamard, sm_scale,
                             out, self.chunk, self.ws, self.dev_err, stream, self.compute2,
                             self.h2d, self.d2h)
        return out

    def check(self, stream=None):
        qattn_check(self.dev_err, stream)


def default_sm_scale(D: int) -> float:
    return 1.0 / math.sqrt(D)
