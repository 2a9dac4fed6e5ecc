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
                   qattn_prep, qattn_quant, qattn_quant_hadamard, qattn_quant_noalloc,
                   qattn_quant_workspace_bytes, qattn_scores, qattn_version)

__all__ = ["Pipeline", "HostRunner", "default_kv_heads_per_chunk", "QAttnError", "qattn_prep", "qattn_quant",
           "qattn_quant_noalloc", "qattn_quant_hadamard",
           "qattn_fwd", "qattn_scores", "qattn_check", "qattn_quant_workspace_bytes",
           "qattn_host_workspace_bytes", "qattn_attention_host",
           "qattn_debug_stall_kv_tile", "qattn_version", "load"]


def _cdiv(a, b):
    return -(-a // b)


class Pipeline:
    """Device buffers for one problem size plus the call sequence
    prep -> quant -> fwd (or quant_hadamard -> fwd) through the C ABI.

    Buffers are allocated once (PyTorch caching allocator) and reused by every
    ``run``; nothing is computed outside the library's kernels.
    """

    def __init__(self, B, Nq, Nkv, Hq, Hkv, D, *, hadamard=False, prep=True, device="cuda"):
        import torch
        self.B, self.Nq, self.Nkv, self.Hq, self.Hkv, self.D = B, Nq, Nkv, Hq, Hkv, D
        self.hadamard, self.prep = hadamard, prep and not hadamard
        nq, nk = _cdiv(Nq, 128), _cdiv(Nkv, 64)
        e = dict(device=device)
        if self.prep:
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
        self.ws = torch.empty(qattn_quant_workspace_bytes(B, Nkv, Hkv, D), dtype=torch.uint8, **e)
        self.dev_err = torch.zeros(1, dtype=torch.int32, **e)

    # --------------------------------------------------------------- steps
    def run_prep(self, q, k, q_weight, k_weight, eps, rotary_dim, theta=10000.0, pos_offset=0,
                 stream=None):
        assert self.Nq == self.Nkv, "prep works on self-attention inputs"
        qattn_prep(self.B, self.Nq, self.Hq, self.Hkv, self.D, q, k, q_weight, k_weight, eps,
                   rotary_dim, theta, pos_offset, self.qp, self.kp, stream)

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
