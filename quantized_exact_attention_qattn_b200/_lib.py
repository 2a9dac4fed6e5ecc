"""ctypes binding of ``libqattn.so`` (argument marshalling only).

Every function here has the same name and arguments as the C entry point in
``include/qattn.h``.  Tensors are PyTorch tensors used purely as device memory:
the binding passes their data pointers and strides and the current CUDA stream.
There is no fallback: if the library is missing or a call fails, it raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libqattn.so")

QATTN_STATUS = {0: "QATTN_OK", 1: "QATTN_ERR_NULL", 2: "QATTN_ERR_SHAPE", 3: "QATTN_ERR_STRIDE",
                4: "QATTN_ERR_UNSUPPORTED", 5: "QATTN_ERR_WORKSPACE", 6: "QATTN_ERR_CUDA",
                7: "QATTN_ERR_TIMEOUT"}

EXPORTED = ("qattn_prep", "qattn_quant_workspace_bytes", "qattn_quant", "qattn_quant_noalloc",
            "qattn_prep_quant_workspace_bytes", "qattn_prep_quant", "qattn_quant_k32",
            "qattn_quant_v16", "qattn_fwd_pv16", "qattn_kcache_append", "qattn_quant_q_hadamard",
            "qattn_quant_v_rotated", "qattn_fwd_int8v",
            "qattn_quant_hadamard",
            "qattn_fwd", "qattn_scores", "qattn_host_workspace_bytes", "qattn_attention_host",
            "qattn_check", "qattn_debug_stall_kv_tile", "qattn_last_error", "qattn_version")
# measurement aid, declared in include/qattn_probe.h
EXPORTED_PROBE = ("qattn_tc_probe",)


class QAttnError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{QATTN_STATUS.get(status, status)}: {msg}")
        self.status = status


class BNHD(ctypes.Structure):
    """C ``qattn_bnhd``: device pointer + element strides of [B, N, H, D]."""
    _fields_ = [("ptr", ctypes.c_void_p), ("stride", ctypes.c_int64 * 4)]


_lib = None


def load(path: str | None = None) -> ctypes.CDLL:
    """Load the library (once).  Raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    path = path or LIB_PATH
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with "
                           "`python -m quantized_exact_attention_qattn_b200.build`")
    lib = ctypes.CDLL(path)
    i, i64, f32, f64, vp, sz = (ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_double,
                                ctypes.c_void_p, ctypes.c_size_t)
    lib.qattn_prep.argtypes = [i, i, i, i, i, BNHD, BNHD, vp, vp, f32, i, f64, i64, vp, vp, vp]
    lib.qattn_quant_workspace_bytes.argtypes = [i, i, i, i]
    lib.qattn_quant_workspace_bytes.restype = sz
    lib.qattn_quant.argtypes = [i, i, i, i, i, i, BNHD, BNHD, BNHD, vp, vp, vp, vp, vp, vp, vp,
                                vp, sz, vp]
    lib.qattn_prep_quant_workspace_bytes.argtypes = [i, i, i, i, i]
    lib.qattn_prep_quant_workspace_bytes.restype = sz
    lib.qattn_prep_quant.argtypes = [i, i, i, i, i, BNHD, BNHD, BNHD, vp, vp, f32, i, f64, i64, vp,
                                     vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.qattn_quant_k32.argtypes = [i, i, i, i, i, i, BNHD, BNHD, BNHD, vp, vp, vp, vp, vp, vp, vp,
                                    vp, sz, vp]
    lib.qattn_quant_v16.argtypes = [i, i, i, i, BNHD, vp, i, vp]
    lib.qattn_fwd_pv16.argtypes = [i, i, i, i, i, i, vp, vp, vp, vp, i, vp, i, f32, vp, vp, vp]
    lib.qattn_kcache_append.argtypes = [i, i, i, i, i, i, BNHD, BNHD, vp, vp, vp, vp]
    lib.qattn_quant_q_hadamard.argtypes = [i, i, i, i, BNHD, vp, vp, vp]
    lib.qattn_quant_v_rotated.argtypes = [i, i, i, i, BNHD, vp, vp, vp, sz, vp]
    lib.qattn_fwd_int8v.argtypes = [i, i, i, i, i, i, vp, vp, vp, vp, i, vp, vp, f32, vp, vp, vp]
    lib.qattn_quant_noalloc.argtypes = [i, i, i, i, i, i, BNHD, BNHD, BNHD, vp, vp, vp, vp, vp,
                                        vp, vp, vp]
    lib.qattn_quant_hadamard.argtypes = [i, i, i, i, i, i, BNHD, BNHD, BNHD, vp, vp, vp, vp, vp,
                                         vp, vp, sz, vp]
    lib.qattn_fwd.argtypes = [i, i, i, i, i, i, vp, vp, vp, vp, i, vp, vp, f32, vp, vp, vp]
    lib.qattn_scores.argtypes = [i, i, i, i, i, i, vp, vp, vp, vp, i, vp, vp, f32, vp, i, vp, vp,
                                 vp, vp]
    lib.qattn_host_workspace_bytes.argtypes = [i, i, i, i, i, i, i]
    lib.qattn_host_workspace_bytes.restype = sz
    lib.qattn_attention_host.argtypes = [i, i, i, i, i, i, BNHD, BNHD, BNHD, vp, vp, f32, i, f64,
                                         i, f32, vp, i, vp, sz, vp, vp, vp, vp, vp]
    lib.qattn_check.argtypes = [vp, vp]
    lib.qattn_tc_probe.argtypes = [i, i, i, vp, vp, vp]
    lib.qattn_debug_stall_kv_tile.argtypes = [i]
    lib.qattn_last_error.restype = ctypes.c_char_p
    lib.qattn_version.restype = ctypes.c_char_p
    for name in ("qattn_prep", "qattn_prep_quant", "qattn_quant", "qattn_quant_noalloc",
                 "qattn_quant_k32", "qattn_quant_v16", "qattn_fwd_pv16", "qattn_kcache_append",
                 "qattn_quant_q_hadamard", "qattn_quant_v_rotated", "qattn_fwd_int8v", "qattn_quant_hadamard", "qattn_fwd",
                 "qattn_scores", "qattn_attention_host", "qattn_check", "qattn_debug_stall_kv_tile",
                 "qattn_tc_probe"):
        getattr(lib, name).restype = ctypes.c_int
    _lib = lib
    return lib


def _ptr(t) -> int | None:
    return None if t is None else t.data_ptr()


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def bnhd(t: torch.Tensor) -> BNHD:
    """A [B, N, H, D] BF16 tensor (any strides) as a ``qattn_bnhd``."""
    if t.dim() != 4 or t.dtype != torch.bfloat16:
        raise ValueError("expected a 4-D bfloat16 tensor [B, N, H, D]")
    v = BNHD()
    v.ptr = t.data_ptr()
    for k, s in enumerate(t.stride()):
        v.stride[k] = s
    return v


def _check(status: int):
    if status != 0:
        raise QAttnError(status, load().qattn_last_error().decode())


def qattn_prep(B, N, Hq, Hkv, D, q, k, q_weight, k_weight, eps, rotary_dim, rope_theta,
               pos_offset, q_out, k_out, stream=None):
    _check(load().qattn_prep(B, N, Hq, Hkv, D, bnhd(q), bnhd(k), _ptr(q_weight), _ptr(k_weight),
                             eps, rotary_dim, rope_theta, pos_offset, _ptr(q_out), _ptr(k_out),
                             _stream(stream)))


def qattn_quant_workspace_bytes(B, Nkv, Hkv, D) -> int:
    return int(load().qattn_quant_workspace_bytes(B, Nkv, Hkv, D))


def qattn_quant(B, Nq, Nkv, Hq, Hkv, D, qp, kp, v, q8, q_scale, k8, k_scale, k_mean, v8t,
                v_scale, workspace, workspace_bytes=None, stream=None):
    nbytes = workspace.numel() * workspace.element_size() if workspace_bytes is None else workspace_bytes
    _check(load().qattn_quant(B, Nq, Nkv, Hq, Hkv, D, bnhd(qp), bnhd(kp), bnhd(v), _ptr(q8),
                              _ptr(q_scale), _ptr(k8), _ptr(k_scale), _ptr(k_mean), _ptr(v8t),
                              _ptr(v_scale), _ptr(workspace), nbytes, _stream(stream)))


def qattn_prep_quant_workspace_bytes(B, N, Hkv, D, rotary_dim) -> int:
    return int(load().qattn_prep_quant_workspace_bytes(B, N, Hkv, D, rotary_dim))


def qattn_prep_quant(B, N, Hq, Hkv, D, q, k, v, q_weight, k_weight, eps, rotary_dim, rope_theta,
                     pos_offset, q8, q_scale, k8, k_scale, k_mean, v8t, v_scale, workspace,
                     workspace_bytes=None, stream=None):
    nbytes = workspace.numel() * workspace.element_size() if workspace_bytes is None else workspace_bytes
    _check(load().qattn_prep_quant(B, N, Hq, Hkv, D, bnhd(q), bnhd(k), bnhd(v), _ptr(q_weight),
                                   _ptr(k_weight), eps, rotary_dim, rope_theta, pos_offset,
                                   _ptr(q8), _ptr(q_scale), _ptr(k8), _ptr(k_scale), _ptr(k_mean),
                                   _ptr(v8t), _ptr(v_scale), _ptr(workspace), nbytes,
                                   _stream(stream)))


def qattn_quant_k32(B, Nq, Nkv, Hq, Hkv, D, qp, kp, v, q8, q_scale, k8, k_scale, k_mean, v8t,
                    v_scale, workspace, workspace_bytes=None, stream=None):
    """qattn_quant with one K scale per 32-row group (k_scale [B,Hkv,ceil(Nkv/32)])."""
    nbytes = workspace.numel() * workspace.element_size() if workspace_bytes is None else workspace_bytes
    _check(load().qattn_quant_k32(B, Nq, Nkv, Hq, Hkv, D, bnhd(qp), bnhd(kp), bnhd(v), _ptr(q8),
                                  _ptr(q_scale), _ptr(k8), _ptr(k_scale), _ptr(k_mean), _ptr(v8t),
                                  _ptr(v_scale), _ptr(workspace), nbytes, _stream(stream)))


def qattn_quant_v16(B, Nkv, Hkv, D, v, v16t, capacity, stream=None):
    _check(load().qattn_quant_v16(B, Nkv, Hkv, D, bnhd(v), _ptr(v16t), int(capacity),
                                  _stream(stream)))


def qattn_fwd_pv16(B, Nq, Nkv, Hq, Hkv, D, q8, q_scale, k8, k_scale, k_scale_mode, v16t,
                   kv_capacity, sm_scale, out, dev_err, stream=None):
    _check(load().qattn_fwd_pv16(B, Nq, Nkv, Hq, Hkv, D, _ptr(q8), _ptr(q_scale), _ptr(k8),
                                 _ptr(k_scale), k_scale_mode, _ptr(v16t), int(kv_capacity),
                                 sm_scale, _ptr(out), _ptr(dev_err), _stream(stream)))


def qattn_kcache_append(B, Hkv, D, n_new, key0, capacity, k, v, k8_cache, k_scale_cache, v16_cache,
                        stream=None):
    _check(load().qattn_kcache_append(B, Hkv, D, n_new, key0, capacity, bnhd(k), bnhd(v),
                                      _ptr(k8_cache), _ptr(k_scale_cache), _ptr(v16_cache),
                                      _stream(stream)))


def qattn_quant_q_hadamard(B, Nq, Hq, D, q, q8, q_scale, stream=None):
    _check(load().qattn_quant_q_hadamard(B, Nq, Hq, D, bnhd(q), _ptr(q8), _ptr(q_scale),
                                         _stream(stream)))


def qattn_quant_v_rotated(B, Nkv, Hkv, D, v, v8t, v_scale, workspace, workspace_bytes=None,
                          stream=None):
    nbytes = workspace.numel() * workspace.element_size() if workspace_bytes is None else workspace_bytes
    _check(load().qattn_quant_v_rotated(B, Nkv, Hkv, D, bnhd(v), _ptr(v8t), _ptr(v_scale),
                                        _ptr(workspace), nbytes, _stream(stream)))


def qattn_fwd_int8v(B, Nq, Nkv, Hq, Hkv, D, q8, q_scale, k8, k_scale, k_scale_mode, v8t, v_scale,
                    sm_scale, out, dev_err, stream=None):
    _check(load().qattn_fwd_int8v(B, Nq, Nkv, Hq, Hkv, D, _ptr(q8), _ptr(q_scale), _ptr(k8),
                                  _ptr(k_scale), k_scale_mode, _ptr(v8t), _ptr(v_scale), sm_scale,
                                  _ptr(out), _ptr(dev_err), _stream(stream)))


def qattn_quant_noalloc(B, Nq, Nkv, Hq, Hkv, D, qp, kp, v, q8, q_scale, k8, k_scale, k_mean, v8t,
                        v_scale, stream=None):
    """qattn_quant on the library's static scratch (no workspace argument)."""
    _check(load().qattn_quant_noalloc(B, Nq, Nkv, Hq, Hkv, D, bnhd(qp), bnhd(kp), bnhd(v), _ptr(q8),
                                      _ptr(q_scale), _ptr(k8), _ptr(k_scale), _ptr(k_mean),
                                      _ptr(v8t), _ptr(v_scale), _stream(stream)))


def qattn_quant_hadamard(B, Nq, Nkv, Hq, Hkv, D, q, k, v, q8, q_scale, k8, k_scale_f16, v8t,
                         v_scale, workspace, workspace_bytes=None, stream=None):
    nbytes = workspace.numel() * workspace.element_size() if workspace_bytes is None else workspace_bytes
    _check(load().qattn_quant_hadamard(B, Nq, Nkv, Hq, Hkv, D, bnhd(q), bnhd(k), bnhd(v),
                                       _ptr(q8), _ptr(q_scale), _ptr(k8), _ptr(k_scale_f16),
                                       _ptr(v8t), _ptr(v_scale), _ptr(workspace), nbytes,
                                       _stream(stream)))


def qattn_fwd(B, Nq, Nkv, Hq, Hkv, D, q8, q_scale, k8, k_scale, k_scale_mode, v8t, v_scale,
              sm_scale, out, dev_err, stream=None):
    _check(load().qattn_fwd(B, Nq, Nkv, Hq, Hkv, D, _ptr(q8), _ptr(q_scale), _ptr(k8),
                            _ptr(k_scale), k_scale_mode, _ptr(v8t), _ptr(v_scale), sm_scale,
                            _ptr(out), _ptr(dev_err), _stream(stream)))


def qattn_scores(B, Nq, Nkv, Hq, Hkv, D, q8, q_scale, k8, k_scale, k_scale_mode, v8t, v_scale,
                 sm_scale, tiles, n_tiles, s_out, out, dev_err, stream=None):
    _check(load().qattn_scores(B, Nq, Nkv, Hq, Hkv, D, _ptr(q8), _ptr(q_scale), _ptr(k8),
                               _ptr(k_scale), k_scale_mode, _ptr(v8t), _ptr(v_scale), sm_scale,
                               _ptr(tiles), n_tiles, _ptr(s_out), _ptr(out), _ptr(dev_err),
                               _stream(stream)))


def qattn_host_workspace_bytes(B, Nq, Nkv, Hq, Hkv, D, kv_heads_per_chunk) -> int:
    return int(load().qattn_host_workspace_bytes(B, Nq, Nkv, Hq, Hkv, D, kv_heads_per_chunk))


def qattn_attention_host(B, Nq, Nkv, Hq, Hkv, D, q, k, v, q_weight, k_weight, eps, rotary_dim,
                         rope_theta, hadamard, sm_scale, out, kv_heads_per_chunk, workspace,
                         dev_err, stream=None, stream2=None, h2d_stream=None, d2h_stream=None,
                         workspace_bytes=None):
    """q, k, v, out: HOST tensors (pinned); workspace, dev_err, weights: device.
    stream2 / h2d_stream / d2h_stream None: that work runs on `stream`."""
    nbytes = workspace.numel() * workspace.element_size() if workspace_bytes is None else workspace_bytes
    copy = lambda st: None if st is None else _stream(st)
    _check(load().qattn_attention_host(B, Nq, Nkv, Hq, Hkv, D, bnhd(q), bnhd(k), bnhd(v),
                                       _ptr(q_weight), _ptr(k_weight), eps, rotary_dim, rope_theta,
                                       int(hadamard), sm_scale, _ptr(out), kv_heads_per_chunk,
                                       _ptr(workspace), nbytes, _ptr(dev_err), _stream(stream),
                                       copy(stream2), copy(h2d_stream), copy(d2h_stream)))


def qattn_tc_probe(kind, iters, n_ctas, cycles, dev_err, stream=None):
    """Tensor-core peak probe (kind 0: INT8, 1: FP8 E4M3); see include/qattn_probe.h."""
    _check(load().qattn_tc_probe(int(kind), int(iters), int(n_ctas), _ptr(cycles), _ptr(dev_err),
                                 _stream(stream)))


def qattn_check(dev_err, stream=None):
    _check(load().qattn_check(_ptr(dev_err), _stream(stream)))


def qattn_debug_stall_kv_tile(kv_tile: int):
    """Test hook: later qattn_fwd launches skip the K/V copy of `kv_tile` (-1: off)."""
    _check(load().qattn_debug_stall_kv_tile(int(kv_tile)))


def qattn_version() -> str:
    return load().qattn_version().decode()
