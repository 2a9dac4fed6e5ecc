"""GPU parity of the variants the pages name beside the FP8 path:

* FP16 P.V (page "Fused FP8 PV preparation": FP16 PV is the default, FP8
  probabilities the option): qattn_quant_v16 bit-exact against the oracle's
  FP16 V, qattn_fwd_pv16 within the output tolerance of the oracle's FP16-P
  attention, also on K/V stored inside larger buffers (kv_capacity).
* K scales per 32-row group (page "npu plan P7", the fallback for outlier
  heads): qattn_quant_k32 bit-exact against the oracle, qattn_fwd with
  k_scale_mode 2 within the output tolerance."""
import numpy as np
import pytest
import torch

import quantized_exact_attention_qattn_b200 as qa
from quantized_exact_attention_qattn_b200 import synth
from oracle import qattn_oracle as O

from gpu_helpers import DEV, assert_out_close, dev_bf16, host, inputs_on_device, oracle_full, run_pipeline

pytestmark = pytest.mark.gpu


def _cap(n):
    return 8 * -(-n // 8)


def _pv16(pipe, v_dev, w, cap=None, mode=None):
    """FP16 V + qattn_fwd_pv16 on a pipeline's quantized Q/K."""
    cap = cap or _cap(w.Nkv)
    v16 = torch.empty((w.B, w.Hkv, w.D, cap), dtype=torch.int16, device=DEV)
    qa.qattn_quant_v16(w.B, w.Nkv, w.Hkv, w.D, v_dev, v16, cap)
    out = torch.empty((w.B, w.Nq, w.Hq, w.D), dtype=torch.bfloat16, device=DEV)
    mode = (1 if w.hadamard else 0) if mode is None else mode
    qa.qattn_fwd_pv16(w.B, w.Nq, w.Nkv, w.Hq, w.Hkv, w.D, pipe.q8, pipe.q_scale, pipe.k8,
                      pipe.k_scale, mode, v16, w.Nkv, 0.0, out, pipe.dev_err)
    qa.qattn_check(pipe.dev_err)
    return host(v16).view(np.uint16), host(out)


@pytest.mark.parametrize("name", ["small", "mid", "encoder"])
def test_pv16_matches_oracle(name):
    w = synth.make(name)
    pipe = run_pipeline(w)
    ref = oracle_full(w)
    _, _, v, _keep = inputs_on_device(w)
    v16, out = _pv16(pipe, v, w)
    exp_v16 = O.quant_v16(w.v, _cap(w.Nkv))
    assert np.array_equal(v16, exp_v16)
    exp, _, _ = O.attention(ref["q8"], ref["q_scale"], ref["k8"], ref["k_scale"], exp_v16, None,
                            w.Nkv, pv="fp16")
    assert_out_close(out, exp, name + " fp16 P.V")


@pytest.mark.parametrize("B,N,H,Hkv,D", [(1, 1, 1, 1, 128), (1, 65, 4, 2, 128), (1, 200, 8, 2, 256),
                                         (3, 129, 2, 2, 64), (1, 1000, 6, 3, 128)])
def test_pv16_edge_shapes(B, N, H, Hkv, D):
    w = synth.custom(3000 + N, B, N, H, D, rope=True, Hkv=Hkv)
    pipe = run_pipeline(w)
    ref = oracle_full(w)
    _, _, v, _keep = inputs_on_device(w)
    v16, out = _pv16(pipe, v, w)
    exp, _, _ = O.attention(ref["q8"], ref["q_scale"], ref["k8"], ref["k_scale"], v16, None,
                            w.Nkv, pv="fp16")
    assert np.array_equal(v16, O.quant_v16(w.v, _cap(w.Nkv)))
    assert_out_close(out, exp, "fp16 P.V edge")


def test_pv16_rotated_gqa_per_token_scales():
    # the rotated int8-K layout (per-token FP16 K scales, D = 256, GQA 4:1)
    w = synth.make("gqa_chunk", Nq=200, Nkv=1000, seed=41)
    pipe = run_pipeline(w)
    ref = oracle_full(w)
    _, _, v, _keep = inputs_on_device(w)
    v16, out = _pv16(pipe, v, w)
    exp, _, _ = O.attention(ref["q8"], ref["q_scale"], ref["k8"], ref["k_scale"], v16, None,
                            w.Nkv, k_scale_mode=1, pv="fp16")
    assert_out_close(out, exp, "fp16 P.V rotated")


def test_pv16_inside_larger_buffers_equals_tight_buffers():
    # K, its per-token scales and V16 stored with room for 300 more keys: the same
    # output bit for bit as tightly sized operands
    w = synth.make("gqa_chunk", Nq=130, Nkv=700, Hq=8, Hkv=2, D=256, seed=42)
    pipe = run_pipeline(w)
    _, _, v, _keep = inputs_on_device(w)
    _, tight = _pv16(pipe, v, w)
    cap = 1000
    k8 = torch.zeros((w.B, w.Hkv, cap, w.D), dtype=torch.int8, device=DEV)
    k8[:, :, :w.Nkv] = pipe.k8
    ks = torch.zeros((w.B, w.Hkv, cap), dtype=torch.float16, device=DEV)
    ks[:, :, :w.Nkv] = pipe.k_scale
    v16 = torch.full((w.B, w.Hkv, w.D, cap), 0x7C00, dtype=torch.int16, device=DEV)   # +inf past Nkv
    qa.qattn_quant_v16(w.B, w.Nkv, w.Hkv, w.D, v, v16, cap)
    v16[:, :, :, _cap(w.Nkv):] = 0x7C00            # stale slots past the written ones
    out = torch.empty_like(pipe.out)
    qa.qattn_fwd_pv16(w.B, w.Nq, w.Nkv, w.Hq, w.Hkv, w.D, pipe.q8, pipe.q_scale, k8, ks, 1, v16,
                      cap, 0.0, out, pipe.dev_err)
    qa.qattn_check(pipe.dev_err)
    assert np.array_equal(host(out), tight)


@pytest.mark.parametrize("B,N,H,Hkv,D", [(1, 256, 2, 2, 128), (1, 75, 2, 1, 64), (2, 300, 4, 2, 256),
                                         (1, 1000, 6, 3, 128)])
def test_k32_scales_match_oracle(B, N, H, Hkv, D):
    w = synth.custom(4000 + N, B, N, H, D, rope=True, Hkv=Hkv)
    q, k, v, _keep = inputs_on_device(w)
    pipe = qa.Pipeline(B, N, N, H, Hkv, D, device=DEV)
    qw, kw = dev_bf16(w.q_weight), dev_bf16(w.k_weight)
    pipe.run_prep(q, k, qw, kw, w.eps, w.rotary_dim, w.theta)
    ks32 = torch.empty((B, Hkv, -(-N // 32)), dtype=torch.float32, device=DEV)
    qa.qattn_quant_k32(B, N, N, H, Hkv, D, pipe.qp, pipe.kp, v, pipe.q8, pipe.q_scale, pipe.k8, ks32,
                       pipe.k_mean, pipe.v8t, pipe.v_scale, pipe.ws)
    out = torch.empty_like(pipe.out)
    qa.qattn_fwd(B, N, N, H, Hkv, D, pipe.q8, pipe.q_scale, pipe.k8, ks32, 2, pipe.v8t, pipe.v_scale,
                 0.0, out, pipe.dev_err)
    qa.qattn_check(pipe.dev_err)
    ref = oracle_full(w)
    k8, ks = O.quant_k32(ref["kp"], ref["k_mean"])
    assert np.array_equal(host(pipe.k8), k8) and np.array_equal(host(ks32), ks)
    assert np.array_equal(host(pipe.q8), ref["q8"]) and np.array_equal(host(pipe.v8t), ref["v8t"])
    exp, _, _ = O.attention(ref["q8"], ref["q_scale"], k8, ks, ref["v8t"], ref["v_scale"], N,
                            k_scale_mode=2)
    assert_out_close(host(out), exp, "k32")


# --------------------------------------------------------------------- rotated INT8 V
def _int8v(pipe, v_dev, w, mode):
    nk = -(-w.Nkv // 64)
    v8t = torch.empty((w.B, w.Hkv, w.D, 64 * nk), dtype=torch.int8, device=DEV)
    vs = torch.empty((w.B, w.Hkv, w.D), dtype=torch.float32, device=DEV)
    qa.qattn_quant_v_rotated(w.B, w.Nkv, w.Hkv, w.D, v_dev, v8t, vs, pipe.ws)
    out = torch.empty((w.B, w.Nq, w.Hq, w.D), dtype=torch.bfloat16, device=DEV)
    qa.qattn_fwd_int8v(w.B, w.Nq, w.Nkv, w.Hq, w.Hkv, w.D, pipe.q8, pipe.q_scale, pipe.k8,
                       pipe.k_scale, mode, v8t, vs, 0.0, out, pipe.dev_err)
    qa.qattn_check(pipe.dev_err)
    return host(v8t), host(vs), host(out)


@pytest.mark.parametrize("Nq,Nkv,Hq,Hkv,D", [(200, 1000, 16, 4, 256), (130, 97, 8, 2, 256),
                                             (64, 3000, 4, 1, 256)])
def test_int8v_rotated_gqa_matches_oracle(Nq, Nkv, Hq, Hkv, D):
    w = synth.make("gqa_chunk", Nq=Nq, Nkv=Nkv, Hq=Hq, Hkv=Hkv, D=D, seed=Nq + Nkv + 7)
    pipe = run_pipeline(w)
    ref = oracle_full(w)
    _, _, v, _keep = inputs_on_device(w)
    v8t, vs, out = _int8v(pipe, v, w, 1)
    exp_v8t, exp_vs = O.quant_v_rotated(w.v)
    assert np.array_equal(v8t, exp_v8t) and np.array_equal(vs, exp_vs)
    exp, _, _ = O.attention(ref["q8"], ref["q_scale"], ref["k8"], ref["k_scale"], exp_v8t, exp_vs,
                            w.Nkv, k_scale_mode=1, pv="int8v")
    assert_out_close(out, exp, "rotated int8 V")


def test_int8v_with_block_k_scales_and_d64_quantizer():
    # D = 256 attention with per-64-row K scales (the standard quantizer), and the
    # D = 64 rotated V quantizer on its own
    w = synth.custom(5151, 1, 300, 4, 256, rope=True, Hkv=2)
    pipe = run_pipeline(w)
    ref = oracle_full(w)
    _, _, v, _keep = inputs_on_device(w)
    v8t, vs, out = _int8v(pipe, v, w, 0)
    exp_v8t, exp_vs = O.quant_v_rotated(w.v)
    assert np.array_equal(v8t, exp_v8t) and np.array_equal(vs, exp_vs)
    exp, _, _ = O.attention(ref["q8"], ref["q_scale"], ref["k8"], ref["k_scale"], exp_v8t, exp_vs,
                            w.Nkv, pv="int8v")
    assert_out_close(out, exp, "rotated int8 V, block K scales")
    w64 = synth.custom(5152, 2, 150, 2, 64, rope=False)
    v64 = dev_bf16(w64.v)
    ws = torch.empty(qa.qattn_quant_workspace_bytes(2, 150, 2, 64), dtype=torch.uint8, device=DEV)
    v8t64 = torch.empty((2, 2, 64, 192), dtype=torch.int8, device=DEV)
    vs64 = torch.empty((2, 2, 64), dtype=torch.float32, device=DEV)
    qa.qattn_quant_v_rotated(2, 150, 2, 64, v64, v8t64, vs64, ws)
    torch.cuda.synchronize()
    e8, es = O.quant_v_rotated(w64.v)
    assert np.array_equal(host(v8t64), e8) and np.array_equal(host(vs64), es)
