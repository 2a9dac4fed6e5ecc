"""GPU parity of the fused prep + quantization entry point (qattn_prep_quant).

Its outputs (INT8 Q and K, their scales, the K mean, FP8 V and its scales) must
equal the oracle's bit for bit, as the two-step path's do, and equal the
two-step path (qattn_prep -> qattn_quant) bit for bit on the same inputs; the
attention output computed from them must be within the output tolerance."""
import numpy as np
import pytest
import torch

import quantized_exact_attention_qattn_b200 as qa
from quantized_exact_attention_qattn_b200 import synth
from oracle import qattn_oracle as O

from gpu_helpers import DEV, assert_out_close, dev_bf16, host, inputs_on_device, oracle_full

pytestmark = pytest.mark.gpu

QUANT_KEYS = ("q8", "q_scale", "k8", "k_scale", "k_mean", "v8t", "v_scale")


def _fused(w, pos_offset=0):
    q, k, v, _keep = inputs_on_device(w)
    pipe = qa.Pipeline(w.B, w.Nq, w.Nkv, w.Hq, w.Hkv, w.D, fused=True, rotary_dim=w.rotary_dim,
                       device=DEV)
    qw = dev_bf16(w.q_weight) if w.q_weight is not None else None
    kw = dev_bf16(w.k_weight) if w.k_weight is not None else None
    pipe.run(q, k, v, qw, kw, w.eps, w.rotary_dim, w.theta, pos_offset)
    pipe.check()
    torch.cuda.synchronize()
    return pipe


def _two_step(w, pos_offset=0):
    q, k, v, _keep = inputs_on_device(w)
    pipe = qa.Pipeline(w.B, w.Nq, w.Nkv, w.Hq, w.Hkv, w.D, device=DEV)
    qw = dev_bf16(w.q_weight) if w.q_weight is not None else None
    kw = dev_bf16(w.k_weight) if w.k_weight is not None else None
    pipe.run(q, k, v, qw, kw, w.eps, w.rotary_dim, w.theta, pos_offset)
    pipe.check()
    torch.cuda.synchronize()
    return pipe


@pytest.mark.parametrize("name", ["small", "mid", "encoder"])
def test_fused_matches_oracle(name):
    w = synth.make(name)
    pipe = _fused(w)
    ref = oracle_full(w)
    for key in QUANT_KEYS:
        assert np.array_equal(host(getattr(pipe, key)), ref[key]), key
    assert_out_close(host(pipe.out), ref["out"], name)


EDGE = [
    # (B, N, H, Hkv, D, rope): tails of 32-row groups, 64-row blocks, 128-row tiles,
    # GQA groups of several query heads per KV head, all three head dims
    (1, 1, 1, 1, 128, True),
    (1, 7, 1, 1, 256, True),
    (2, 15, 2, 1, 128, True),
    (1, 17, 3, 3, 64, False),
    (1, 65, 4, 2, 128, True),
    (3, 129, 2, 2, 64, True),
    (1, 200, 8, 2, 256, True),
    (1, 500, 2, 2, 128, True),
    (1, 1000, 6, 3, 128, True),
]


@pytest.mark.parametrize("B,N,H,Hkv,D,rope", EDGE)
def test_fused_edge_shapes(B, N, H, Hkv, D, rope):
    w = synth.custom(2000 + N, B, N, H, D, rope=rope, Hkv=Hkv)
    pipe = _fused(w)
    ref = oracle_full(w)
    for key in QUANT_KEYS:
        assert np.array_equal(host(getattr(pipe, key)), ref[key]), key
    assert_out_close(host(pipe.out), ref["out"], w.name)


def test_fused_position_offset():
    w = synth.custom(31, 1, 300, 2, 128, rope=True)
    pipe = _fused(w, pos_offset=777)
    qp = O.prep(w.q, w.q_weight, w.eps, w.rotary_dim, w.theta, pos_offset=777)
    kp = O.prep(w.k, w.k_weight, w.eps, w.rotary_dim, w.theta, pos_offset=777)
    q8, qs = O.quant_q(qp)
    mu = O.k_mean(kp)
    k8, ks = O.quant_k(kp, mu)
    for key, exp in (("q8", q8), ("q_scale", qs), ("k_mean", mu), ("k8", k8), ("k_scale", ks)):
        assert np.array_equal(host(getattr(pipe, key)), exp), key


def test_fused_equals_two_step_canonical():
    # the canonical interleaved call at full size: every quantized tensor equal to
    # the two-step path's (itself checked against the oracle in the full-size tests)
    w = synth.make("canonical")
    a = _fused(w)
    b = _two_step(w)
    for key in QUANT_KEYS:
        assert torch.equal(getattr(a, key).view(torch.uint8), getattr(b, key).view(torch.uint8)), key
    assert torch.equal(a.out.view(torch.int16), b.out.view(torch.int16))
