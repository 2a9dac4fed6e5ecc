"""Edge shapes, GQA, cross-length, metamorphic and sentinel checks on the GPU.

Ragged sequence lengths exercise partial 32-row Q groups, partial 128-row Q
tiles, partial 64-key tiles (masked scores, zero V rows) and single-row cases;
the p2 validation grid (1/2/6/7 rows, 1..768 keys) appears through N.
"""
import numpy as np
import pytest
import torch

import quantized_exact_attention_qattn_b200 as qa
from quantized_exact_attention_qattn_b200 import synth
from oracle import qattn_oracle as O

from gpu_helpers import DEV, assert_out_close, dev_bf16, host, oracle_full, run_pipeline

pytestmark = pytest.mark.gpu

EDGE = [
    # (B, N, H, Hkv, D, rope)
    (1, 1, 1, 1, 128, True),
    (1, 2, 2, 2, 64, False),
    (1, 7, 1, 1, 256, True),
    (2, 15, 2, 1, 128, True),
    (1, 17, 3, 3, 64, False),
    (1, 31, 2, 2, 256, False),
    (1, 64, 2, 2, 128, True),
    (1, 65, 4, 2, 128, True),
    (3, 129, 2, 2, 64, False),
    (1, 200, 8, 2, 256, True),
    (1, 729, 2, 2, 64, False),
    (2, 768, 2, 2, 128, True),
    (1, 500, 2, 2, 128, True),       # four query tiles: a last group of one
    (1, 1000, 6, 3, 128, True),
]


def _check_all(w, pipe, ref):
    for key in ("qp", "kp", "k_mean", "q8", "q_scale", "k8", "k_scale", "v8t", "v_scale"):
        assert np.array_equal(host(getattr(pipe, key)), ref[key]), key
    assert_out_close(host(pipe.out), ref["out"], w.name)


@pytest.mark.parametrize("B,N,H,Hkv,D,rope", EDGE)
def test_edge_shapes(B, N, H, Hkv, D, rope):
    w = synth.custom(1000 + N, B, N, H, D, rope=rope, Hkv=Hkv)
    pipe = run_pipeline(w)
    _check_all(w, pipe, oracle_full(w))


@pytest.mark.parametrize("Nq,Nkv,Hq,Hkv,D", [(100, 300, 4, 2, 128), (300, 65, 2, 1, 64),
                                             (1, 129, 2, 2, 256)])
def test_cross_length_without_prep(Nq, Nkv, Hq, Hkv, D):
    w = synth.custom(7 + Nq, 1, Nq, Hq, D, Hkv=Hkv, Nkv=Nkv, rope=False)
    pipe = qa.Pipeline(1, Nq, Nkv, Hq, Hkv, D, prep=False, device=DEV)
    pipe.run(dev_bf16(w.q), dev_bf16(w.k), dev_bf16(w.v))
    pipe.check()
    q8, qs = O.quant_q(w.q)
    k8, ks = O.quant_k(w.k, O.k_mean(w.k))
    v8t, vs = O.quant_v(w.v)
    out, _, _ = O.attention(q8, qs, k8, ks, v8t, vs, Nkv)
    assert np.array_equal(host(pipe.q8), q8) and np.array_equal(host(pipe.k8), k8)
    assert np.array_equal(host(pipe.v8t), v8t)
    assert_out_close(host(pipe.out), out, "cross-length")


@pytest.mark.parametrize("Nq,Nkv,Hq,Hkv,D", [(65, 200, 4, 1, 256), (130, 97, 2, 2, 64),
                                             (1, 64, 8, 4, 256)])
def test_hadamard_small(Nq, Nkv, Hq, Hkv, D):
    w = synth.make("gqa_chunk", Nq=Nq, Nkv=Nkv, Hq=Hq, Hkv=Hkv, D=D, seed=Nq + Nkv)
    pipe = run_pipeline(w)
    ref = oracle_full(w)
    for key in ("q8", "q_scale", "k8", "k_scale", "v8t", "v_scale"):
        assert np.array_equal(host(getattr(pipe, key)), ref[key]), key
    assert_out_close(host(pipe.out), ref["out"], "hadamard")


@pytest.mark.parametrize("Nq,Nkv,Hq,Hkv", [(300, 500, 4, 2), (700, 1000, 2, 1)])
def test_per_token_k_scales_d128(Nq, Nkv, Hq, Hkv):
    # qattn_fwd with per-token FP16 K scales at D = 128 (the rotated quantization
    # of the oracle only serves to produce per-token-scaled inputs here)
    w = synth.make("gqa_chunk", Nq=Nq, Nkv=Nkv, Hq=Hq, Hkv=Hkv, D=128, seed=Nq + Nkv)
    q8, qs, k8, ks16, v8t, vs = O.quant_hadamard(w.q, w.k, w.v)
    out, _, _ = O.attention(q8, qs, k8, ks16, v8t, vs, Nkv, k_scale_mode=1)
    pipe = qa.Pipeline(1, Nq, Nkv, Hq, Hkv, 128, hadamard=True, device=DEV)
    for name, arr in (("q8", q8), ("q_scale", qs), ("k8", k8), ("k_scale", ks16.view(np.int16)),
                      ("v8t", v8t), ("v_scale", vs)):
        dst = getattr(pipe, name)
        src = torch.from_numpy(np.ascontiguousarray(arr))
        dst.copy_(src.view(dst.dtype) if src.dtype.itemsize == dst.dtype.itemsize else src)
    pipe.run_fwd()
    pipe.check()
    assert_out_close(host(pipe.out), out, "per-token K scales, D=128")


def test_prep_position_offset():
    # RoPE positions pos_offset + n ("Preparation" step 3), bit-exact against the oracle
    w = synth.custom(25, 1, 300, 2, 128)
    pipe = qa.Pipeline(1, 300, 300, 2, 2, 128, device=DEV)
    pipe.run_prep(dev_bf16(w.q), dev_bf16(w.k), dev_bf16(w.q_weight), dev_bf16(w.k_weight), w.eps,
                  w.rotary_dim, w.theta, pos_offset=777)
    torch.cuda.synchronize()
    assert np.array_equal(host(pipe.qp), O.prep(w.q, w.q_weight, w.eps, w.rotary_dim, w.theta,
                                                 pos_offset=777))
    assert np.array_equal(host(pipe.kp), O.prep(w.k, w.k_weight, w.eps, w.rotary_dim, w.theta,
                                                 pos_offset=777))


def test_prep_without_norm_and_partial_rotary():
    # NULL weight: no RMSNorm for that tensor (Q here), RoPE still applied; K with
    # its norm; rotary_dim 64 of D = 128 (dims 64.. pass through)
    w = synth.custom(26, 1, 200, 3, 128)
    pipe = qa.Pipeline(1, 200, 200, 3, 3, 128, device=DEV)
    pipe.run_prep(dev_bf16(w.q), dev_bf16(w.k), None, dev_bf16(w.k_weight), w.eps, 64, w.theta)
    torch.cuda.synchronize()
    assert np.array_equal(host(pipe.qp), O.prep(w.q, None, w.eps, 64, w.theta))
    assert np.array_equal(host(pipe.kp), O.prep(w.k, w.k_weight, w.eps, 64, w.theta))


def test_custom_softmax_scale():
    # qattn_fwd's sm_scale: c = FP32(log2(e) * sm_scale) instead of log2(e)/sqrt(D)
    w = synth.make("small")
    pipe = run_pipeline(w)
    default = host(pipe.out).copy()
    pipe.run_fwd(sm_scale=0.05)
    pipe.check()
    ref = oracle_full(w)
    out, _, _ = O.attention(ref["q8"], ref["q_scale"], ref["k8"], ref["k_scale"], ref["v8t"],
                            ref["v_scale"], w.Nkv, sm_scale=0.05)
    assert_out_close(host(pipe.out), out, "sm_scale 0.05")
    assert not np.array_equal(host(pipe.out), default)


def test_interleaved_strided_equals_contiguous():
    # GPU-vs-GPU: the interleaved QKV buffer and contiguous copies give identical bytes
    B, N, H, D = 1, 333, 4, 128
    rng = np.random.default_rng(5)
    buf = torch.from_numpy(rng.standard_normal((B, N, 3, H, D), dtype=np.float32)).to(torch.bfloat16).to(DEV)
    w = synth.custom(5, B, N, H, D)
    qw, kw = dev_bf16(w.q_weight), dev_bf16(w.k_weight)
    a = qa.Pipeline(B, N, N, H, H, D, device=DEV)
    a.run(buf[:, :, 0], buf[:, :, 1], buf[:, :, 2], qw, kw, 1e-5, 96)
    b = qa.Pipeline(B, N, N, H, H, D, device=DEV)
    b.run(buf[:, :, 0].contiguous(), buf[:, :, 1].contiguous(), buf[:, :, 2].contiguous(), qw, kw,
          1e-5, 96)
    a.check(); b.check()
    assert torch.equal(a.out.view(torch.int16), b.out.view(torch.int16))
    assert torch.equal(a.v8t, b.v8t)


def test_batch_entries_are_independent():
    w = synth.custom(6, 3, 150, 2, 64, rope=False)
    full = run_pipeline(w)
    for bi in range(3):
        one = synth.custom(6, 3, 150, 2, 64, rope=False)
        one.q, one.k, one.v, one.B = one.q[bi:bi + 1], one.k[bi:bi + 1], one.v[bi:bi + 1], 1
        p1 = run_pipeline(one)
        assert torch.equal(p1.out.view(torch.int16), full.out[bi:bi + 1].view(torch.int16))


def test_head_permutation_permutes_output():
    w = synth.custom(8, 1, 200, 4, 128)
    base = run_pipeline(w)
    perm = [2, 0, 3, 1]
    w2 = synth.custom(8, 1, 200, 4, 128)
    w2.q, w2.k, w2.v = w.q[:, :, perm], w.k[:, :, perm], w.v[:, :, perm]
    p2 = run_pipeline(w2)
    assert torch.equal(p2.out.view(torch.int16), base.out[:, :, perm].view(torch.int16))


def test_outputs_leave_neighbouring_memory_untouched():
    # each output is a window inside a larger buffer of sentinel bytes
    B, N, H, D = 1, 77, 2, 128
    w = synth.custom(9, B, N, H, D)
    q, k, v = dev_bf16(w.q), dev_bf16(w.k), dev_bf16(w.v)
    pad = 4096

    def window(shape, dtype, fill):
        n = int(np.prod(shape))
        big = torch.full((n + 2 * pad,), fill, dtype=dtype, device=DEV)
        return big, big[pad:pad + n].view(shape)

    qp_b, qp = window((B, N, H, D), torch.int16, -12345)
    kp_b, kp = window((B, N, H, D), torch.int16, -12345)
    qattn_args = (B, N, H, H, D)
    qa.qattn_prep(*qattn_args, q, k, dev_bf16(w.q_weight), dev_bf16(w.k_weight), 1e-5, 96, 1e4, 0,
                  qp, kp)
    nk = O.ceil_div(N, 64)
    q8_b, q8 = window((B, H, N, D), torch.int8, 77)
    k8_b, k8 = window((B, H, N, D), torch.int8, 77)
    qs_b, qs = window((B, H, 4 * O.ceil_div(N, 128)), torch.float32, 123.0)
    ks_b, ks = window((B, H, nk), torch.float32, 123.0)
    mu_b, mu = window((B, H, D), torch.float32, 123.0)
    v8_b, v8 = window((B, H, D, 64 * nk), torch.uint8, 0xAB)
    vs_b, vs = window((B, H, D), torch.float32, 123.0)
    ws = torch.empty(qa.qattn_quant_workspace_bytes(B, N, H, D), dtype=torch.uint8, device=DEV)
    qa.qattn_quant(B, N, N, H, H, D, qp.view(torch.bfloat16), kp.view(torch.bfloat16), v, q8, qs,
                   k8, ks, mu, v8, vs, ws)
    out_b, out = window((B, N, H, D), torch.int16, 0x5A5A)
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    qa.qattn_fwd(B, N, N, H, H, D, q8, qs, k8, ks, 0, v8, vs, 0.0, out, err)
    qa.qattn_check(err)
    for big, fill in ((qp_b, -12345), (kp_b, -12345), (q8_b, 77), (k8_b, 77), (qs_b, 123.0),
                      (ks_b, 123.0), (mu_b, 123.0), (v8_b, 0xAB), (vs_b, 123.0), (out_b, 0x5A5A)):
        assert bool((big[:pad] == fill).all()) and bool((big[-pad:] == fill).all())
    ref = oracle_full(w)
    assert_out_close(host(out.view(torch.bfloat16)), ref["out"], "windowed")
    assert np.array_equal(host(v8), ref["v8t"])       # padded key rows are written as 0x00


def test_repeat_calls_are_deterministic():
    w = synth.make("mid")
    a = run_pipeline(w)
    first = a.out.clone()
    a.run_fwd()
    a.check()
    assert torch.equal(first.view(torch.int16), a.out.view(torch.int16))


@pytest.mark.parametrize("pos_offset,theta", [(0, 1e4), ((1 << 20) - 2048, 1e4),
                                              ((1 << 24) - 2048, 1e4), ((1 << 24) - 2048, 5e5)])
def test_rope_coefficients_wide_positions(pos_offset, theta):
    # The BF16 RoPE coefficients the library derives on the device (FP64 frequency,
    # angle, cos and sin, one rounding each; "Preparation" step 3) against the
    # oracle's numpy FP64 tables, up to position 2^24.  Head h of every row holds a
    # one-hot 1.0 at dim h and no norm is applied, so the prepared row carries
    # cos_h(pos) at dim h and sin_h(pos) at dim h + R/2, exactly.
    N, R, D = 2048, 96, 128
    half = R // 2
    x = np.zeros((1, N, half, D), np.uint16)
    x[0, :, np.arange(half), np.arange(half)] = 0x3F80            # BF16 1.0
    q = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).to(DEV)
    pipe = qa.Pipeline(1, N, N, half, half, D, device=DEV)
    pipe.run_prep(q, q, None, None, 1e-5, R, theta, pos_offset=pos_offset)
    torch.cuda.synchronize()
    got = host(pipe.qp)[0]                                         # [N, half, D] BF16 bits
    cos_ref, sin_ref = O.rope_tables(N, R, theta, pos_offset)
    h = np.arange(half)
    assert np.array_equal(got[:, h, h], cos_ref)
    assert np.array_equal(got[:, h, h + half], sin_ref)
