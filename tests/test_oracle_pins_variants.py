"""Pins of the oracle's variant readings: K scales per 32-row group (page "npu
plan P7": per-32-group scales for outlier heads), FP16 V and FP16 probabilities
for the P.V product (page "Fused FP8 PV preparation": FP16 PV is the default,
FP8 probabilities the option).  Hand-built cases, closed forms, brute force and
FP64 attention, each able to catch a plausible slip in the oracle."""
import math

import numpy as np

from oracle import qattn_oracle as O
from oracle.encoders import bf16_bits_from_f32, f32_from_bf16_bits, f32_from_f16_bits, f16_bits_from_f32
from quantized_exact_attention_qattn_b200 import synth


def _bf(x):
    return bf16_bits_from_f32(np.asarray(x, np.float32))


def _f(b):
    return f32_from_bf16_bits(b).astype(np.float64)


def test_quant_k32_groups_are_32_rows_brute_force():
    rng = np.random.default_rng(21)
    n, d = 75, 64
    k = rng.standard_normal((1, n, 1, d)).astype(np.float32)
    k[0, 40, 0, 7] = 30.0                                  # only group 1 (rows 32..63) sees it
    kb = _bf(k)
    mu = O.k_mean(kb)
    k8, ks = O.quant_k32(kb, mu)
    assert ks.shape == (1, 1, 3) and k8.shape == (1, 1, n, d)
    x = (f32_from_bf16_bits(kb)[0, :, 0] - mu[0, 0]).astype(np.float32)   # FP32 subtraction
    for g in range(3):
        rows = range(32 * g, min(n, 32 * g + 32))           # tail rows take no part
        amax = np.float32(max(1e-7, max(abs(float(x[r, c])) for r in rows for c in range(d))))
        assert ks[0, 0, g] == np.float32(amax / np.float32(127.0)), g
        f = np.float32(np.float32(127.0) / amax)
        for r in rows:
            for c in range(0, d, 9):
                t = float(np.float32(x[r, c] * f))
                assert k8[0, 0, r, c] == max(-128, min(127, int(np.rint(t)))), (r, c)
    assert ks[0, 0, 1] > 4 * ks[0, 0, 0] and ks[0, 0, 1] > 4 * ks[0, 0, 2]


def test_quant_k32_equals_quant_k_when_both_halves_share_the_maximum():
    # each 64-row block's two 32-row halves hold the same magnitudes (the second a
    # sign-flipped copy of the first, mean zero by construction): one scale per
    # block or per half is the same number, so the codes agree bit for bit
    rng = np.random.default_rng(22)
    half = rng.standard_normal((1, 32, 1, 64)).astype(np.float32)
    k = np.concatenate([half, -half, 2 * half, -2 * half], axis=1)
    kb = _bf(k)
    mu = O.k_mean(kb)
    assert np.all(mu == 0)
    k8a, ksa = O.quant_k(kb, mu)
    k8b, ksb = O.quant_k32(kb, mu)
    assert np.array_equal(k8a, k8b)
    assert np.array_equal(np.repeat(ksa, 2, axis=2), ksb)


def test_quant_v16_is_an_exact_fp16_copy_in_range_and_pads_with_zero():
    rng = np.random.default_rng(23)
    v = rng.standard_normal((2, 13, 3, 64)).astype(np.float32)
    v[1, 5, 2, 9] = 1.25 * 2.0 ** -24                      # below FP16's smallest subnormal step
    v[0, 3, 1, 0] = 3.0 * 2.0 ** -24                       # an exact FP16 subnormal
    vb = _bf(v)
    v16 = O.quant_v16(vb)
    assert v16.shape == (2, 3, 64, 16) and v16.dtype == np.uint16
    assert np.all(v16[..., 13:] == 0)
    back = f32_from_f16_bits(v16[..., :13]).transpose(0, 3, 1, 2)   # [B,N,H,D]
    ref = f32_from_bf16_bits(vb)
    ok = np.abs(ref) >= 2.0 ** -14
    assert np.array_equal(back[ok], ref[ok])
    assert v16[1, 2, 9, 5] == 0x0001                       # rounds to 2^-24 (nearest)
    assert v16[0, 1, 0, 3] == 0x0003
    assert O.quant_v16(vb, capacity=24).shape == (2, 3, 64, 24)


def test_fp16_pv_single_key_closed_form():
    # one key: m starts at -5e6, so old = 0 cancels d = 1 and p = 2^(s - mn) with
    # mn = s - 8.807 rounded as the oracle rounds; out = bf16((fp16(p) * v) / p)
    d = 64
    rng = np.random.default_rng(24)
    q8 = rng.integers(-127, 128, (1, 1, 1, d)).astype(np.int8)
    k8 = rng.integers(-127, 128, (1, 1, 1, d)).astype(np.int8)
    qs = np.full((1, 1, 4), 0.013, np.float32)
    ks = np.full((1, 1, 1), 0.021, np.float32)
    v = _bf(rng.standard_normal((1, 1, 1, d)))
    v16 = O.quant_v16(v)
    out, m, den = O.attention(q8, qs, k8, ks, v16, None, 1, pv="fp16")
    s_int = int(np.sum(q8.astype(np.int64) * k8.astype(np.int64)))
    c = O.score_constant(d)
    a = np.float32(np.float32(qs[0, 0, 0] * ks[0, 0, 0]) * c)
    mn = np.float32(np.float32(np.float32(s_int) * a) - np.float32(8.807))
    e = np.float32(s_int * float(a) - float(mn))
    p = np.float32(2.0 ** float(e))
    p16 = float(f32_from_f16_bits(f16_bits_from_f32(np.array([p], np.float32)))[0])
    assert den[0, 0, 0] == p
    exp = bf16_bits_from_f32(np.float32((p16 * _f(v)[0, 0, 0]) / float(p)))
    assert np.array_equal(out[0, 0, 0], exp)
    assert p16 != float(p)                                  # the FP16 rounding matters here


def _exact_attention(qp, kp, v, scale):
    qf, kf, vf = _f(qp), _f(kp), _f(v)
    out = np.zeros(qf.shape)
    for bi in range(qf.shape[0]):
        for hi in range(qf.shape[2]):
            s = qf[bi, :, hi] @ kf[bi, :, hi].T * scale
            pr = np.exp(s - s.max(1, keepdims=True))
            out[bi, :, hi] = (pr / pr.sum(1, keepdims=True)) @ vf[bi, :, hi]
    return out


def test_fp16_pv_is_the_more_accurate_control():
    # the FP16 P.V path is the accuracy control for FP8 probabilities: against FP64
    # attention on the small workload it is closer than the FP8 path, and close
    w = synth.make("small")
    r = O.pipeline(w.q, w.k, w.v, w.q_weight, w.k_weight, w.eps, w.rotary_dim)
    ref = _exact_attention(r["qp"], r["kp"], w.v, 1 / math.sqrt(w.D))
    v16 = O.quant_v16(w.v)
    o16, _, _ = O.attention(r["q8"], r["q_scale"], r["k8"], r["k_scale"], v16, None, w.Nkv,
                            pv="fp16")
    e8 = np.linalg.norm(_f(r["out"]) - ref) / np.linalg.norm(ref)
    e16 = np.linalg.norm(_f(o16) - ref) / np.linalg.norm(ref)
    assert e16 < e8
    cos = float((_f(o16).ravel() @ ref.ravel()) / np.linalg.norm(_f(o16)) / np.linalg.norm(ref))
    assert cos >= 0.9995


def test_per_32_scales_equal_to_the_block_scale_reproduce_block_mode():
    # k_scale_mode 2 takes key j's scale from its 32-row group; with both groups of
    # every block at the block's scale, A is the same number and the output equals
    # mode 0 bit for bit; one differing group scale changes it
    rng = np.random.default_rng(25)
    d, nq, nkv = 64, 40, 150
    nk = -(-nkv // 64)
    q8 = rng.integers(-127, 128, (1, 1, nq, d)).astype(np.int8)
    qs = (0.01 + 0.01 * rng.random((1, 1, 4))).astype(np.float32)
    k8 = rng.integers(-127, 128, (1, 1, nkv, d)).astype(np.int8)
    ks = (0.01 + 0.01 * rng.random((1, 1, nk))).astype(np.float32)
    ks32 = np.repeat(ks, 2, axis=2)[:, :, :-(-nkv // 32)]
    v8t = rng.integers(0, 0x7E, (1, 1, d, 64 * nk)).astype(np.uint8)
    vs = (0.1 + rng.random((1, 1, d))).astype(np.float32)
    a, _, _ = O.attention(q8, qs, k8, ks, v8t, vs, nkv, k_scale_mode=0)
    b, _, _ = O.attention(q8, qs, k8, ks32, v8t, vs, nkv, k_scale_mode=2)
    assert np.array_equal(a, b)
    ks32[0, 0, 3] *= np.float32(1.5)
    c, _, _ = O.attention(q8, qs, k8, ks32, v8t, vs, nkv, k_scale_mode=2)
    assert not np.array_equal(a, c)


def test_kcache_chunks_equal_the_one_shot_rotated_quantization():
    # the cache stores K per token, so appending three chunks gives the same codes,
    # scales and FP16 V as quantizing the whole key sequence at once
    rng = np.random.default_rng(26)
    b, h, d = 1, 2, 64
    chunks = [40, 24, 33]
    k = _bf(rng.standard_normal((b, sum(chunks), h, d)))
    v = _bf(rng.standard_normal((b, sum(chunks), h, d)))
    cache = O.kcache_new(b, h, d, 104)
    n0 = 0
    for n in chunks:
        O.kcache_append(cache, k[:, n0:n0 + n], v[:, n0:n0 + n])
        n0 += n
    k8, ks = O.quant_k_rotated(k)
    assert cache["n"] == 97
    assert np.array_equal(cache["k8"][:, :, :97], k8)
    assert np.array_equal(cache["k_scale"][:, :, :97], ks)
    assert np.array_equal(cache["v16"][..., :97], O.quant_v16(v, 97))
    assert not cache["k8"][:, :, 97:].any()


def test_kcache_attention_tracks_unrotated_fp64_attention():
    # Q and K rotated by the same H leave the scores unchanged, so the cache's
    # attention (rotated int8 K, FP16 P.V) stays close to plain FP64 attention;
    # rotating only one side would not
    rng = np.random.default_rng(27)
    b, h, d = 1, 1, 64
    kk = rng.standard_normal((b, 150, h, d))
    kk[..., 5] *= 8.0                                       # an outlier channel
    q, k, v = _bf(rng.standard_normal((b, 70, h, d))), _bf(kk), _bf(rng.standard_normal((b, 150, h, d)))
    cache = O.kcache_new(b, h, d, 160)
    O.kcache_append(cache, k[:, :64], v[:, :64])
    O.kcache_append(cache, k[:, 64:], v[:, 64:])
    out = _f(O.kcache_attend(cache, q))
    ref = _exact_attention(q, k, v, 1 / math.sqrt(d))
    cos = float(out.ravel() @ ref.ravel() / np.linalg.norm(out) / np.linalg.norm(ref))
    assert cos >= 0.999
    q8u, qsu = O.quant_q(q)                                  # unrotated Q against rotated K
    bad, _, _ = O.attention(q8u, qsu, cache["k8"][:, :, :150], cache["k_scale"][:, :, :150],
                            cache["v16"][..., :150], None, 150, k_scale_mode=1, pv="fp16")
    cos_bad = float(_f(bad).ravel() @ ref.ravel() / np.linalg.norm(_f(bad)) / np.linalg.norm(ref))
    assert cos_bad < 0.95


def _sylvester(n):
    h = np.array([[1.0]])
    while h.shape[0] < n:
        h = np.block([[h, h], [h, -h]])
    return h


def test_quant_v_rotated_round_trip_and_channel_maxima():
    rng = np.random.default_rng(28)
    b, n, h, d = 1, 90, 2, 64
    v = rng.standard_normal((b, n, h, d)).astype(np.float32)
    v[:, :, :, 3] *= 8.0                                   # an outlier channel
    vb = _bf(v)
    v8t, vs = O.quant_v_rotated(vb)
    assert v8t.shape == (b, h, d, 128) and v8t.dtype == np.int8 and vs.shape == (b, h, d)
    assert not v8t[..., n:].any()
    # every channel's maximum code is +-127 (amax maps to 127)
    assert np.all(np.abs(v8t[..., :n]).max(axis=-1) == 127)
    # decode, rotate back with an independent dense Sylvester matrix: V within half a
    # scale step of the rotation of each channel
    vr_dec = v8t[..., :n].astype(np.float64) * vs[..., None]          # [B,H,D,N]
    back = np.einsum("bhdn,de->bnhe", vr_dec, _sylvester(d) / math.sqrt(d))
    err = np.abs(back - _f(vb))
    bound = 0.5 * np.sqrt(np.sum(vs.astype(np.float64) ** 2, axis=-1)) * 1.0001   # per (b, h)
    assert np.all(err <= bound[:, None, :, None])


def test_int8v_output_is_the_inverse_rotation_of_the_fp16_path():
    # with the codes as FP16 V in the FP16 path (exact: |code| <= 127) and unit-power
    # scales, the rotated-V output must be bf16(H (o * s) / sqrt(D)) of the FP16
    # path's o; an independent dense Sylvester matrix stands in for the oracle's FWHT
    rng = np.random.default_rng(29)
    d, nq, nkv = 64, 20, 100
    q8 = rng.integers(-127, 128, (1, 1, nq, d)).astype(np.int8)
    qs = (0.01 + 0.01 * rng.random((1, 1, 4))).astype(np.float32)
    k8 = rng.integers(-127, 128, (1, 1, nkv, d)).astype(np.int8)
    ks = (0.01 + 0.01 * rng.random((1, 1, 2))).astype(np.float32)
    v8t = np.zeros((1, 1, d, 128), np.int8)
    v8t[..., :nkv] = rng.integers(-127, 128, (1, 1, d, nkv))
    s = (2.0 ** rng.integers(-4, 3, (1, 1, d))).astype(np.float32)
    v16 = f16_bits_from_f32(v8t.astype(np.float32))
    o16, _, _ = O.attention(q8, qs, k8, ks, v16, None, nkv, pv="fp16")
    o8, _, _ = O.attention(q8, qs, k8, ks, v8t, s, nkv, pv="int8v")
    pre = _f(o16)[0, :, 0] * s[0, 0].astype(np.float64)               # [nq, d]
    ref = (pre @ _sylvester(d).T) / math.sqrt(d)
    got = _f(o8)[0, :, 0]
    assert np.max(np.abs(got - ref)) <= 4 * 2.0 ** -8 * np.max(np.abs(ref))
    wrong = (pre @ _sylvester(d)[::-1].T) / math.sqrt(d)               # a permuted transform
    assert np.max(np.abs(got - wrong)) > 0.1 * np.max(np.abs(ref))
