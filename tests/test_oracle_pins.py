"""Pins of the CPU oracle against what the pages and the mathematics fix:
closed forms, hand-built rows, printed constants, brute force on tiny inputs,
FP64 attention and identities.  Each test is chosen so that a plausible slip
in the oracle (dropped term, wrong sign or index, transposed operand) fails."""
import math
import os

import numpy as np
import pytest

from oracle import qattn_oracle as O
from oracle.encoders import (bf16_bits_from_f32, f32_from_bf16_bits, f32_from_e4m3_bits,
                             f32_from_f16_bits)
from quantized_exact_attention_qattn_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _pages_constants():
    out = {}
    with open(os.path.join(GOLDEN, "pages_constants.txt")) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                k, v = (s.strip() for s in line.split("=", 1))
                out[k] = v
    return out


PC = _pages_constants()


def _bf(x):
    return bf16_bits_from_f32(np.asarray(x, np.float32))


def _f(b):
    return f32_from_bf16_bits(b).astype(np.float64)


# ================================================================ constants
def test_oracle_constants_match_pages():
    assert float(O.M_INIT) == float(PC["softmax.m_init"])
    assert float(O.FP8_OFFSET) == np.float32(float(PC["softmax.fp8_offset"]))
    assert float(O.MASKED_SCORE) == float(PC["tails.masked_score"])
    assert float(O.AMAX_FLOOR) == np.float32(float(PC["quant.amax_floor"]))
    assert float(O.V_RANGE) == float(PC["v.range"])
    # 8.807 is log2(448) rounded down: 2^8.807 stays below the E4M3 maximum
    assert 2.0 ** float(O.FP8_OFFSET) < 448.0 < 2.0 ** (float(O.FP8_OFFSET) + 0.001)


def test_canonical_shape_counts_match_pages():
    n, h = int(PC["canonical.N"]), int(PC["canonical.H"])
    g = 4 * O.ceil_div(n, 128)
    nk = O.ceil_div(n, 64)
    assert [1, h, g] == [int(s) for s in PC["canonical.q_scale_shape"].split(",")]
    assert [1, h, nk] == [int(s) for s in PC["canonical.k_scale_shape"].split(",")]
    assert 64 * nk == int(PC["v.padded_rows"])
    assert nk - 1 == int(PC["softmax.last_tile"])
    assert n - 128 * (O.ceil_div(n, 128) - 1) == int(PC["tails.valid_rows_last_q128"])
    assert n - 64 * (nk - 1) == int(PC["tails.valid_rows_last_k64"])
    w = int(PC["canonical.qkv_row_width"])
    assert [int(s) for s in PC["canonical.strides"].split(",")] == [n * w, w, 128, 1]
    assert [int(s) for s in PC["canonical.offsets"].split(",")] == [0, h * 128, 2 * h * 128]


# ================================================================ RMSNorm
def test_rmsnorm_constant_row_returns_weight():
    # x = a on every dim: mean(x^2) = a^2, x*r = a/sqrt(a^2+eps) rounds to 1.0 in BF16,
    # so the output is exactly the weight.  (Wrong divisor or a dropped sqrt breaks it.)
    rng = np.random.default_rng(5)
    w = _bf(1.0 + 0.1 * rng.standard_normal(128))
    for a in (2.0, -0.75, 13.0):
        x = _bf(np.full((1, 1, 1, 128), a))
        y = O.prep(x, w, 1e-5, 0)
        expect = bf16_bits_from_f32(np.sign(a) * f32_from_bf16_bits(w))
        assert np.array_equal(y[0, 0, 0], expect)


def test_rmsnorm_one_hot_row():
    # a single nonzero a at dim i: the output there is sign(a)*sqrt(D) (to BF16), 0 elsewhere
    for d in (64, 128, 256):
        x = np.zeros((1, 1, 1, d), np.float32)
        x[..., 7] = -3.0
        y = O.prep(_bf(x), _bf(np.ones(d)), 1e-5, 0)
        assert abs(_f(y)[0, 0, 0, 7] + math.sqrt(d)) <= math.sqrt(d) * 2 ** -8
        assert np.count_nonzero(_f(y)) == 1


def test_rmsnorm_close_to_fp64_definition():
    rng = np.random.default_rng(6)
    for d in (64, 128, 256):
        x = _bf(rng.standard_normal((2, 9, 3, d)) * 3.0)
        w = _bf(1.0 + 0.1 * rng.standard_normal(d))
        y = _f(O.prep(x, w, 1e-5, 0))
        xf = _f(x)
        ref = xf / np.sqrt(np.mean(xf ** 2, axis=-1, keepdims=True) + 1e-5) * _f(w)
        # two BF16 roundings (normalized value, weighted value): <= ~2 BF16 ulps
        assert np.all(np.abs(y - ref) <= 2.0 ** -7 * np.abs(ref) + 1e-30)


def test_rms_sum_of_squares_follows_the_lane_tree():
    # brute force of the documented order with Python float32 scalars on rows
    # chosen so that FP32 order matters (mixed magnitudes)
    rng = np.random.default_rng(7)
    for d in (64, 128, 256):
        x = f32_from_bf16_bits(_bf(rng.standard_normal((40, d)) * np.exp2(rng.integers(-9, 9, (40, d)))))
        got = O.rms_sum_of_squares(x)
        lanes = d // 8
        for r in range(x.shape[0]):
            part = []
            for l in range(lanes):
                acc = np.float32(x[r, 8 * l] * x[r, 8 * l])
                for k in range(1, 8):
                    acc = np.float32(acc + np.float32(x[r, 8 * l + k] * x[r, 8 * l + k]))
                part.append(acc)
            off = lanes // 2
            while off:
                part = [np.float32(part[l] + part[l ^ off]) for l in range(lanes)]
                off //= 2
            assert got[r] == part[0]
        seq = np.zeros(x.shape[0], np.float32)
        for k in range(d):
            seq = (seq + x[:, k] * x[:, k]).astype(np.float32)
        assert not np.array_equal(seq, got), "test rows do not exercise the reduction order"


# ================================================================ RoPE
def test_rope_table_hand_values():
    # pair 0 has frequency 1: cos(1) = 0.5403 -> BF16 0x3F0A, sin(1) = 0.8415 -> 0x3F57.
    # pair R/4 = 24 has frequency theta^-0.5 = 0.01: at position 100 the angle is 1 again.
    c, s = O.rope_tables(101, 96, 10000.0)
    assert c[1, 0] == 0x3F0A and s[1, 0] == 0x3F57
    assert c[100, 24] == 0x3F0A and s[100, 24] == 0x3F57
    assert c[0].tolist() == [0x3F80] * 48 and s[0].tolist() == [0] * 48


def test_rope_split_half_pairing_and_sign():
    # one-hot inputs reveal the pair (i, i+R/2) and the rotate-half sign convention
    c, s = O.rope_tables(8, 96, 10000.0)
    p = 5
    x = np.zeros((1, 8, 1, 128), np.float32)
    x[0, :, 0, 0] = 1.0
    y = O.prep(_bf(x), None, 0.0, 96)
    assert y[0, p, 0, 0] == c[p, 0] and y[0, p, 0, 48] == s[p, 0]
    x = np.zeros((1, 8, 1, 128), np.float32)
    x[0, :, 0, 48] = 1.0
    y = O.prep(_bf(x), None, 0.0, 96)
    assert y[0, p, 0, 0] == (s[p, 0] ^ 0x8000) and y[0, p, 0, 48] == c[p, 0]
    assert np.count_nonzero(_f(y[0, p, 0])) == 2


def test_rope_position_zero_is_identity_and_tail_passes_through():
    rng = np.random.default_rng(8)
    x = _bf(rng.standard_normal((1, 6, 3, 128)))
    w = _bf(1.0 + 0.1 * rng.standard_normal(128))
    normed = O.prep(x, w, 1e-5, 0)
    roped = O.prep(x, w, 1e-5, 96)
    assert np.array_equal(roped[:, 0], normed[:, 0])
    assert np.array_equal(roped[..., 96:], normed[..., 96:])
    assert not np.array_equal(roped[:, 1:, :, :96], normed[:, 1:, :, :96])


def test_rope_preserves_pair_norm_and_relative_position():
    rng = np.random.default_rng(9)
    n = 300
    q = _bf(np.repeat(rng.standard_normal((1, 1, 1, 128)), n, axis=1))
    k = _bf(np.repeat(rng.standard_normal((1, 1, 1, 128)), n, axis=1))
    rq, rk = _f(O.prep(q, None, 0.0, 96)), _f(O.prep(k, None, 0.0, 96))
    qf = _f(q)
    n0 = qf[..., :48] ** 2 + qf[..., 48:96] ** 2
    n1 = rq[..., :48] ** 2 + rq[..., 48:96] ** 2
    assert np.allclose(n0, n1, rtol=2e-2, atol=1e-3)
    # <R_m q, R_n k> depends on m - n only (up to BF16 rounding of the table/values)
    dots = lambda m, nn: float(np.dot(rq[0, m, 0], rk[0, nn, 0]))
    ref = np.linalg.norm(qf[0, 0, 0]) * np.linalg.norm(_f(k)[0, 0, 0])
    for m, nn, dlt in ((10, 3, 100), (250, 7, 40), (5, 5, 200)):
        assert abs(dots(m, nn) - dots(m + dlt, nn + dlt)) < 2e-2 * ref


# ================================================================ K mean
def test_rope_position_offset_shifts_positions():
    # "Preparation" step 3 with positions pos_offset + n: prep at offset p equals
    # prep of the same rows placed at n + p with offset 0, and the explicit list
    rng = np.random.default_rng(24)
    n, p = 12, 1000
    x = _bf(rng.standard_normal((1, n, 2, 128)).astype(np.float32))
    w = _bf((1 + 0.1 * rng.standard_normal(128)).astype(np.float32))
    shifted = O.prep(x, w, 1e-5, 96, pos_offset=p)
    big = np.zeros((1, n + p, 2, 128), dtype=np.uint16)
    big[:, p:] = x
    assert np.array_equal(shifted, O.prep(big, w, 1e-5, 96)[:, p:])
    assert np.array_equal(shifted, O.prep(x, w, 1e-5, 96, positions=np.arange(p, p + n)))
    assert not np.array_equal(shifted, O.prep(x, w, 1e-5, 96))


def test_k_mean_closed_forms():
    n = 200
    k = np.zeros((1, n, 2, 64), np.float32)
    k[0, :, 0, :] = 3.5                                # constant column -> exact mean
    k[0, :, 1, 0] = np.arange(1, n + 1)                # 1..200 -> 100.5 exactly
    k[0, :, 1, 1] = np.where(np.arange(n) % 2 == 0, 1.0, -1.0)
    mu = O.k_mean(_bf(k))
    assert mu.shape == (1, 2, 64) and mu.dtype == np.float32
    assert np.all(mu[0, 0] == 3.5) and mu[0, 1, 0] == 100.5 and mu[0, 1, 1] == 0.0


def test_k_mean_centres_columns_and_leaves_softmax_invariant():
    rng = np.random.default_rng(10)
    k = _bf(rng.standard_normal((1, 130, 2, 64)) + 4.0 * rng.standard_normal((1, 1, 2, 64)))
    q = _f(_bf(rng.standard_normal((1, 7, 2, 64))))
    mu = O.k_mean(k).astype(np.float64)
    kf = _f(k)
    centred = kf - mu[:, None]
    assert np.all(np.abs(centred.sum(axis=1)) < 1e-4 * np.abs(kf).sum(axis=1))
    # softmax over keys is invariant to subtracting a per-(head, dim) constant from K
    for h in range(2):
        s0 = q[0, :, h] @ kf[0, :, h].T / 8.0
        s1 = q[0, :, h] @ centred[0, :, h].T / 8.0
        p0 = np.exp(s0 - s0.max(1, keepdims=True)); p0 /= p0.sum(1, keepdims=True)
        p1 = np.exp(s1 - s1.max(1, keepdims=True)); p1 /= p1.sum(1, keepdims=True)
        assert np.allclose(p0, p1, atol=1e-12)


# ================================================================ quantization
def test_quant_int8_hand_rows():
    # a group whose max is 127 has scale 1.0 and q = rint(x), ties to even
    x = np.zeros((1, 1, 32, 128), np.float32)
    x[0, 0, 0, :6] = [127.0, 2.5, 3.5, -2.5, -127.0, 0.49]
    q8, sc = O.quant_q(_bf(x).transpose(0, 2, 1, 3))
    assert sc.shape == (1, 1, 4) and sc[0, 0, 0] == 1.0
    assert q8[0, 0, 0, :6].tolist() == [127, 2, 4, -2, -127, 0]
    # the other three groups of the 128-row CTA hold no rows: all-zero scale
    assert np.all(sc[0, 0, 1:] == np.float32(np.float32(1e-7) / np.float32(127.0)))
    # +-amax map to +-127 for an arbitrary amax
    x = np.zeros((1, 1, 32, 128), np.float32)
    x[0, 0, 3, 9] = -0.3125
    x[0, 0, 31, 0] = 0.3125
    q8, sc = O.quant_q(_bf(x).transpose(0, 2, 1, 3))
    assert q8[0, 0, 3, 9] == -127 and q8[0, 0, 31, 0] == 127
    assert sc[0, 0, 0] == np.float32(np.float32(0.3125) / np.float32(127.0))


def test_quant_q_groups_are_32_rows_and_tail_rows_do_not_count():
    rng = np.random.default_rng(11)
    n = 150                                          # 2 CTAs: groups 0..7, rows >= 150 invalid
    q = rng.standard_normal((1, n, 1, 128)).astype(np.float32)
    q[0, 64, 0, 5] = 50.0                            # only group 2 sees it
    q8, sc = O.quant_q(_bf(q))
    assert sc.shape == (1, 1, 8) and q8.shape == (1, 1, n, 128)
    amax = [np.abs(_f(_bf(q))[0, 32 * g:min(n, 32 * g + 32)]).max() if 32 * g < n else 1e-7
            for g in range(8)]
    assert sc[0, 0, 2] == np.float32(np.float32(50.0) / np.float32(127.0))
    assert np.allclose(sc[0, 0], np.array(amax, np.float32) / 127.0, rtol=1e-6)
    assert np.all(sc[0, 0, 5:] == np.float32(np.float32(1e-7) / np.float32(127.0)))
    # a larger buffer with huge rows past N changes nothing
    q2 = np.concatenate([q, np.full((1, 10, 1, 128), 1e4, np.float32)], axis=1)
    q82, sc2 = O.quant_q(_bf(q2)[:, :n])
    assert np.array_equal(sc2, sc) and np.array_equal(q82, q8)


def test_quant_k_subtracts_mean_and_uses_64_row_blocks():
    rng = np.random.default_rng(12)
    k = _bf(rng.standard_normal((1, 130, 1, 64)) + 100.0)
    mu = O.k_mean(k)
    k8, ks = O.quant_k(k, mu)
    assert ks.shape == (1, 1, 3) and k8.shape == (1, 1, 130, 64)
    x = _f(k)[0, :, 0] - mu[0, 0].astype(np.float64)
    for j in range(3):
        blk = x[64 * j:64 * j + 64]
        assert abs(ks[0, 0, j] - np.abs(blk).max() / 127.0) <= 1e-6 * ks[0, 0, j]
    recon = k8[0, 0].astype(np.float64) * np.repeat(ks[0, 0], 64)[:130, None]
    assert np.max(np.abs(recon - x)) <= 0.5 * ks.max() * 1.0001


def test_quant_v_per_channel_fp8():
    rng = np.random.default_rng(13)
    v = rng.standard_normal((1, 100, 2, 64)).astype(np.float32)
    v[0, 17, 1, 3] = -9.0
    v8t, vs = O.quant_v(_bf(v))
    assert v8t.shape == (1, 2, 64, 128) and vs.shape == (1, 2, 64)
    assert np.all(v8t[..., 100:] == 0)
    assert vs[0, 1, 3] == np.float32(np.float32(9.0) / np.float32(2.25))
    assert v8t[0, 1, 3, 17] == 0xC1                  # -2.25 -> sign | 0x41
    dec = f32_from_e4m3_bits(v8t[..., :100]).astype(np.float64) * vs[..., None]
    ref = _f(_bf(v)).transpose(0, 2, 3, 1)
    # E4M3 keeps 3 mantissa bits: relative error <= 2^-4 above the subnormal range
    big = np.abs(ref) > vs[..., None] * 2.0 ** -6
    assert np.all(np.abs(dec - ref)[big] <= 2.0 ** -4 * np.abs(ref)[big] * 1.0001)


# ================================================================ scores
def test_scores_brute_force():
    rng = np.random.default_rng(14)
    q8 = rng.integers(-128, 128, (2, 5, 32), dtype=np.int64).astype(np.int8)
    k8 = rng.integers(-128, 128, (2, 7, 32), dtype=np.int64).astype(np.int8)
    s = O.scores(q8, k8)
    for h in range(2):
        for i in range(5):
            for j in range(7):
                assert s[h, i, j] == sum(int(q8[h, i, d]) * int(k8[h, j, d]) for d in range(32))
    big = O.scores(np.full((1, 1, 256), -128, np.int8), np.full((1, 1, 256), -128, np.int8))
    assert big[0, 0, 0] == 256 * 16384


# ================================================================ attention
def _exact_attention(qp, kp, v, scale):
    qf, kf, vf = _f(qp), _f(kp), _f(v)
    b, n, h, d = qf.shape
    out = np.zeros((b, n, h, d))
    for bi in range(b):
        for hi in range(h):
            s = qf[bi, :, hi] @ kf[bi, :, hi].T * scale
            p = np.exp(s - s.max(1, keepdims=True))
            out[bi, :, hi] = (p / p.sum(1, keepdims=True)) @ vf[bi, :, hi]
    return out


def _cos(a, b):
    a, b = a.ravel(), b.ravel()
    return float(a @ b / np.linalg.norm(a) / np.linalg.norm(b))


def test_pipeline_cosine_vs_fp64_attention_small_config():
    w = synth.make("small")
    r = O.pipeline(w.q, w.k, w.v, w.q_weight, w.k_weight, w.eps, w.rotary_dim)
    ref = _exact_attention(r["qp"], r["kp"], w.v, 1 / math.sqrt(w.D))
    assert _cos(_f(r["out"]), ref) >= 0.999


@pytest.mark.parametrize("rows", [1, 2, 6, 7])
@pytest.mark.parametrize("keys", [1, 2, 15, 16, 17, 31, 64, 65, 729, 768])
def test_edge_grid_random_scores(rows, keys):
    # the page's softmax check grid (rows 1/2/6/7 x keys 1..768)
    rng = np.random.default_rng(rows * 1000 + keys)
    d = 64
    q = _bf(rng.standard_normal((1, rows, 1, d)))
    k = _bf(rng.standard_normal((1, keys, 1, d)))
    v = _bf(rng.standard_normal((1, keys, 1, d)))
    q8, qs = O.quant_q(q)
    k8, ks = O.quant_k(k, O.k_mean(k))
    v8t, vs = O.quant_v(v)
    out, m, den = O.attention(q8, qs, k8, ks, v8t, vs, keys)
    ref = _exact_attention(q, k, v, 1 / math.sqrt(d))
    got = _f(out)
    assert out.shape == (1, rows, 1, d)
    assert np.max(np.abs(got - ref)) < 0.08
    assert _cos(got, ref) > 0.995


@pytest.mark.parametrize("keys", [1, 17, 64, 65, 729])
def test_constant_scores_give_uniform_weights_and_unquantized_denominator(keys):
    # q = 0 makes every score 0: each tile's max offset gives p = 2^8.807 for every key,
    # P8 = 448, and the denominator sums the UNQUANTIZED p (page 2, Validation).
    d = 64
    q8 = np.zeros((1, 1, 3, d), np.int8)
    qs = np.full((1, 1, 4), 0.01, np.float32)
    rng = np.random.default_rng(keys)
    k8 = rng.integers(-127, 128, (1, 1, keys, d)).astype(np.int8)
    ks = np.full((1, 1, O.ceil_div(keys, 64)), 0.02, np.float32)
    v = _bf(rng.standard_normal((1, keys, 1, d)))
    v8t, vs = O.quant_v(v)
    out, m, den = O.attention(q8, qs, k8, ks, v8t, vs, keys)
    p = np.float32(np.exp2(np.float64(np.float32(8.807))))
    assert np.all(m == -np.float32(8.807))
    # FP32 sequential sums drift by ~1e-5 relative; 448 vs 447.89 differs by 2.5e-4
    assert np.all(np.abs(den - keys * float(p)) <= 2e-5 * keys * float(p))
    assert np.all(np.abs(den - keys * 448.0) > 1e-4 * keys * 448.0)
    v8 = f32_from_e4m3_bits(v8t[0, 0, :, :keys]).astype(np.float64)
    expect = 448.0 * v8.sum(1) / float(den[0, 0, 0]) * vs[0, 0]
    assert np.allclose(_f(out)[0, 0, 0], expect, rtol=2 ** -7, atol=1e-6)


def test_extreme_scores_select_one_key():
    # one key scores far above the others: the output is that key's V (through FP8)
    d = 64
    keys = 200
    q8 = np.full((1, 1, 1, d), 100, np.int8)
    k8 = np.full((1, 1, keys, d), -100, np.int8)
    k8[0, 0, 150] = 100
    qs = np.full((1, 1, 4), 0.05, np.float32)
    ks = np.full((1, 1, 4), 0.05, np.float32)
    rng = np.random.default_rng(3)
    v = _bf(rng.standard_normal((1, keys, 1, d)))
    v8t, vs = O.quant_v(v)
    out, m, den = O.attention(q8, qs, k8, ks, v8t, vs, keys)
    v150 = f32_from_e4m3_bits(v8t[0, 0, :, 150]).astype(np.float64) * vs[0, 0]
    assert np.allclose(_f(out)[0, 0, 0], v150 * 448.0 / float(den[0, 0, 0]), rtol=2 ** -7, atol=1e-6)


def test_online_softmax_tile_order_matters_only_through_rounding():
    # reversing the key order changes tile membership; results agree to FP8 noise
    w = synth.custom(21, 1, 200, 1, 64, rope=False)
    q8, qs = O.quant_q(w.q)
    k8, ks = O.quant_k(w.k, O.k_mean(w.k))
    v8t, vs = O.quant_v(w.v)
    out1, _, _ = O.attention(q8, qs, k8, ks, v8t, vs, 200)
    kr = w.k[:, ::-1].copy()
    vr = w.v[:, ::-1].copy()
    k8r, ksr = O.quant_k(kr, O.k_mean(kr))
    v8tr, vsr = O.quant_v(vr)
    out2, _, _ = O.attention(q8, qs, k8r, ksr, v8tr, vsr, 200)
    assert _cos(_f(out1), _f(out2)) > 0.999


def test_gqa_maps_query_head_to_kv_head_by_division():
    rng = np.random.default_rng(15)
    d, n = 64, 70
    q8 = rng.integers(-127, 128, (1, 4, 33, d)).astype(np.int8)
    qs = (0.01 + 0.01 * rng.random((1, 4, 8))).astype(np.float32)
    k8 = rng.integers(-127, 128, (1, 2, n, d)).astype(np.int8)
    ks = (0.01 + 0.01 * rng.random((1, 2, 2))).astype(np.float32)
    v8t = rng.integers(0, 0x7E, (1, 2, d, 128)).astype(np.uint8)
    vs = (0.1 + rng.random((1, 2, d))).astype(np.float32)
    out, _, _ = O.attention(q8, qs, k8, ks, v8t, vs, n)
    rep = [0, 0, 1, 1]
    out2, _, _ = O.attention(q8, qs, k8[:, rep], ks[:, rep], v8t[:, rep], vs[:, rep], n)
    assert np.array_equal(out, out2)


def test_per_token_scales_equal_to_the_block_scale_reproduce_block_mode():
    # "Q And K Quantization" scales K per 64-row block; the rotated variant scales it
    # per token.  With every token's FP16 scale equal to its block's scale (values
    # exact in FP16), A = (q_scale * k_scale) * c is the same number per key, so the
    # per-token path must give the per-block output bit for bit (ragged last tile).
    rng = np.random.default_rng(16)
    d, nq, nkv = 64, 70, 150
    nk = -(-nkv // 64)
    q8 = rng.integers(-127, 128, (1, 2, nq, d)).astype(np.int8)
    qs = (0.01 + 0.01 * rng.random((1, 2, 4))).astype(np.float32)
    k8 = rng.integers(-127, 128, (1, 1, nkv, d)).astype(np.int8)
    ks = (2.0 ** -7 * (1 + rng.integers(0, 8, (1, 1, nk)) / 8.0)).astype(np.float32)
    ks_tok = np.repeat(ks, 64, axis=2)[:, :, :nkv]
    ks16 = ks_tok.astype(np.float16).view(np.uint16)
    assert np.array_equal(ks16.view(np.float16).astype(np.float32), ks_tok)   # exact in FP16
    v8t = rng.integers(0, 0x7E, (1, 1, d, 64 * nk)).astype(np.uint8)
    vs = (0.1 + rng.random((1, 1, d))).astype(np.float32)
    block, mb, db = O.attention(q8, qs, k8, ks, v8t, vs, nkv, k_scale_mode=0)
    token, mt, dt = O.attention(q8, qs, k8, ks16, v8t, vs, nkv, k_scale_mode=1)
    assert np.array_equal(block, token)
    assert np.array_equal(mb, mt) and np.array_equal(db, dt)
    # and a per-token scale that differs inside a block changes the output
    ks16b = ks16.copy()
    ks16b[0, 0, 3] = np.float16(ks_tok[0, 0, 3] * 2).view(np.uint16)
    other, _, _ = O.attention(q8, qs, k8, ks16b, v8t, vs, nkv, k_scale_mode=1)
    assert not np.array_equal(block, other)


def test_v_scale_is_applied_per_output_channel():
    # "Finalization And Tails": out[d] = bf16((O[d] / l) * v_scale[d]).  A power of two
    # 2^e_d on v_scale[d] commutes with every rounding, so output channel d (and only
    # it) moves by exactly 2^e_d: the scale is applied on the right axis.
    rng = np.random.default_rng(17)
    d, n = 64, 100
    q8 = rng.integers(-127, 128, (1, 1, n, d)).astype(np.int8)
    qs = (0.01 + 0.01 * rng.random((1, 1, 4))).astype(np.float32)
    k8 = rng.integers(-127, 128, (1, 1, n, d)).astype(np.int8)
    ks = (0.01 + 0.01 * rng.random((1, 1, 2))).astype(np.float32)
    v8t = rng.integers(0, 0x7E, (1, 1, d, 128)).astype(np.uint8)
    vs = (0.1 + rng.random((1, 1, d))).astype(np.float32)
    e = rng.integers(-3, 4, d)
    base, _, _ = O.attention(q8, qs, k8, ks, v8t, vs, n)
    moved, _, _ = O.attention(q8, qs, k8, ks, v8t, (vs * 2.0 ** e).astype(np.float32), n)
    expect = f32_from_bf16_bits(base) * (2.0 ** e).astype(np.float32)
    assert np.array_equal(f32_from_bf16_bits(moved), expect)


def test_batch_entries_are_independent_problems():
    # each batch entry is its own problem (per-(b, h) means, scales and softmax):
    # the B = 2 pipeline equals the two B = 1 pipelines stacked, bit for bit
    w = synth.custom(23, 2, 140, 2, 64, rope=False)
    both = O.pipeline(w.q, w.k, w.v, w.q_weight, w.k_weight, w.eps, w.rotary_dim, w.theta)
    for b in range(2):
        one = O.pipeline(w.q[b:b + 1], w.k[b:b + 1], w.v[b:b + 1], w.q_weight, w.k_weight,
                         w.eps, w.rotary_dim, w.theta)
        for key in ("q8", "q_scale", "k8", "k_scale", "k_mean", "v8t", "v_scale", "out"):
            assert np.array_equal(both[key][b:b + 1], one[key]), (b, key)


def test_row_sample_is_exact():
    w = synth.custom(22, 1, 300, 2, 64, rope=False)
    q8, qs = O.quant_q(w.q)
    k8, ks = O.quant_k(w.k, O.k_mean(w.k))
    v8t, vs = O.quant_v(w.v)
    full, _, _ = O.attention(q8, qs, k8, ks, v8t, vs, 300)
    rows = np.array([0, 31, 32, 128, 299])
    part, _, _ = O.attention(q8, qs, k8, ks, v8t, vs, 300, rows=rows)
    assert np.array_equal(full[:, rows], part)


# ================================================================ Hadamard
def _sylvester(n):
    h = np.array([[1.0]])
    while h.shape[0] < n:
        h = np.block([[h, h], [h, -h]])
    return h


def test_fwht_equals_dense_sylvester_matrix():
    rng = np.random.default_rng(16)
    for n in (4, 64, 256):
        x = rng.standard_normal((5, n)).astype(np.float32)
        hm = _sylvester(n)
        assert np.array_equal(hm @ hm.T, n * np.eye(n))
        got = O.fwht(x).astype(np.float64)
        ref = x.astype(np.float64) @ hm            # symmetric: x H == (H x^T)^T
        assert np.allclose(got, ref, rtol=0, atol=1e-4 * np.abs(ref).max())
    # an exactly representable case is bit exact
    x = np.zeros((1, 256), np.float32)
    x[0, 3] = 1.0
    assert np.array_equal(O.fwht(x)[0], _sylvester(256)[3].astype(np.float32))


def test_hadamard_rotation_preserves_scores():
    rng = np.random.default_rng(17)
    q = _bf(rng.standard_normal((1, 64, 1, 256)))
    k = _bf(rng.standard_normal((1, 96, 1, 256)))
    qr, kr = O.hadamard_rotate(q), O.hadamard_rotate(k)
    s0 = _f(q)[0, :, 0] @ _f(k)[0, :, 0].T
    s1 = qr[0, :, 0].astype(np.float64) @ kr[0, :, 0].astype(np.float64).T
    rel = np.abs(s1 - s0).max() / np.abs(s0).max()
    assert rel <= 1e-6          # page reports 1.6e-9 relative in f32; FP32 FWHT here


def test_hadamard_int8_k_per_token_scales():
    w = synth.make("gqa_chunk", Nq=64, Nkv=200)
    q8, qs, k8, ks16, v8t, vs = O.quant_hadamard(w.q, w.k, w.v)
    assert q8.shape == (1, 16, 64, 256) and qs.shape == (1, 16, 4)
    assert k8.shape == (1, 4, 200, 256) and ks16.shape == (1, 4, 200)
    kr = O.hadamard_rotate(w.k).transpose(0, 2, 1, 3).astype(np.float64)
    sc = f32_from_f16_bits(ks16).astype(np.float64)
    assert np.allclose(sc, np.abs(kr).max(-1) / 127.0, rtol=2 ** -11)
    assert np.all(np.abs(k8).max(-1) == 127)


def _kld_int8_k(k_bits, q_f, rotate, rng):
    """Attention-weight KLD of an int8 (per token) K cache against the BF16 K."""
    kf = _f(k_bits)[0, :, 0]
    if rotate:
        k_use = O.hadamard_rotate(k_bits)[0, :, 0].astype(np.float64)
        q_use = O.hadamard_rotate(_bf(q_f[None, :, None]))[0, :, 0].astype(np.float64)
    else:
        k_use, q_use = kf, _f(_bf(q_f[None, :, None]))[0, :, 0]
    amax = np.maximum(1e-7, np.abs(k_use).max(-1, keepdims=True))
    kq = np.clip(np.rint(k_use * (127.0 / amax)), -128, 127) * (amax / 127.0)
    s_ref = (_f(_bf(q_f[None, :, None]))[0, :, 0] @ kf.T) / 16.0
    s_q = (q_use @ kq.T) / 16.0
    p = np.exp(s_ref - s_ref.max(1, keepdims=True)); p /= p.sum(1, keepdims=True)
    r = np.exp(s_q - s_q.max(1, keepdims=True)); r /= r.sum(1, keepdims=True)
    return float(np.mean(np.sum(p * (np.log(p) - np.log(r)), axis=1)))


def test_hadamard_reduces_kld_with_outlier_channels():
    # page "npu plan P7", PR #1273: with 8x outlier channels the rotated int8 K is
    # about an order of magnitude closer than the unrotated one.  Statistical check.
    rng = np.random.default_rng(18)
    un, ro = [], []
    for _ in range(4):
        k = rng.standard_normal((512, 256))
        k[:, rng.choice(256, 13, replace=False)] *= 8.0
        kb = _bf(k[None, :, None])
        q = rng.standard_normal((16, 256))
        un.append(_kld_int8_k(kb, q, False, rng))
        ro.append(_kld_int8_k(kb, q, True, rng))
    assert np.mean(ro) < 0.3 * np.mean(un)
    assert np.mean(ro) < 1e-3


def _f32_round_exact(fr):
    """Correct float32 rounding of a Fraction (nearest, ties to even)."""
    from fractions import Fraction
    c = np.float32(float(fr))
    cands = [np.nextafter(c, np.float32(-np.inf)), c, np.nextafter(c, np.float32(np.inf))]
    best = None
    for v in cands:
        d = abs(Fraction(float(v)) - fr)
        if best is None or d < best[0] or (d == best[0] and (int(np.float32(v).view(np.uint32)) & 1) == 0):
            best = (d, v)
    return best[1]


def test_fused_probability_exponent_is_a_single_rounding():
    # the oracle evaluates fma(S, A, -m) as float64 arithmetic rounded to float32;
    # check it against exact rational arithmetic over the regimes the path produces
    from fractions import Fraction
    rng = np.random.default_rng(19)
    n_ok = 0
    for _ in range(3000):
        S = int(rng.integers(-2_064_512, 2_064_513))
        A = np.float32(np.exp2(rng.uniform(-30, 0)) * rng.uniform(1, 2))
        mn = np.float32(rng.choice([1.0, 1e-6, 1e3]) * rng.standard_normal())
        emu = np.float32(np.float64(S) * np.float64(A) - np.float64(mn))
        exact = _f32_round_exact(Fraction(S) * Fraction(float(A)) - Fraction(float(mn)))
        assert emu == exact, (S, A, mn)
        n_ok += 1
    assert n_ok == 3000
