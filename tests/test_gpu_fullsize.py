"""Full-size parity at the canonical call (B1 N37810 H56 D128, interleaved QKV,
the launch configuration the benchmark times) and at the GQA prefill chunk
(Nq1024 x Nkv32768, 16/4 heads, D256, Hadamard-rotated int8 K).

The oracle is evaluated head by head (every prep/quant quantity is per head),
on all keys, and on a fixed sample of query tiles; rows are independent, so a
sampled row is computed exactly as in a full run."""
import numpy as np
import pytest
import torch

import quantized_exact_attention_qattn_b200 as qa
from quantized_exact_attention_qattn_b200 import synth
from oracle import qattn_oracle as O

from gpu_helpers import assert_out_close, assert_scores_tile, host, hot_path_scores, run_pipeline

pytestmark = pytest.mark.gpu

Q_TILES = (0, 1, 147, 294, 295)
SCORE_Q = (0, 147, 295)
SCORE_K = (0, 295, 590)
SCORE_H = (0, 27, 55)


@pytest.fixture(scope="module")
def canonical():
    w = synth.make("canonical")
    pipe = run_pipeline(w)
    return w, pipe


def _rows(n, tiles):
    return np.concatenate([np.arange(128 * t, min(n, 128 * t + 128)) for t in tiles])


def test_canonical_prep_quant_bit_exact(canonical):
    w, pipe = canonical
    rows = _rows(w.Nq, Q_TILES)
    groups = np.concatenate([np.arange(4 * t, 4 * t + 4) for t in Q_TILES])
    kp_g, k8_g, ks_g, mu_g = host(pipe.kp), host(pipe.k8), host(pipe.k_scale), host(pipe.k_mean)
    v8_g, vs_g = host(pipe.v8t), host(pipe.v_scale)
    qp_g, q8_g, qs_g = host(pipe.qp), host(pipe.q8), host(pipe.q_scale)
    for h0 in range(0, w.Hq, 8):
        hs = slice(h0, h0 + 8)
        kp = O.prep(np.ascontiguousarray(w.k[:, :, hs]), w.k_weight, w.eps, w.rotary_dim, w.theta)
        assert np.array_equal(kp_g[:, :, hs], kp), f"prepared K heads {h0}.."
        mu = O.k_mean(kp)
        assert np.array_equal(mu_g[:, hs], mu), f"K mean heads {h0}.."
        k8, ks = O.quant_k(kp, mu)
        assert np.array_equal(ks_g[:, hs], ks) and np.array_equal(k8_g[:, hs], k8), f"K int8 {h0}"
        v8t, vs = O.quant_v(np.ascontiguousarray(w.v[:, :, hs]))
        assert np.array_equal(vs_g[:, hs], vs) and np.array_equal(v8_g[:, hs], v8t), f"V fp8 {h0}"
        qp = O.prep(np.ascontiguousarray(w.q[:, rows][:, :, hs]), w.q_weight, w.eps, w.rotary_dim,
                    w.theta, positions=rows)
        assert np.array_equal(qp_g[:, rows][:, :, hs], qp), f"prepared Q {h0}"
        q8, qs = O.quant_q(qp)
        assert np.array_equal(q8_g[:, hs][:, :, rows], q8), f"Q int8 {h0}"
        assert np.array_equal(qs_g[:, hs][:, :, groups], qs), f"Q scales {h0}"


def test_canonical_scores_bit_exact(canonical):
    # the INT32 scores of qattn_fwd's own QK (the launch the benchmark times),
    # query tiles {0, 147, 295 (50-row tail)} x key tiles {0, 295, 590 (50-key tail)}
    w, pipe = canonical
    tl = [(0, h, i, j) for h in SCORE_H for i in SCORE_Q for j in SCORE_K]
    s = hot_path_scores(pipe, tl)
    # oracle INT8 operands of the sampled heads, from the inputs alone
    hs = list(SCORE_H)
    rows = _rows(w.Nq, SCORE_Q)
    kp = O.prep(np.ascontiguousarray(w.k[:, :, hs]), w.k_weight, w.eps, w.rotary_dim, w.theta)
    k8, _ = O.quant_k(kp, O.k_mean(kp))
    qp = O.prep(np.ascontiguousarray(w.q[:, rows][:, :, hs]), w.q_weight, w.eps, w.rotary_dim,
                w.theta, positions=rows)
    q8, _ = O.quant_q(qp)
    starts = {t: 128 * k for k, t in enumerate(SCORE_Q)}
    for n, (b, h, i, j) in enumerate(tl):
        hi = hs.index(h)
        r0 = starts[i]
        nrows = min(128, w.Nq - 128 * i)
        assert_scores_tile(s[n], q8[b, hi, r0:r0 + nrows], k8[b, hi, 64 * j:64 * j + 64], (h, i, j))


def test_canonical_output_sampled_rows(canonical):
    w, pipe = canonical
    rows = _rows(w.Nq, Q_TILES)
    out_g = host(pipe.out)[:, rows]
    for h0 in range(0, w.Hq, 14):
        hs = slice(h0, h0 + 14)
        kp = O.prep(np.ascontiguousarray(w.k[:, :, hs]), w.k_weight, w.eps, w.rotary_dim, w.theta)
        k8, ks = O.quant_k(kp, O.k_mean(kp))
        v8t, vs = O.quant_v(np.ascontiguousarray(w.v[:, :, hs]))
        qp = O.prep(np.ascontiguousarray(w.q[:, rows][:, :, hs]), w.q_weight, w.eps, w.rotary_dim,
                    w.theta, positions=rows)
        q8, qs = O.quant_q(qp)
        out, _, _ = O.attention(q8, qs, k8, ks, v8t, vs, w.Nkv)
        assert_out_close(out_g[:, :, hs], out, f"canonical heads {h0}..{h0 + 13}")


def test_gqa_chunk_hadamard_full():
    w = synth.make("gqa_chunk")
    pipe = run_pipeline(w)
    ref = O.pipeline_hadamard(w.q, w.k, w.v)
    for key in ("q8", "q_scale", "k8", "k_scale", "v8t", "v_scale"):
        assert np.array_equal(host(getattr(pipe, key)), ref[key]), key
    assert_out_close(host(pipe.out), ref["out"], "gqa_chunk")
    # D = 256 split softmax (Q in tensor memory, QK overwriting S, integer-to-float
    # conversion by the warps), GQA head mapping h -> h / 4, per-token K scales
    tl = [(0, h, i, j) for h in (0, 5, 15) for i in (0, 7) for j in (0, 255, 511)]
    s = hot_path_scores(pipe, tl)
    for n, (b, h, i, j) in enumerate(tl):
        assert_scores_tile(s[n], ref["q8"][b, h, 128 * i:128 * i + 128],
                           ref["k8"][b, h // 4, 64 * j:64 * j + 64], (h, i, j))
