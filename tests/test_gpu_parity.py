"""GPU parity of the CUDA path (through the C ABI) against the CPU oracle.

Bit-exact: prepared Q/K, INT8 Q/K, their scales, the K mean, FP8 V and its
scales, and the INT32 score tiles as the attention mainloop itself computes them.  Tolerance (max-abs <= 2e-2, rel-L2 <= 5e-3): the
BF16 attention output."""
import numpy as np
import pytest
import torch

import quantized_exact_attention_qattn_b200 as qa
from quantized_exact_attention_qattn_b200 import synth
from oracle import qattn_oracle as O

from gpu_helpers import (DEV, SENTINEL, assert_out_close, assert_scores_tile, dev_bf16, host,
                         hot_path_scores, oracle_full, run_pipeline)

pytestmark = pytest.mark.gpu

SMALL_CONFIGS = ["small", "mid", "encoder"]


def _check_quant(pipe, ref, w):
    if not w.hadamard:
        assert np.array_equal(host(pipe.qp), ref["qp"]), "prepared Q"
        assert np.array_equal(host(pipe.kp), ref["kp"]), "prepared K"
        assert np.array_equal(host(pipe.k_mean), ref["k_mean"]), "K mean"
    assert np.array_equal(host(pipe.q_scale), ref["q_scale"]), "Q scales"
    assert np.array_equal(host(pipe.q8), ref["q8"]), "Q int8"
    assert np.array_equal(host(pipe.k_scale), ref["k_scale"]), "K scales"
    assert np.array_equal(host(pipe.k8), ref["k8"]), "K int8"
    assert np.array_equal(host(pipe.v_scale), ref["v_scale"]), "V scales"
    assert np.array_equal(host(pipe.v8t), ref["v8t"]), "V fp8"


@pytest.mark.parametrize("name", SMALL_CONFIGS)
def test_pipeline_parity(name):
    w = synth.make(name)
    pipe = run_pipeline(w)
    ref = oracle_full(w)
    _check_quant(pipe, ref, w)
    assert_out_close(host(pipe.out), ref["out"], name)


def test_scores_all_tiles_small():
    # every tile of the small workload through the mainloop's own QK (Q in tensor
    # memory, S accumulated onto the 1.5 * 2^23 preload), including the tail keys
    w = synth.make("small")
    pipe = run_pipeline(w)
    ref = oracle_full(w)
    nq, nk = O.ceil_div(w.Nq, 128), O.ceil_div(w.Nkv, 64)
    tl = [(0, h, i, j) for h in range(w.Hq) for i in range(nq) for j in range(nk)]
    s = hot_path_scores(pipe, tl)
    for n, (b, h, i, j) in enumerate(tl):
        assert_scores_tile(s[n], ref["q8"][b, h, 128 * i:128 * i + 128],
                           ref["k8"][b, h, 64 * j:64 * j + 64], (h, i, j))


def test_scores_encoder_d64_tails():
    # D = 64 (Q in shared memory, three query tiles per CTA), B = 32: the last query
    # tile has 89 rows, the last key tile 25 keys
    w = synth.make("encoder")
    pipe = run_pipeline(w)
    nq, nk = O.ceil_div(w.Nq, 128), O.ceil_div(w.Nkv, 64)
    tl = [(b, h, i, j) for b in (0, 31) for h in (0, 15) for i in (0, 2, nq - 1)
          for j in (0, 5, nk - 1)]
    s = hot_path_scores(pipe, tl)
    q8, k8 = host(pipe.q8), host(pipe.k8)      # bit-exact against the oracle elsewhere
    ref = oracle_full(w)
    assert np.array_equal(q8, ref["q8"]) and np.array_equal(k8, ref["k8"])
    for n, (b, h, i, j) in enumerate(tl):
        assert_scores_tile(s[n], ref["q8"][b, h, 128 * i:128 * i + 128],
                           ref["k8"][b, h, 64 * j:64 * j + 64], (b, h, i, j))


def test_scores_requests_outside_the_problem_leave_slots_untouched():
    w = synth.make("small")
    pipe = run_pipeline(w)
    tl = [(0, 0, 0, 0), (0, 5, 0, 0), (1, 0, 0, 0), (0, 0, 9, 0), (0, 0, 0, 99), (0, 0, 0, 0)]
    s = hot_path_scores(pipe, tl)
    assert np.array_equal(s[0], s[5])
    for n in range(1, 5):
        assert (s[n] == SENTINEL).all(), tl[n]


@pytest.mark.parametrize("D", [64, 128, 256])
def test_scores_at_the_int8_extremes(D):
    # Codes of +-127 in every lane give the largest |S| the quantizers can produce,
    # D * 127^2 (4,129,024 at D = 256): the scores that the mainloop recovers from
    # the bits of its score-bias MMA output stay exact at both ends of the range.
    N, nq, nk = 192, 2, 3
    rng = np.random.default_rng(D)
    q8 = rng.choice(np.array([127, -127], np.int8), size=(1, 1, N, D))
    k8 = rng.choice(np.array([127, -127], np.int8), size=(1, 1, N, D))
    q8[0, 0, :40] = 127                         # rows of all +127 ...
    q8[0, 0, 130:150] = -127                    # ... and of all -127
    k8[0, 0, :20] = 127
    k8[0, 0, 64:90] = -127
    k8[0, 0, 150:170] = 127
    pipe = qa.Pipeline(1, N, N, 1, 1, D, device=DEV)
    pipe.q8.copy_(torch.from_numpy(q8))
    pipe.k8.copy_(torch.from_numpy(k8))
    pipe.q_scale.fill_(1.0 / 127)
    pipe.k_scale.fill_(1.0 / 127)
    codes = rng.integers(0, 256, size=tuple(pipe.v8t.shape), dtype=np.uint8) & 0x77   # finite E4M3
    pipe.v8t.copy_(torch.from_numpy(codes))
    pipe.v_scale.fill_(1.0)
    pipe.run_fwd()
    pipe.check()
    tl = [(0, 0, qt, kt) for qt in range(nq) for kt in range(nk)]
    s = hot_path_scores(pipe, tl)
    assert s.min() == -D * 127 * 127 and s.max() == D * 127 * 127
    for i, (_, _, qt, kt) in enumerate(tl):
        assert_scores_tile(s[i], q8[0, 0, qt * 128:(qt + 1) * 128], k8[0, 0, kt * 64:(kt + 1) * 64],
                           ("D", D, qt, kt))
