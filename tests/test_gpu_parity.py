"""GPU parity of the CUDA path (through the C ABI) against the CPU oracle.

Bit-exact: prepared Q/K, INT8 Q/K, their scales, the K mean, FP8 V and its
scales, INT32 score tiles.  Tolerance (max-abs <= 2e-2, rel-L2 <= 5e-3): the
BF16 attention output."""
import numpy as np
import pytest
import torch

import quantized_exact_attention_qattn_b200 as qa
from quantized_exact_attention_qattn_b200 import synth
from oracle import qattn_oracle as O

from gpu_helpers import (DEV, assert_out_close, dev_bf16, host, oracle_full, run_pipeline)

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
    w = synth.make("small")
    pipe = run_pipeline(w)
    ref = oracle_full(w)
    nq, nk = O.ceil_div(w.Nq, 128), O.ceil_div(w.Nkv, 64)
    tl = [(0, h, i, j) for h in range(w.Hq) for i in range(nq) for j in range(nk)]
    tiles = torch.tensor(tl, dtype=torch.int32, device=DEV)
    s = torch.empty((len(tl), 128, 64), dtype=torch.int32, device=DEV)
    qa.qattn_scores(w.B, w.Nq, w.Nkv, w.Hq, w.Hkv, w.D, pipe.q8, pipe.k8, tiles, len(tl), s,
                    pipe.dev_err)
    qa.qattn_check(pipe.dev_err)
    s = host(s)
    full = O.scores(ref["q8"], ref["k8"])          # [B,H,Nq,Nk]
    for n, (b, h, i, j) in enumerate(tl):
        exp = full[b, h, 128 * i:128 * i + 128, 64 * j:64 * j + 64]
        assert np.array_equal(s[n, :exp.shape[0], :exp.shape[1]], exp), (h, i, j)
