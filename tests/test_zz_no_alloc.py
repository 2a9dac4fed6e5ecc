"""The allocation-free quantizer entry point.

qattn_quant_noalloc serves callers that cannot allocate device memory while
they quantize: an embedder whose memory manager owns all device memory and hands
out only the tensors, or a runtime that must not allocate on its hot path because
cudaMalloc and cudaFree can synchronize the device.  Its reduction scratch is a
static device array inside the library.  It must give exactly what qattn_quant gives with a
caller-provided workspace, on consecutive calls that reuse the same array, and
refuse problems whose scratch would not fit.  This file is collected last so a
stop-at-first-failure run has already run every other test.
"""
import numpy as np
import pytest
import torch

import quantized_exact_attention_qattn_b200 as qa
from quantized_exact_attention_qattn_b200 import _lib, synth

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _bf(a):
    return torch.from_numpy(np.ascontiguousarray(a)).view(torch.bfloat16).to(DEV)


def _outputs(B, Nq, Nkv, Hq, Hkv, D, fill):
    nq, nk = -(-Nq // 128), -(-Nkv // 64)
    kw = dict(device=DEV)
    return dict(
        q8=torch.full((B, Hq, Nq, D), fill, dtype=torch.int8, **kw),
        q_scale=torch.full((B, Hq, 4 * nq), float(fill), dtype=torch.float32, **kw),
        k8=torch.full((B, Hkv, Nkv, D), fill, dtype=torch.int8, **kw),
        k_scale=torch.full((B, Hkv, nk), float(fill), dtype=torch.float32, **kw),
        k_mean=torch.full((B, Hkv, D), float(fill), dtype=torch.float32, **kw),
        v8t=torch.full((B, Hkv, D, 64 * nk), fill & 0xFF, dtype=torch.uint8, **kw),
        v_scale=torch.full((B, Hkv, D), float(fill), dtype=torch.float32, **kw),
    )


def _run_both(w):
    q, k, v = _bf(w.q), _bf(w.k), _bf(w.v)
    args = (w.B, w.Nq, w.Nkv, w.Hq, w.Hkv, w.D, q, k, v)
    ref = _outputs(w.B, w.Nq, w.Nkv, w.Hq, w.Hkv, w.D, 3)
    ws = torch.empty(qa.qattn_quant_workspace_bytes(w.B, w.Nkv, w.Hkv, w.D), dtype=torch.uint8,
                     device=DEV)
    qa.qattn_quant(*args, ref["q8"], ref["q_scale"], ref["k8"], ref["k_scale"], ref["k_mean"],
                   ref["v8t"], ref["v_scale"], ws)
    got = _outputs(w.B, w.Nq, w.Nkv, w.Hq, w.Hkv, w.D, 5)
    qa.qattn_quant_noalloc(*args, got["q8"], got["q_scale"], got["k8"], got["k_scale"],
                           got["k_mean"], got["v8t"], got["v_scale"])
    torch.cuda.synchronize()
    return ref, got


def test_noalloc_matches_workspace_entry_point_on_consecutive_calls():
    # two calls in a row on different problems: the second reuses the static
    # scratch the first left behind
    for w in (synth.make("mid"), synth.custom(77, 2, 333, 3, 64, rope=False)):
        ref, got = _run_both(w)
        for key in ref:
            assert torch.equal(ref[key], got[key]), (w.name, key)


def test_noalloc_refuses_problems_beyond_its_scratch():
    need = qa.qattn_quant_workspace_bytes(1, 37810, 56, 128)
    assert need > 16 << 20
    big = torch.empty(128, dtype=torch.bfloat16, device=DEV)
    view = _lib.bnhd(big.view(1, 1, 1, 128).expand(1, 37810, 56, 128))
    lib = qa.load()
    st = lib.qattn_quant_noalloc(1, 37810, 37810, 56, 56, 128, view, view, view, big.data_ptr(),
                                 big.data_ptr(), big.data_ptr(), big.data_ptr(), big.data_ptr(),
                                 big.data_ptr(), big.data_ptr(), None)
    assert st == 5 and "static array" in lib.qattn_last_error().decode()
