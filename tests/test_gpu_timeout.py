"""Failure detection on the GPU without a fault.

The test hook qattn_debug_stall_kv_tile makes the attention producer skip one
K/V copy, so the waits on that tile's barrier are never completed by anything.
Each such wait gives up after its bound (about one second), the kernel drains its
in-flight copies and MMAs and returns, and qattn_check reports QATTN_ERR_TIMEOUT
with the error bits.  The CUDA context stays usable: the next call, with the hook
off, gives exactly the output of the call before the failure.  Covered for the
layout with one softmax warpgroup per query tile (D=128, two query tiles with Q
in tensor memory; D=64, three query tiles with Q in shared memory) and the
layout with two threads per query row in eight warps (D=256, per-token K scales).
"""
import pytest
import torch

import quantized_exact_attention_qattn_b200 as qa
from quantized_exact_attention_qattn_b200 import synth

from gpu_helpers import run_pipeline

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name, tile", [("small", 1), ("mid", 5), ("encoder", 3), ("gqa_chunk", 7)])
def test_stalled_copy_times_out_and_the_context_recovers(name, tile):
    w = synth.make(name)
    pipe = run_pipeline(w)                      # a good call first
    good = pipe.out.clone()
    qa.qattn_debug_stall_kv_tile(tile)
    try:
        pipe.dev_err.zero_()
        pipe.out.fill_(0)
        pipe.run_fwd()
        with pytest.raises(qa.QAttnError) as err:
            pipe.check()
        assert err.value.status == 7, str(err.value)          # QATTN_ERR_TIMEOUT
        assert "error bits" in str(err.value)
    finally:
        qa.qattn_debug_stall_kv_tile(-1)
    pipe.dev_err.zero_()
    pipe.run_fwd()
    pipe.check()
    torch.cuda.synchronize()
    assert torch.equal(pipe.out.view(torch.int16), good.view(torch.int16)), name
