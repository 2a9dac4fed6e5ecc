"""qattn_attention_host: host Q/K/V in, host output back, chunks of KV heads
streamed through two device buffer sets on three streams.

Every (batch, KV head) is an independent problem, so the chunked call must give
the device pipeline's output bit for bit, for any chunk size (ragged last chunks
included), strided interleaved host inputs, several batch entries and the
Hadamard GQA path.  One small case is also held against the oracle.
"""
import numpy as np
import pytest
import torch

import quantized_exact_attention_qattn_b200 as qa
from quantized_exact_attention_qattn_b200 import synth

from gpu_helpers import DEV, assert_out_close, dev_bf16, host, oracle_full, run_pipeline

pytestmark = pytest.mark.gpu


def host_inputs(w):
    """Pinned host views of q, k, v in the workload's own layout, plus the owner."""
    if w.qkv is not None:
        buf = torch.from_numpy(w.qkv).view(torch.bfloat16).pin_memory()
        view = buf.view(w.B, w.Nq, 3, w.Hq, w.D)
        return view[:, :, 0], view[:, :, 1], view[:, :, 2], buf
    pin = lambda a: torch.from_numpy(np.ascontiguousarray(a)).view(torch.bfloat16).pin_memory()
    return pin(w.q), pin(w.k), pin(w.v), None


def run_host(w, chunk, copy_streams=True):
    q, k, v, _keep = host_inputs(w)
    runner = qa.HostRunner(w.B, w.Nq, w.Nkv, w.Hq, w.Hkv, w.D, hadamard=w.hadamard,
                           kv_heads_per_chunk=chunk, device=DEV)
    if not copy_streams:
        runner.compute2 = runner.h2d = runner.d2h = None
    out = torch.empty((w.B, w.Nq, w.Hq, w.D), dtype=torch.bfloat16).pin_memory()
    out.view(torch.int16).fill_(0x7fc0)                      # NaN sentinel: every element is written
    qw = dev_bf16(w.q_weight) if w.q_weight is not None else None
    kw = dev_bf16(w.k_weight) if w.k_weight is not None else None
    runner.run(q, k, v, out, qw, kw, w.eps, w.rotary_dim, w.theta)
    runner.check()
    torch.cuda.synchronize()
    return out


@pytest.mark.parametrize("chunk", [1, 3, 8])
def test_host_pipeline_equals_device_pipeline(chunk):
    w = synth.make("mid")                                    # B1 N4096 H8 D128, norm + RoPE
    got = run_host(w, chunk)
    ref = run_pipeline(w).out.cpu()
    assert torch.equal(got.view(torch.int16), ref.view(torch.int16)), chunk


def test_host_pipeline_ramped_chunks():
    # 16 KV heads in chunks of 2: eight or more chunks, so the first two are
    # shortened (1 and 1 heads) and the rest follow at 2
    w = synth.custom(31, 1, 700, 16, 128)
    got = run_host(w, 2)
    ref = run_pipeline(w).out.cpu()
    assert torch.equal(got.view(torch.int16), ref.view(torch.int16))


def test_host_pipeline_interleaved_inputs_and_serial_copies():
    w = synth.make("canonical", N=700, H=6)                  # interleaved [N, 3*H*D] host buffer
    ref = run_pipeline(w).out.cpu()
    for chunk, streams in ((4, True), (2, False)):
        got = run_host(w, chunk, copy_streams=streams)
        assert torch.equal(got.view(torch.int16), ref.view(torch.int16)), (chunk, streams)


def test_host_pipeline_batch_entries():
    w = synth.custom(21, 2, 333, 4, 64, rope=False)
    got = run_host(w, 3)
    ref = run_pipeline(w).out.cpu()
    assert torch.equal(got.view(torch.int16), ref.view(torch.int16))


def test_host_pipeline_hadamard_gqa():
    w = synth.make("gqa_chunk", Nq=200, Nkv=700, Hq=8, Hkv=2, D=256, seed=9)
    got = run_host(w, 1)
    ref = run_pipeline(w).out.cpu()
    assert torch.equal(got.view(torch.int16), ref.view(torch.int16))


def test_host_pipeline_against_the_oracle():
    w = synth.make("small")
    got = run_host(w, 1)
    assert_out_close(host(got), oracle_full(w)["out"], "host pipeline, small")
