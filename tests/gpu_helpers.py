"""Helpers shared by the GPU parity tests: move synthetic inputs to the device,
run the library through its C ABI and compute the oracle for the same inputs."""
from __future__ import annotations

import numpy as np
import torch

import quantized_exact_attention_qattn_b200 as qa
from oracle import qattn_oracle as O
from oracle.encoders import f32_from_bf16_bits

# Output tolerance of the BF16 attention result against the oracle.
MAX_ABS = 2e-2
REL_L2 = 5e-3

DEV = "cuda"


def dev_bf16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).view(torch.bfloat16).to(DEV)


def host(t: torch.Tensor) -> np.ndarray:
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16 or t.dtype == torch.float16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def inputs_on_device(w):
    """Device views of q, k, v with the workload's own layout (interleaved or not)."""
    if w.qkv is not None:
        buf = torch.from_numpy(w.qkv).view(torch.bfloat16).to(DEV)
        view = buf.view(w.B, w.Nq, 3, w.Hq, w.D)
        return view[:, :, 0], view[:, :, 1], view[:, :, 2], buf
    return dev_bf16(w.q), dev_bf16(w.k), dev_bf16(w.v), None


def run_pipeline(w):
    q, k, v, _keep = inputs_on_device(w)
    pipe = qa.Pipeline(w.B, w.Nq, w.Nkv, w.Hq, w.Hkv, w.D, hadamard=w.hadamard, device=DEV)
    qw = dev_bf16(w.q_weight) if w.q_weight is not None else None
    kw = dev_bf16(w.k_weight) if w.k_weight is not None else None
    pipe.run(q, k, v, qw, kw, w.eps, w.rotary_dim, w.theta)
    pipe.check()
    torch.cuda.synchronize()
    return pipe


def out_errors(got_bits: np.ndarray, exp_bits: np.ndarray):
    g = f32_from_bf16_bits(got_bits).astype(np.float64)
    e = f32_from_bf16_bits(exp_bits).astype(np.float64)
    return float(np.max(np.abs(g - e))), float(np.linalg.norm(g - e) / np.linalg.norm(e))


def assert_out_close(got_bits, exp_bits, what=""):
    mx, rel = out_errors(got_bits, exp_bits)
    assert mx <= MAX_ABS and rel <= REL_L2, f"{what}: max_abs={mx:.3e} rel_l2={rel:.3e}"
    return mx, rel


def oracle_full(w):
    if w.hadamard:
        return O.pipeline_hadamard(w.q, w.k, w.v)
    return O.pipeline(w.q, w.k, w.v, w.q_weight, w.k_weight, w.eps, w.rotary_dim, w.theta)


SENTINEL = 0x7EADBEEF


def hot_path_scores(pipe, tiles_list, sm_scale=0.0):
    """INT32 score tiles of the quads in `tiles_list` as qattn_fwd's own kernel
    computes them (qattn_scores: the mainloop's debug build), plus a check that
    the attention output of that launch equals the pipeline's qattn_fwd output bit
    for bit (the copy-out changes nothing else).  Slots start at a sentinel, so a
    tile the kernel never reached shows up as a mismatch."""
    tiles = torch.tensor(tiles_list, dtype=torch.int32, device=DEV)
    s = torch.full((len(tiles_list), 128, 64), SENTINEL, dtype=torch.int32, device=DEV)
    out = torch.empty_like(pipe.out)
    qa.qattn_scores(pipe.B, pipe.Nq, pipe.Nkv, pipe.Hq, pipe.Hkv, pipe.D, pipe.q8, pipe.q_scale,
                    pipe.k8, pipe.k_scale, 1 if pipe.hadamard else 0, pipe.v8t, pipe.v_scale,
                    sm_scale, tiles, len(tiles_list), s, out, pipe.dev_err)
    qa.qattn_check(pipe.dev_err)
    assert torch.equal(out.view(torch.int16), pipe.out.view(torch.int16)), \
        "the score copy-out build changed the attention output"
    return host(s)


def assert_scores_tile(got, q8_rows, k8_rows, what):
    """got: one [128, 64] slot; q8_rows / k8_rows: the oracle's INT8 rows of that
    query tile / key tile (fewer than 128 / 64 at a tail).  Valid entries equal
    the integer dot products; rows past Nq and keys past Nkv read 0."""
    from oracle import qattn_oracle as O
    exp = O.scores(q8_rows, k8_rows)
    nr, nc = exp.shape
    assert np.array_equal(got[:nr, :nc], exp), what
    assert not got[nr:].any() and not got[:, nc:].any(), f"{what}: tail not zero"
