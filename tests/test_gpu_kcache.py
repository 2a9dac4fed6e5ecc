"""GPU parity of the chunked-prefill key cache (page "npu plan P7": int8 K
rotated by a per-head Hadamard with a per-token FP16 scale sidecar, V in 16
bits, prefill in 1024/2048-token chunks).  Three chunks are appended one after
the other; after each, the cache contents equal the oracle's bit for bit and a
query chunk's attention over every key cached so far is within the output
tolerance of the oracle's."""
import numpy as np
import pytest
import torch

import quantized_exact_attention_qattn_b200 as qa
from quantized_exact_attention_qattn_b200 import synth
from oracle import qattn_oracle as O

from gpu_helpers import DEV, assert_out_close, dev_bf16, host

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("chunks,Hq,Hkv,D,seed", [((1024, 1024, 1000), 16, 4, 256, 51),
                                                  ((200, 96, 77), 4, 2, 64, 52)])
def test_kcache_three_chunks(chunks, Hq, Hkv, D, seed):
    n_tot = sum(chunks)
    w = synth.make("gqa_chunk", Nq=chunks[0], Nkv=n_tot, Hq=Hq, Hkv=Hkv, D=D, seed=seed)
    cap = 8 * -(-(n_tot + 16) // 8)
    cache = qa.KCache(w.B, Hkv, D, cap, device=DEV)
    ref = O.kcache_new(w.B, Hkv, D, cap)
    k, v = dev_bf16(w.k), dev_bf16(w.v)
    q = dev_bf16(w.q)
    n0 = 0
    for c, n in enumerate(chunks):
        cache.append(k[:, n0:n0 + n], v[:, n0:n0 + n])
        O.kcache_append(ref, w.k[:, n0:n0 + n], w.v[:, n0:n0 + n])
        n0 += n
        out = cache.attend(q)
        cache.check()
        assert cache.n == ref["n"] == n0
        assert np.array_equal(host(cache.k8)[:, :, :n0], ref["k8"][:, :, :n0]), c
        assert np.array_equal(host(cache.k_scale)[:, :, :n0], ref["k_scale"][:, :, :n0]), c
        assert np.array_equal(host(cache.v16)[..., :n0], ref["v16"][..., :n0]), c
        assert_out_close(host(out), O.kcache_attend(ref, w.q), f"chunk {c}")
