"""Seeded synthetic inputs shaped like the workloads on the pages.

This module holds none of the attention method's arithmetic: it draws random
numbers, adds the offsets the workload recipe names and stores BF16.  Both the
CUDA path (tests, bench, smoke) and the CPU oracle consume exactly these bytes.
It imports nothing else from this package, so loading it never loads the CUDA
library.

Recipe (numpy PCG64, ``default_rng(seed)``, float32 standard normals rounded
once to BF16 round-to-nearest-even):

* ``small``      B1 N256  H2  D128, contiguous Q/K/V, seed 0
* ``mid``        B1 N4096 H8  D128, contiguous Q/K/V, seed 1
* ``canonical``  B1 N37810 H56 D128, one interleaved QKV buffer [N, 21504]
                 with Q/K/V at element offsets 0/7168/14336, seed 2
* ``encoder``    B32 N729 H16 D64, contiguous, no K offset, no RoPE, seed 3
* ``gqa_chunk``  B1 Nq1024 Nkv32768 Hq16 Hkv4 D256, seed 4; K has a fixed 5%
                 of dims (13 of 256, per KV head, drawn from the seed) scaled
                 by 8 (outlier channels); no norm, no RoPE (rotated int8 K)

Q, K, V ~ N(0, 1).  Except for ``encoder`` and ``gqa_chunk``, K gets a
per-(head, dim) offset ~ N(0, 2^2).  RMSNorm weights are 1 + 0.1 N(0, 1),
drawn separately for Q and K (shape [D]), eps 1e-5; split-half RoPE on dims
0..95 with theta 10000 at positions 0..N-1.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch

CONFIG_NAMES = ("small", "mid", "canonical", "encoder", "gqa_chunk")


def _bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 numpy -> BF16 bit patterns (uint16), round to nearest even."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


@dataclass
class Workload:
    """One synthetic problem.  BF16 tensors are uint16 bit-pattern arrays in
    [B, N, H, D] order (views into ``qkv`` for the interleaved layout)."""
    name: str
    B: int
    Nq: int
    Nkv: int
    Hq: int
    Hkv: int
    D: int
    q: np.ndarray
    k: np.ndarray
    v: np.ndarray
    q_weight: np.ndarray | None
    k_weight: np.ndarray | None
    eps: float
    rotary_dim: int
    theta: float
    hadamard: bool
    qkv: np.ndarray | None = None          # interleaved buffer when present
    extra: dict = field(default_factory=dict)

    @property
    def attn_ops(self) -> float:
        """4 * B * Hq * Nq * Nkv * D (QK^T and PV multiply-adds, x2)."""
        return 4.0 * self.B * self.Hq * self.Nq * self.Nkv * self.D


def _normals(rng, shape) -> np.ndarray:
    return rng.standard_normal(shape, dtype=np.float32)


def _contig(name, seed, B, N, H, D, k_offset=True, rope=True, Hkv=None, Nkv=None):
    rng = np.random.default_rng(seed)
    Hkv = H if Hkv is None else Hkv
    Nkv = N if Nkv is None else Nkv
    q = _normals(rng, (B, N, H, D))
    k = _normals(rng, (B, Nkv, Hkv, D))
    v = _normals(rng, (B, Nkv, Hkv, D))
    if k_offset:
        k = k + 2.0 * _normals(rng, (Hkv, D))[None, None]
    qw = 1.0 + 0.1 * _normals(rng, (D,))
    kw = 1.0 + 0.1 * _normals(rng, (D,))
    return Workload(name, B, N, Nkv, H, Hkv, D, _bf16_bits(q), _bf16_bits(k), _bf16_bits(v),
                    _bf16_bits(qw), _bf16_bits(kw), 1e-5, 96 if (rope and D >= 96) else 0,
                    10000.0, False)


def _canonical(seed=2, N=37810, H=56, D=128):
    rng = np.random.default_rng(seed)
    width = 3 * H * D
    qkv = np.empty((N, width), dtype=np.uint16)
    koff = 2.0 * _normals(rng, (H * D,))
    chunk = 2048
    for r0 in range(0, N, chunk):
        r1 = min(N, r0 + chunk)
        blk = _normals(rng, (r1 - r0, width))
        blk[:, H * D:2 * H * D] += koff[None, :]
        qkv[r0:r1] = _bf16_bits(blk)
    qw = _bf16_bits(1.0 + 0.1 * _normals(rng, (D,)))
    kw = _bf16_bits(1.0 + 0.1 * _normals(rng, (D,)))
    view = qkv.reshape(1, N, 3, H, D)
    return Workload("canonical", 1, N, N, H, H, D, view[:, :, 0], view[:, :, 1], view[:, :, 2],
                    qw, kw, 1e-5, 96, 10000.0, False, qkv=qkv)


def _gqa_chunk(seed=4, Nq=1024, Nkv=32768, Hq=16, Hkv=4, D=256):
    rng = np.random.default_rng(seed)
    q = _normals(rng, (1, Nq, Hq, D))
    k = _normals(rng, (1, Nkv, Hkv, D))
    v = _normals(rng, (1, Nkv, Hkv, D))
    n_out = max(1, round(0.05 * D))
    chans = np.stack([rng.choice(D, size=n_out, replace=False) for _ in range(Hkv)])
    for h in range(Hkv):
        k[:, :, h, chans[h]] *= 8.0
    return Workload("gqa_chunk", 1, Nq, Nkv, Hq, Hkv, D, _bf16_bits(q), _bf16_bits(k),
                    _bf16_bits(v), None, None, 1e-5, 0, 10000.0, True,
                    extra={"outlier_channels": chans})


def make(name: str, **overrides) -> Workload:
    """Build the named workload; keyword overrides shrink sizes for tests."""
    if name == "small":
        kw = dict(seed=0, B=1, N=256, H=2, D=128)
        kw.update(overrides)
        return _contig("small", **kw)
    if name == "mid":
        kw = dict(seed=1, B=1, N=4096, H=8, D=128)
        kw.update(overrides)
        return _contig("mid", **kw)
    if name == "canonical":
        return _canonical(**overrides)
    if name == "encoder":
        kw = dict(seed=3, B=32, N=729, H=16, D=64, k_offset=False, rope=False)
        kw.update(overrides)
        return _contig("encoder", **kw)
    if name == "gqa_chunk":
        return _gqa_chunk(**overrides)
    raise KeyError(name)


def custom(seed, B, N, H, D, *, k_offset=True, rope=True, Hkv=None, Nkv=None,
           name="custom") -> Workload:
    """A contiguous workload of arbitrary size with the standard recipe
    (GQA when ``Hkv`` < ``H``; cross-length when ``Nkv`` != ``N``, which
    the RoPE/RMSNorm preparation does not accept)."""
    return _contig(name, seed, B, N, H, D, k_offset=k_offset, rope=rope, Hkv=Hkv, Nkv=Nkv)
