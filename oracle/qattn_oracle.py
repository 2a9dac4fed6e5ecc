"""Plain, slow CPU oracle of the quantized attention prefill path.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
the ``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import
this module.  It shares no code with the CUDA library and imports nothing
from it; the inputs come from the seeded generators (``synth``), which hold
none of the method's arithmetic.

Authority: the page "Exact Numerical Contract" (SageAttention-2.2.0-derived
INT8-QK / FP8-PV attention).  Section names below refer to that page unless
another page is named.  The Hadamard-rotated int8-K variant follows the page
"npu plan P7: int8 KV with per-head Hadamard rotation" (design note and the
PR #1273 comment).

Arrays use numpy.  BF16 tensors are carried as uint16 bit patterns, E4M3 as
uint8 bit patterns, FP16 scales as uint16 bit patterns.  Where the page fixes
FP32 arithmetic the oracle computes in float32 with one IEEE rounding per
operation (numpy float32 ufuncs, no fused multiply-add); elsewhere it uses
float64.  Where the pages are silent the oracle takes one plain reading,
listed in the design notes and repeated at each function.

Parity pins: every function is pinned by ``tests/test_oracle_pins.py``
(closed forms, hand-built rows, brute force on tiny inputs, FP64 attention,
identities).  None is "parity unpinned".
"""
from __future__ import annotations

import math

import numpy as np

from .encoders import (bf16_bits_from_f32, bf16_bits_from_f64, f32_from_bf16_bits,
                       e4m3_bits_from_f32, e4m3_value_from_f32, f32_from_e4m3_bits, f16_bits_from_f32,
                       f32_from_f16_bits)

F32 = np.float32

#: Initial running maximum, FP8 probability offset (log2 448 rounded down) and
#: the masked-score value ("Online Softmax", "Finalization And Tails").
M_INIT = F32(-5000000.0)
FP8_OFFSET = F32(8.807)
MASKED_SCORE = F32(-5000000.0)
#: Floor of every quantization maximum ("Q And K Quantization").
AMAX_FLOOR = F32(1e-7)
#: V scaling constant ("V And PV").
V_RANGE = F32(2.25)
Q_ROWS_PER_SCALE = 32
Q_ROWS_PER_CTA = 128
K_ROWS_PER_SCALE = 64
KV_TILE = 64


def ceil_div(a: int, b: int) -> int:
    return -(-a // b)


# ============================================================ preparation
def rope_tables(n_pos: int, rotary_dim: int, theta: float, pos_offset: int = 0,
                positions=None):
    """BF16 cos/sin coefficients for split-half RoPE ("Preparation" step 3).

    Reading (the page says only "BF16 coefficients"): frequency
    ``theta^(-(2i)/R)`` for pair i < R/2, angle ``pos * freq``, cos and sin,
    all in FP64, each rounded once to BF16 RN.  Positions are
    ``pos_offset + 0..n_pos-1`` unless ``positions`` lists them.  Returns two
    uint16 arrays of shape [n_pos, R/2].
    """
    half = rotary_dim // 2
    i = np.arange(half, dtype=np.float64)
    inv_freq = np.power(np.float64(theta), -(2.0 * i) / np.float64(rotary_dim))
    if positions is None:
        positions = np.arange(n_pos, dtype=np.int64) + pos_offset
    pos = np.asarray(positions, dtype=np.int64).astype(np.float64)
    ang = pos[:, None] * inv_freq[None, :]
    return bf16_bits_from_f64(np.cos(ang)), bf16_bits_from_f64(np.sin(ang))


def rms_sum_of_squares(x: np.ndarray) -> np.ndarray:
    """Sum of squares over the last axis (D) in a fixed FP32 order.

    Reading of "the production reduction order" (not retained by the page):
    the row is split into L = D/8 lanes of 8 consecutive dims.  Each lane sums
    its 8 squares left to right in FP32; then, for off = L/2, ..., 2, 1, every
    lane adds the partial of lane ``l XOR off`` (all lanes at once).  The
    result is lane 0's value.  Squares of BF16 values are exact in FP32.
    """
    d = x.shape[-1]
    lanes = d // 8
    sq = (x * x).astype(F32).reshape(*x.shape[:-1], lanes, 8)
    p = sq[..., 0]
    for k in range(1, 8):
        p = (p + sq[..., k]).astype(F32)
    idx = np.arange(lanes)
    off = lanes // 2
    while off >= 1:
        p = (p + p[..., idx ^ off]).astype(F32)
        off //= 2
    return p[..., 0]


def prep(x_bits: np.ndarray, weight_bits, eps: float, rotary_dim: int,
         theta: float = 10000.0, pos_offset: int = 0, positions=None) -> np.ndarray:
    """Per-head RMSNorm then split-half RoPE on one BF16 [B,N,H,D] tensor.

    "Preparation" steps 1-3:
      r = 1 / sqrt(mean(x^2) + eps)            (FP32, IEEE sqrt and divide)
      n = bf16_rn(x * r)                       (normalize in FP32, round BF16)
      y = bf16_rn(n * w[d])                    (reading: the weight [D], shared
                                                by all heads, multiplies the
                                                BF16-rounded normalized value;
                                                the BF16 product is exact in FP32)
      dims i < R/2:  y_i       = bf16_rn(y_i*c - y_{i+R/2}*s)
                     y_{i+R/2} = bf16_rn(y_{i+R/2}*c + y_i*s)
      dims >= R pass through.
    ``weight_bits`` None skips the norm (and its weight); ``rotary_dim`` 0
    skips RoPE.  Positions are ``pos_offset + n`` unless ``positions`` gives
    one per token (for a sample of tokens).
    """
    x = f32_from_bf16_bits(x_bits)
    b, n, h, d = x.shape
    if weight_bits is not None:
        ss = rms_sum_of_squares(x)
        ms = (ss * F32(1.0 / d)).astype(F32)        # exact power-of-two scale
        r = (F32(1.0) / np.sqrt((ms + F32(eps)).astype(F32))).astype(F32)
        nb = bf16_bits_from_f32((x * r[..., None]).astype(F32))
        w = f32_from_bf16_bits(np.asarray(weight_bits, np.uint16))
        y = bf16_bits_from_f32((f32_from_bf16_bits(nb) * w).astype(F32))
    else:
        y = np.array(x_bits, dtype=np.uint16, copy=True)
    if rotary_dim:
        half = rotary_dim // 2
        cb, sb = rope_tables(n, rotary_dim, theta, pos_offset, positions)
        c = f32_from_bf16_bits(cb)[None, :, None, :]
        s = f32_from_bf16_bits(sb)[None, :, None, :]
        yf = f32_from_bf16_bits(y)
        a = yf[..., :half]
        bb = yf[..., half:rotary_dim]
        lo = ((a * c).astype(F32) - (bb * s).astype(F32)).astype(F32)
        hi = ((bb * c).astype(F32) + (a * s).astype(F32)).astype(F32)
        y = y.copy()
        y[..., :half] = bf16_bits_from_f32(lo)
        y[..., half:rotary_dim] = bf16_bits_from_f32(hi)
    return y


# ============================================================ K mean, V max
def k_mean(kp_bits: np.ndarray) -> np.ndarray:
    """Exact global sequence mean per K (batch, head, dim), FP32 [B,H,D].

    "Preparation" step 4.  Reading of "exact": FP64 sums in a fixed order:
    each 64-row block summed row by row ascending, the block partials then
    summed in ascending block order, the total divided by N in FP64 and
    rounded once to FP32.
    """
    k = f32_from_bf16_bits(kp_bits).astype(np.float64)    # [B,N,H,D]
    b, n, h, d = k.shape
    nblk = ceil_div(n, K_ROWS_PER_SCALE)
    total = np.zeros((b, h, d), dtype=np.float64)
    for j in range(nblk):
        part = np.zeros((b, h, d), dtype=np.float64)
        for r in range(j * K_ROWS_PER_SCALE, min(n, (j + 1) * K_ROWS_PER_SCALE)):
            part = part + k[:, r]
        total = total + part
    return (total / np.float64(n)).astype(F32)


# ============================================================ quantization
def quant_int8(x: np.ndarray, axis_groups) -> tuple:
    """INT8 quantization of one group ("Q And K Quantization").

      amax  = max(1e-7f, max|x|)
      scale = amax / 127.0f
      q8    = cvt.rni.sat.s8.f32(x * (127.0f / amax))

    ``x`` is float32 with the group's elements along ``axis_groups`` (a tuple
    of axes reduced for the maximum).  Returns (int8 values, float32 scale).
    """
    amax = np.maximum(AMAX_FLOOR, np.max(np.abs(x), axis=axis_groups, keepdims=True)).astype(F32)
    scale = (amax / F32(127.0)).astype(F32)
    f = (F32(127.0) / amax).astype(F32)
    t = (x * f).astype(F32)
    q = np.clip(np.rint(t), -128, 127).astype(np.int8)    # rint: ties to even
    return q, np.squeeze(scale, axis=axis_groups)


def quant_q(qp_bits: np.ndarray):
    """Q: one INT8 scale per 32-row group, 4 groups per 128-row CTA.

    Input BF16 [B,N,H,D]; returns q8 int8 [B,H,N,D] and q_scale FP32
    [B,H,4*ceil(N/128)].  A group's maximum spans its valid rows and all D
    dims; invalid tail rows contribute nothing and are not written.  Reading
    for groups with no valid row (past N inside the last 128-row CTA): the
    scale is that of an all-zero group, 1e-7f/127.
    """
    q = f32_from_bf16_bits(qp_bits).transpose(0, 2, 1, 3)      # [B,H,N,D]
    b, h, n, d = q.shape
    g_total = 4 * ceil_div(n, Q_ROWS_PER_CTA)
    npad = g_total * Q_ROWS_PER_SCALE
    qpad = np.zeros((b, h, npad, d), dtype=F32)
    qpad[:, :, :n] = q
    grp = qpad.reshape(b, h, g_total, Q_ROWS_PER_SCALE, d)
    q8, scale = quant_int8(grp, (3, 4))
    q8 = q8.reshape(b, h, npad, d)[:, :, :n]
    return np.ascontiguousarray(q8), np.ascontiguousarray(scale.astype(F32))


def quant_k(kp_bits: np.ndarray, mean: np.ndarray):
    """K: subtract the FP32 mean in FP32, then one INT8 scale per 64 rows.

    Returns k8 int8 [B,H,N,D] and k_scale FP32 [B,H,ceil(N/64)].  The
    subtraction result stays FP32 (no BF16 re-rounding).
    """
    k = f32_from_bf16_bits(kp_bits).transpose(0, 2, 1, 3)      # [B,H,N,D]
    b, h, n, d = k.shape
    x = (k - mean[:, :, None, :]).astype(F32)
    nblk = ceil_div(n, K_ROWS_PER_SCALE)
    xpad = np.zeros((b, h, nblk * K_ROWS_PER_SCALE, d), dtype=F32)
    xpad[:, :, :n] = x
    grp = xpad.reshape(b, h, nblk, K_ROWS_PER_SCALE, d)
    k8, scale = quant_int8(grp, (3, 4))
    k8 = k8.reshape(b, h, -1, d)[:, :, :n]
    return np.ascontiguousarray(k8), np.ascontiguousarray(scale.astype(F32))


def quant_v(v_bits: np.ndarray):
    """V: per-(batch, head, dim) global maximum, FP8 E4M3 ("V And PV").

      amax    = max|V| over all N rows (reading: floored at 1e-7f like Q/K)
      v_scale = amax / 2.25f
      V8      = cvt.rn.satfinite.e4m3(V * (2.25f / amax))

    Returns v8t uint8 [B,H,D,64*ceil(N/64)] (dim-major, keys contiguous, rows
    past N are 0x00) and v_scale FP32 [B,H,D].
    """
    v = f32_from_bf16_bits(v_bits)                              # [B,N,H,D]
    b, n, h, d = v.shape
    amax = np.maximum(AMAX_FLOOR, np.max(np.abs(v), axis=1)).astype(F32)   # [B,H,D]
    v_scale = (amax / V_RANGE).astype(F32)
    f = (V_RANGE / amax).astype(F32)
    t = (v * f[:, None, :, :]).astype(F32)
    codes = e4m3_bits_from_f32(t)                               # [B,N,H,D]
    npad = KV_TILE * ceil_div(n, KV_TILE)
    v8t = np.zeros((b, h, d, npad), dtype=np.uint8)
    v8t[:, :, :, :n] = codes.transpose(0, 2, 3, 1)
    return v8t, v_scale


def quant_k32(kp_bits: np.ndarray, mean: np.ndarray):
    """K with one INT8 scale per 32-row group (the finer grouping the page "npu
    plan P7" names for outlier heads: "per-32-group scales at a small byte
    cost").  Reading: the same arithmetic as ``quant_k`` ("Q And K Quantization":
    x = (f32)k - mean, amax/127, rint_sat) over 32 rows instead of 64; tail rows
    take no part.  Returns k8 int8 [B,H,N,D] and k_scale FP32 [B,H,ceil(N/32)].
    """
    k = f32_from_bf16_bits(kp_bits).transpose(0, 2, 1, 3)      # [B,H,N,D]
    x = (k - mean[:, :, None, :].astype(F32)).astype(F32)
    b, h, n, d = x.shape
    ng = ceil_div(n, 32)
    xpad = np.zeros((b, h, ng * 32, d), dtype=F32)
    xpad[:, :, :n] = x
    valid = np.zeros((b, h, ng * 32, d), dtype=bool)
    valid[:, :, :n] = True
    amax = np.max(np.where(valid, np.abs(xpad), F32(0)).reshape(b, h, ng, 32, d), axis=(3, 4))
    amax = np.maximum(AMAX_FLOOR, amax).astype(F32)
    scale = (amax / F32(127.0)).astype(F32)
    f = (F32(127.0) / amax).astype(F32)
    t = (xpad.reshape(b, h, ng, 32, d) * f[..., None, None]).astype(F32)
    k8 = np.clip(np.rint(t), -128, 127).astype(np.int8).reshape(b, h, ng * 32, d)[:, :, :n]
    return np.ascontiguousarray(k8), scale


def quant_v16(v_bits: np.ndarray, capacity: int | None = None):
    """V for the FP16 P.V variant (page "Fused FP8 PV preparation": FP16 PV is the
    default, FP8 probabilities the option).  Reading: V is converted from BF16 to
    FP16 round-to-nearest-even with no scale (exact wherever |v| lies in FP16's
    normal range, 2^-14 .. 65504) and stored dim-major like the FP8 V, keys
    contiguous: uint16 FP16 bits [B,H,D,capacity] (capacity >= N, default N
    rounded up to 8); entries past N are 0.
    """
    v = f32_from_bf16_bits(v_bits)                              # [B,N,H,D]
    b, n, h, d = v.shape
    cap = capacity if capacity is not None else 8 * ceil_div(n, 8)
    out = np.zeros((b, h, d, cap), dtype=np.uint16)
    out[:, :, :, :n] = f16_bits_from_f32(v).transpose(0, 2, 3, 1)
    return out


def quant_v_rotated(v_bits: np.ndarray):
    """INT8 V rotated by the per-head Walsh-Hadamard matrix (page "npu plan P7":
    P7c, "an int8 V needs an inverse transform on the output that K does not").
    Reading: V' = V H/sqrt(D) per token (the FP32 rotation of ``hadamard_rotate``),
    INT8 with one scale per (batch, head, channel) over all tokens, the per-channel
    maximum of "V And PV" with the INT8 formulas of "Q And K Quantization":
    amax = max(1e-7f, max_n |v'|), v_scale = amax/127, v8 = rint_sat(v' * (127/amax)).
    Returns v8t int8 [B,H,D,64*ceil(N/64)] (dim-major, keys contiguous, rows past N
    are 0) and v_scale FP32 [B,H,D].
    """
    vr = hadamard_rotate(v_bits)                                # [B,N,H,D]
    b, n, h, d = vr.shape
    amax = np.maximum(AMAX_FLOOR, np.max(np.abs(vr), axis=1)).astype(F32)   # [B,H,D]
    scale = (amax / F32(127.0)).astype(F32)
    f = (F32(127.0) / amax).astype(F32)
    codes = np.clip(np.rint((vr * f[:, None]).astype(F32)), -128, 127).astype(np.int8)
    npad = KV_TILE * ceil_div(n, KV_TILE)
    v8t = np.zeros((b, h, d, npad), dtype=np.int8)
    v8t[:, :, :, :n] = codes.transpose(0, 2, 3, 1)
    return v8t, scale


# ============================================================ Hadamard variant
def fwht(x: np.ndarray) -> np.ndarray:
    """Unnormalized Walsh-Hadamard transform along the last axis, FP32.

    Reading (page "npu plan P7", design note and PR #1273: per-head rotation
    with an optional sign vector): Sylvester order, no signs.  Stages
    h = 1, 2, 4, ..., D/2; each maps the pair (a, b) at (i, i+h) inside every
    block of 2h to (a + b, a - b), one FP32 rounding per add.
    """
    y = np.array(x, dtype=F32, copy=True)
    d = y.shape[-1]
    h = 1
    while h < d:
        y = y.reshape(*x.shape[:-1], d // (2 * h), 2, h)
        a = y[..., 0, :]
        b = y[..., 1, :]
        y = np.stack([(a + b).astype(F32), (a - b).astype(F32)], axis=-2)
        y = y.reshape(*x.shape[:-1], d)
        h *= 2
    return y


def hadamard_rotate(x_bits: np.ndarray) -> np.ndarray:
    """x H / sqrt(D) in FP32 for BF16 input [..., D]; D = 4^k keeps the
    1/sqrt(D) scale a power of two (1/16 at D=256), so the scale is exact."""
    x = f32_from_bf16_bits(x_bits)
    d = x.shape[-1]
    return (fwht(x) * F32(1.0 / math.sqrt(d))).astype(F32)


def quant_hadamard(q_bits, k_bits, v_bits):
    """Rotated INT8 Q/K, per-token FP16 K scale, per-channel FP8 V.

    Q' = Q H/sqrt(D): INT8 per 32-row group as ``quant_q``.
    K' = K H/sqrt(D): INT8 with one scale per (batch, head, token):
        amax = max(1e-7f, max|k'|), scale stored as fp16_rn(amax/127.0f),
        q8 = rint_sat(k' * (127.0f/amax)).  No K mean is subtracted.
    V: ``quant_v``.
    Returns q8 [B,Hq,Nq,D], q_scale [B,Hq,G], k8 [B,Hkv,Nkv,D],
    k_scale_f16 uint16 [B,Hkv,Nkv], v8t, v_scale.
    """
    q8, q_scale = quant_q_rotated(q_bits)
    k8, k_scale_f16 = quant_k_rotated(k_bits)
    v8t, v_scale = quant_v(v_bits)
    return q8, q_scale.astype(F32), k8, k_scale_f16, v8t, v_scale


def quant_k_rotated(k_bits):
    """K' = K H/sqrt(D), INT8 with one FP16 scale per (batch, head, token) (the K
    half of ``quant_hadamard``): amax = max(1e-7f, max|k'|), scale fp16_rn(amax/127),
    q8 = rint_sat(k' * (127.0f/amax)).  Returns k8 [B,H,N,D], scales uint16 [B,H,N]."""
    kr = hadamard_rotate(k_bits).transpose(0, 2, 1, 3)           # [B,Hkv,N,D]
    amax = np.maximum(AMAX_FLOOR, np.max(np.abs(kr), axis=3, keepdims=True)).astype(F32)
    f = (F32(127.0) / amax).astype(F32)
    k8 = np.clip(np.rint((kr * f).astype(F32)), -128, 127).astype(np.int8)
    k_scale_f16 = f16_bits_from_f32((amax / F32(127.0)).astype(F32))[..., 0]
    return k8, k_scale_f16


def quant_q_rotated(q_bits):
    """Q' = Q H/sqrt(D), INT8 per 32-row group (the Q half of ``quant_hadamard``)."""
    qr = hadamard_rotate(q_bits).transpose(0, 2, 1, 3)
    b, h, n, d = qr.shape
    g_total = 4 * ceil_div(n, Q_ROWS_PER_CTA)
    qpad = np.zeros((b, h, g_total * Q_ROWS_PER_SCALE, d), dtype=F32)
    qpad[:, :, :n] = qr
    q8, q_scale = quant_int8(qpad.reshape(b, h, g_total, Q_ROWS_PER_SCALE, d), (3, 4))
    return np.ascontiguousarray(q8.reshape(b, h, -1, d)[:, :, :n]), q_scale.astype(F32)


# ============================================================ key cache (chunked prefill)
def kcache_new(b: int, h: int, d: int, capacity: int) -> dict:
    """An empty rotated int8 key cache (page "npu plan P7": int8 K rotated by a
    per-head Hadamard with a per-token scale sidecar, V kept in 16 bits), room for
    ``capacity`` keys per (batch, head)."""
    return dict(k8=np.zeros((b, h, capacity, d), np.int8),
                k_scale=np.zeros((b, h, capacity), np.uint16),
                v16=np.zeros((b, h, d, capacity), np.uint16), n=0)


def kcache_append(cache: dict, k_bits, v_bits) -> dict:
    """Write one prefill chunk's keys after those already cached: K rows through
    ``quant_k_rotated`` (each token on its own, so a chunk's codes do not depend
    on the other chunks), V through ``quant_v16``; the cache grows by the chunk."""
    n0, n = cache["n"], k_bits.shape[1]
    k8, ks = quant_k_rotated(k_bits)
    cache["k8"][:, :, n0:n0 + n] = k8
    cache["k_scale"][:, :, n0:n0 + n] = ks
    cache["v16"][:, :, :, n0:n0 + n] = quant_v16(v_bits, n)
    cache["n"] = n0 + n
    return cache


def kcache_attend(cache: dict, q_bits, rows=None):
    """A query chunk against every cached key: Q rotated and quantized
    (``quant_q_rotated``), then ``attention`` with per-token K scales and the
    FP16 P.V product (V is FP16 in the cache)."""
    n = cache["n"]
    q8, qs = quant_q_rotated(q_bits)
    out, _, _ = attention(q8, qs, cache["k8"][:, :, :n], cache["k_scale"][:, :, :n],
                          cache["v16"][..., :n], None, n, k_scale_mode=1, rows=rows, pv="fp16")
    return out


# ============================================================ scores
def scores(q8: np.ndarray, k8: np.ndarray) -> np.ndarray:
    """INT32 scores S = Q8 K8^T per (batch, head) ("INT8 QK And Score Domain").

    Exact integer arithmetic (int64 accumulation, |S| < 2^31).
    ``q8`` [..., Nq, D], ``k8`` [..., Nk, D] -> int32 [..., Nq, Nk].
    """
    s = np.matmul(q8.astype(np.int64), np.swapaxes(k8.astype(np.int64), -1, -2))
    return s.astype(np.int32)


# ============================================================ attention
def score_constant(d: int, sm_scale: float = 0.0) -> np.float32:
    """log2(e) * softmax scale (default 1/sqrt(D)), FP64 rounded once to FP32."""
    sc = 1.0 / math.sqrt(d) if sm_scale == 0.0 else float(sm_scale)
    return F32(math.log2(math.e) * sc)


def attention(q8, q_scale, k8, k_scale, v8t, v_scale, n_kv: int, *,
              k_scale_mode: int = 0, sm_scale: float = 0.0, rows=None, pv: str = "fp8"):
    """Online base-2 softmax attention over 64-key tiles, BF16 output.

    Follows "Online Softmax", "V And PV" and "Finalization And Tails":

    per query row:  m = -5e6f, d = 1.0f, RO = 0
    for each 64-key tile t = 0, 1, ... in increasing order:
      A     = (q_s * k_s) * c                   (FP32 dequantization x softmax
                                                 scale, c = log2(e)/sqrt(D))
      s_j   = (f32)S_j * A                      (scaled score, FP32; keys past N
                                                 get -5e6f)
      mt    = max_j s_j - 8.807f
      mn    = max(m, mt)
      old   = 2^(m - mn);  d *= old;  RO *= old
      p_j   = 2^fma(S_j, A, -mn)                (reading of "the reference fused
                                                 multiply-add placement": the
                                                 exponent is S*A - mn rounded
                                                 once; 2^x is the FP32 value of
                                                 exp2 in FP64; masked keys: 0)
      d    += p_j, j ascending, FP32, unquantized p
      P8_j  = e4m3_rn_satfinite(p_j)
      RO   += sum_j P8_j * V8[j, :]             (reading: exact tile sum, FP64)
      m     = mn
    out = bf16_rn((f32)(RO / d) * v_scale)      (reading: exact division)

    pv="int8v" is the rotated INT8 V of the page "npu plan P7" (P7c): v8t holds the
    INT8 codes of ``quant_v_rotated`` and v_scale its per-channel scales.  Reading:
    probabilities as in pv="fp16" (P16 = fp16_rn(p)); RO += sum_j P16_j * V'8[j, :]
    (exact tile sum); o' = (f32)(RO / d) * v_scale (FP32); the inverse rotation
    out = bf16_rn(FWHT(o') / sqrt(D)) (H/sqrt(D) is symmetric and orthonormal, so
    it is its own inverse; FP32 stages as ``fwht``, the 1/sqrt(D) scale exact).

    pv="fp16" is the FP16 P.V control of the page "Fused FP8 PV preparation"
    (softmax, maximum and denominator unchanged, only the probability encoding
    and V differ).  Reading: P16_j = fp16_rn(p_j), RO += sum_j P16_j * V16[j, :]
    (exact tile sum) with V16 from ``quant_v16`` (no V scale), and
    out = bf16_rn((f32)(RO / d)).

    Shapes: q8 [B,Hq,Nq,D], q_scale [B,Hq,G], k8 [B,Hkv,Nkv,D], k_scale
    [B,Hkv,nK] FP32 (mode 0), FP16 bits [B,Hkv,Nkv] (mode 1, per token) or
    FP32 [B,Hkv,ceil(Nkv/32)] (mode 2, per 32-row group: A_j uses the scale of
    key j's group), v8t [B,Hkv,D,>=64*nK] E4M3 bits, v_scale [B,Hkv,D]; for
    pv="fp16" v8t holds the FP16 bits of ``quant_v16`` and v_scale is unused.  GQA: query head h
    reads KV head h // (Hq/Hkv).  ``rows`` optionally restricts the query
    rows (independent of one another, so a sample is exact).
    Returns (out bf16 bits [B,len(rows),Hq,D], final m, final d).
    """
    b, hq, nq, d = q8.shape
    hkv = k8.shape[1]
    grp = hq // hkv
    rows = np.arange(nq) if rows is None else np.asarray(rows)
    c = score_constant(d, sm_scale)
    nk = ceil_div(n_kv, KV_TILE)
    kvh = np.arange(hq) // grp
    qsel = q8[:, :, rows].astype(np.float64)                         # [B,Hq,R,D]
    qs = q_scale[:, :, rows // Q_ROWS_PER_SCALE].astype(F32)         # [B,Hq,R]
    nr = len(rows)
    m = np.full((b, hq, nr), M_INIT, dtype=F32)
    den = np.ones((b, hq, nr), dtype=F32)
    ro = np.zeros((b, hq, nr, d), dtype=np.float64)
    if pv == "fp8":
        vv = f32_from_e4m3_bits(v8t).astype(np.float64)              # [B,Hkv,D,Np]
    elif pv == "fp16":
        vv = f32_from_f16_bits(v8t).astype(np.float64)
    elif pv == "int8v":
        vv = v8t.astype(np.float64)
    else:
        raise ValueError(pv)
    for t in range(nk):
        j0, j1 = t * KV_TILE, min(n_kv, (t + 1) * KV_TILE)
        kt = k8[:, kvh, j0:j1].astype(np.float64)                    # [B,Hq,w,D]
        s_int = np.matmul(qsel, np.swapaxes(kt, -1, -2))             # exact integers
        sf = s_int.astype(F32)                                       # exact (|S| < 2^24)
        if k_scale_mode == 0:
            ks = k_scale[:, kvh, t].astype(F32)                      # [B,Hq]
            a = ((qs * ks[:, :, None]).astype(F32) * c).astype(F32)[..., None]   # [B,Hq,R,1]
        else:
            if k_scale_mode == 1:
                ks = f32_from_f16_bits(k_scale[:, kvh, j0:j1])       # [B,Hq,w]
            else:
                ks = k_scale[:, kvh][:, :, np.arange(j0, j1) // 32].astype(F32)
            a = ((qs[..., None] * ks[:, :, None, :]).astype(F32) * c).astype(F32)  # [B,Hq,R,w]
        s = (sf * a).astype(F32)
        w = j1 - j0
        if w < KV_TILE:                                              # masked tail
            pad = np.full(s.shape[:-1] + (KV_TILE - w,), MASKED_SCORE, F32)
            s = np.concatenate([s, pad], axis=-1)
        mt = (np.max(s, axis=-1) - FP8_OFFSET).astype(F32)
        mn = np.maximum(m, mt)
        old = np.exp2((m - mn).astype(F32).astype(np.float64)).astype(F32)
        den = (den * old).astype(F32)
        ro = ro * old.astype(np.float64)[..., None]
        # fma(S, A, -mn): the float64 product S*A is exact (22 + 24 bits) and the
        # float64 difference is exact or below half a float32 ulp of rounding
        e = (s_int * a.astype(np.float64) - mn.astype(np.float64)[..., None]).astype(F32)
        p = np.exp2(e.astype(np.float64)).astype(F32)
        if w < KV_TILE:
            p = np.concatenate([p, np.zeros(p.shape[:-1] + (KV_TILE - w,), F32)], axis=-1)
        for j in range(KV_TILE):
            den = (den + p[..., j]).astype(F32)
        if pv == "fp8":
            pq = e4m3_value_from_f32(p)[..., : j1 - j0]               # exact values
        else:
            pq = f32_from_f16_bits(f16_bits_from_f32(p[..., : j1 - j0]))
        vt = np.swapaxes(vv[:, kvh, :, j0:j1], -1, -2)              # [B,Hq,w,D]
        ro = ro + np.matmul(pq.astype(np.float64), vt)
        m = mn
    o = (ro / den.astype(np.float64)[..., None]).astype(F32)
    if pv in ("fp8", "int8v"):
        vs = v_scale[:, kvh].astype(F32)[:, :, None, :]
        o = (o * vs).astype(F32)
    if pv == "int8v":
        o = (fwht(o) * F32(1.0 / math.sqrt(d))).astype(F32)
    out = bf16_bits_from_f32(o).transpose(0, 2, 1, 3)                 # [B,R,Hq,D]
    return np.ascontiguousarray(out), m, den


# ============================================================ whole path
def pipeline(q_bits, k_bits, v_bits, q_w, k_w, eps, rotary_dim, theta=10000.0,
             pos_offset=0, rows=None):
    """prep -> K mean -> quant -> attention for Hq == Hkv style inputs
    (BF16 [B,N,H,D] bit arrays).  Returns a dict of every intermediate."""
    qp = prep(q_bits, q_w, eps, rotary_dim, theta, pos_offset)
    kp = prep(k_bits, k_w, eps, rotary_dim, theta, pos_offset)
    mu = k_mean(kp)
    q8, q_scale = quant_q(qp)
    k8, k_scale = quant_k(kp, mu)
    v8t, v_scale = quant_v(v_bits)
    out, _, _ = attention(q8, q_scale, k8, k_scale, v8t, v_scale, kp.shape[1], rows=rows)
    return dict(qp=qp, kp=kp, k_mean=mu, q8=q8, q_scale=q_scale, k8=k8, k_scale=k_scale,
                v8t=v8t, v_scale=v_scale, out=out)


def pipeline_hadamard(q_bits, k_bits, v_bits, rows=None):
    """Hadamard-rotated int8-K variant: quant_hadamard -> attention (mode 1)."""
    q8, q_scale, k8, ks16, v8t, v_scale = quant_hadamard(q_bits, k_bits, v_bits)
    out, _, _ = attention(q8, q_scale, k8, ks16, v8t, v_scale, k_bits.shape[1],
                          k_scale_mode=1, rows=rows)
    return dict(q8=q8, q_scale=q_scale, k8=k8, k_scale=ks16, v8t=v8t, v_scale=v_scale,
                out=out)
