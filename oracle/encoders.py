"""Number-format encoders for the CPU oracle (test infrastructure only).

Only the tests, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` leg of
``bench.py`` may import this package.  The product path never does.

Every encoder is written from the format's published definition, operates on
numpy arrays and rounds exactly once from the (exactly representable) input
value:

* BF16: IEEE-754 binary32 with the low 16 mantissa bits dropped (8 exponent
  bits, 7 stored mantissa bits).  Round to nearest, ties to even.
* FP16: IEEE-754 binary16 (5 exponent bits, bias 15, 10 mantissa bits,
  subnormals down to 2^-24).  Round to nearest, ties to even; overflow to inf.
* E4M3: OCP 8-bit floating point, E4M3 variant (4 exponent bits, bias 7,
  3 mantissa bits, subnormal quantum 2^-9, no infinities, largest finite
  magnitude 448).  Round to nearest, ties to even, then "satfinite": any
  magnitude above 448 becomes 448.

The "Exact Numerical Contract" page (sections "Preparation", "Q And K
Quantization", "V And PV") fixes BF16 round-to-nearest storage, the
``cvt.rni.sat.s8.f32`` integer rounding and the E4M3 RN satfinite conversion;
the int8 rounding lives in ``qattn_oracle.quant_int8``.
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "bf16_bits_from_f32", "f32_from_bf16_bits", "bf16_bits_from_f64",
    "f16_bits_from_f32", "f32_from_f16_bits",
    "e4m3_value_from_f32", "e4m3_bits_from_f32", "f32_from_e4m3_bits",
    "E4M3_MAX",
]

E4M3_MAX = 448.0


# --------------------------------------------------------------------- BF16
def bf16_bits_from_f32(x) -> np.ndarray:
    """float32 -> bf16 bit pattern (uint16), round to nearest even.

    The bf16 value is the float32 whose low 16 bits are zero; rounding adds
    0x7FFF plus the lowest kept bit before truncation (the textbook RNE
    carry), so a carry out of the mantissa correctly bumps the exponent.
    NaN inputs are outside the contract and are mapped to a quiet NaN.
    """
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) >> 16).astype(np.uint16)
    nan = np.isnan(x)
    if nan.any():
        r = np.where(nan, np.uint16(0x7FC0), r)
    return r


def f32_from_bf16_bits(b) -> np.ndarray:
    """bf16 bit pattern -> float32 (exact)."""
    b = np.asarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


def _round_to_quantum(a: np.ndarray, quantum: np.ndarray) -> np.ndarray:
    """Round non-negative float64 ``a`` to a multiple of a power-of-two
    ``quantum``, ties to even (numpy ``rint`` is round-half-even; the
    division and multiplication by a power of two are exact)."""
    return np.rint(a / quantum) * quantum


def bf16_bits_from_f64(x) -> np.ndarray:
    """float64 -> bf16 bit pattern with ONE rounding (nearest, ties to even).

    The value is rounded to the bf16 quantum of its binade, 2^(e-7) where
    e = floor(log2|x|), or to the subnormal quantum 2^-133 below 2^-126.
    The result has at most 8 significant bits, so its float32 image is
    exact and the bf16 pattern is the float32's top half.
    """
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    _, e2 = np.frexp(a)                    # a = m * 2^e2, m in [0.5, 1)
    e = e2.astype(np.int64) - 1            # floor(log2 a) for a > 0
    e = np.maximum(e, -126)                # below the normal range use 2^-133
    quantum = np.ldexp(1.0, (e - 7).astype(np.int32))
    r = _round_to_quantum(a, quantum)
    r = np.where(a == 0, 0.0, r)
    y = np.copysign(r, x).astype(np.float32)   # exact: <= 8 significant bits
    return (y.view(np.uint32) >> 16).astype(np.uint16)


# --------------------------------------------------------------------- FP16
def f16_bits_from_f32(x) -> np.ndarray:
    """float32 -> IEEE binary16 bit pattern, round to nearest even."""
    x = np.asarray(x, dtype=np.float32)
    a = np.abs(x.astype(np.float64))
    sign = np.signbit(x)
    _, e2 = np.frexp(a)
    e = e2.astype(np.int64) - 1
    e = np.maximum(e, -14)                 # subnormal quantum 2^-24
    quantum = np.ldexp(1.0, (e - 10).astype(np.int32))
    r = _round_to_quantum(a, quantum)
    r = np.where(a == 0, 0.0, r)
    # encode the (exactly representable or overflowing) magnitude
    out = np.zeros(x.shape, dtype=np.uint16)
    inf = r >= 65536.0                     # 65520 and above round to inf
    fin = ~inf
    rf = r[fin]
    _, re2 = np.frexp(rf)
    re = re2.astype(np.int64) - 1
    normal = rf >= 2.0 ** -14
    expf = np.where(normal, re + 15, 0)
    mant = np.where(normal,
                    np.rint(rf / np.ldexp(1.0, (re - 10).astype(np.int32))) - 1024,
                    np.rint(rf / 2.0 ** -24))
    mant = np.where(rf == 0, 0, mant)
    expf = np.where(rf == 0, 0, expf)
    out[fin] = (expf.astype(np.uint16) << 10) | mant.astype(np.uint16)
    out[inf] = 0x7C00
    out = np.where(sign, out | np.uint16(0x8000), out).astype(np.uint16)
    return out


def f32_from_f16_bits(b) -> np.ndarray:
    """IEEE binary16 bit pattern -> float32 (exact), finite values only."""
    b = np.asarray(b, dtype=np.uint16).astype(np.int64)
    s = np.where(b & 0x8000, -1.0, 1.0)
    ef = (b >> 10) & 0x1F
    m = b & 0x3FF
    v = np.where(ef == 0, m * 2.0 ** -24,
                 np.ldexp(1.0 + m / 1024.0, (ef - 15).astype(np.int32)))
    v = np.where(ef == 31, np.inf, v)
    return (s * v).astype(np.float32)


# --------------------------------------------------------------------- E4M3
def _e4m3_table() -> np.ndarray:
    """Value of every non-negative finite E4M3 code 0x00..0x7E (OCP spec)."""
    vals = []
    for code in range(0x7F):
        ef, m = code >> 3, code & 7
        if ef == 0:
            vals.append(m * 2.0 ** -9)
        else:
            vals.append((1.0 + m / 8.0) * 2.0 ** (ef - 7))
    return np.array(vals, dtype=np.float64)


_E4M3_POS = _e4m3_table()


def e4m3_value_from_f32(x) -> np.ndarray:
    """float32 -> value of its E4M3 RN-satfinite encoding (as float64).

    The magnitude is rounded to the E4M3 quantum of its binade (2^(e-3) for
    e = floor(log2|x|) >= -6, else the subnormal quantum 2^-9), ties to even,
    then clamped to 448.
    """
    x = np.asarray(x, dtype=np.float32).astype(np.float64)
    a = np.abs(x)
    _, e2 = np.frexp(a)
    e = e2.astype(np.int64) - 1
    e = np.maximum(e, -6)
    quantum = np.ldexp(1.0, (e - 3).astype(np.int32))
    r = _round_to_quantum(a, quantum)
    r = np.where(a == 0, 0.0, r)
    r = np.minimum(r, E4M3_MAX)
    return np.copysign(r, x)


def e4m3_bits_from_f32(x) -> np.ndarray:
    """float32 -> E4M3 bit pattern (uint8), RN satfinite."""
    v = e4m3_value_from_f32(x)
    a = np.abs(v)
    code = np.searchsorted(_E4M3_POS, a).astype(np.uint8)
    assert np.array_equal(_E4M3_POS[code], a), "rounded value not on the E4M3 grid"
    return np.where(np.signbit(v), code | np.uint8(0x80), code).astype(np.uint8)


def f32_from_e4m3_bits(b) -> np.ndarray:
    """E4M3 bit pattern -> float32 (exact); 0x7F/0xFF (NaN) are not expected."""
    b = np.asarray(b, dtype=np.uint8)
    mag = _E4M3_POS[np.minimum(b & 0x7F, 0x7E)]
    return np.where(b & 0x80, -mag, mag).astype(np.float32)
