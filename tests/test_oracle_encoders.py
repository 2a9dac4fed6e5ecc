"""Pins of the oracle's number-format encoders against their definitions,
hand-computed codes and (where one exists) an independent library conversion."""
import numpy as np
import pytest
import torch

from oracle import encoders as E


def _rand_f32(n, seed=0, lo=-40, hi=40):
    rng = np.random.default_rng(seed)
    m = rng.standard_normal(n)
    e = rng.integers(lo, hi, n)
    return (m * np.exp2(e)).astype(np.float32)


# ---------------------------------------------------------------- BF16
def test_bf16_matches_torch_round_to_nearest_even():
    x = np.concatenate([_rand_f32(2_000_000, 1, -130, 128),
                        np.array([0.0, -0.0, 1.0, -1.0, 3.0e38, 1e-40, -1e-42], np.float32)])
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(E.bf16_bits_from_f32(x), ref)


def test_bf16_hand_ties():
    # 1 + 2^-8 is exactly halfway between 1 and 1+2^-7: ties to even -> 1.0 (0x3F80)
    # 1 + 3*2^-8 is halfway between 1+2^-7 and 1+2^-6: ties to even -> 1+2^-6 (0x3F82)
    x = np.array([1 + 2 ** -8, 1 + 3 * 2 ** -8, -(1 + 2 ** -8), 1 + 2 ** -8 + 2 ** -20], np.float32)
    assert E.bf16_bits_from_f32(x).tolist() == [0x3F80, 0x3F82, 0xBF80, 0x3F81]
    assert np.array_equal(E.f32_from_bf16_bits(np.array([0x3F80, 0xC040], np.uint16)),
                          np.array([1.0, -3.0], np.float32))


def test_bf16_from_f64_single_rounding():
    # exact float32 inputs agree with the float32 path
    x = _rand_f32(200_000, 2, -100, 100)
    assert np.array_equal(E.bf16_bits_from_f64(x.astype(np.float64)), E.bf16_bits_from_f32(x))
    # a double just above a bf16 midpoint whose float32 image IS the midpoint:
    # single rounding goes up, double rounding (via float32 RNE) would tie-to-even down
    x = 1.0 + 2.0 ** -8 + 2.0 ** -40
    assert E.bf16_bits_from_f64(np.array([x])).tolist() == [0x3F81]
    assert E.bf16_bits_from_f32(np.array([x], np.float32)).tolist() == [0x3F80]
    # cos(1) = 0.5403023...; bf16 neighbours 0.5390625 (0x3F0A) and 0.54296875 (0x3F0B)
    assert E.bf16_bits_from_f64(np.array([np.cos(1.0)])).tolist() == [0x3F0A]
    # tiny values below the bf16 normal range round on the 2^-133 grid
    assert E.bf16_bits_from_f64(np.array([2.0 ** -133 * 1.4])).tolist() == [0x0001]
    assert E.bf16_bits_from_f64(np.array([0.0, -0.0])).tolist() == [0x0000, 0x8000]


# ---------------------------------------------------------------- FP16
def test_f16_matches_numpy_cast():
    x = np.concatenate([_rand_f32(2_000_000, 3, -30, 17),
                        np.array([65504.0, 65519.0, 65520.0, 2.0 ** -24, 2.0 ** -25,
                                  2.0 ** -25 * 1.0001, 0.0, -0.0, 1e-9], np.float32)])
    with np.errstate(over="ignore"):
        ref = x.astype(np.float16).view(np.uint16)
    assert np.array_equal(E.f16_bits_from_f32(x), ref)
    back = E.f32_from_f16_bits(ref)
    fin = np.isfinite(back)
    assert np.array_equal(back[fin], ref.view(np.float16).astype(np.float32)[fin])


def test_f16_hand_codes():
    x = np.array([1.0, -2.0, 65504.0, 2.0 ** -24, 1.0 + 2.0 ** -11, 1.0 + 3 * 2.0 ** -11], np.float32)
    # 1+2^-11 is a tie between 1 and 1+2^-10 -> even (1.0); 1+3*2^-11 -> 1+2^-9
    assert E.f16_bits_from_f32(x).tolist() == [0x3C00, 0xC000, 0x7BFF, 0x0001, 0x3C00, 0x3C02]


# ---------------------------------------------------------------- E4M3
def test_e4m3_code_table_from_ocp_definition():
    # every finite code decodes to the OCP value and re-encodes to itself
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], np.uint8)
    vals = E.f32_from_e4m3_bits(codes)
    assert np.array_equal(E.e4m3_bits_from_f32(vals), codes)
    assert vals[codes.tolist().index(0x7E)] == 448.0          # largest finite
    assert vals[codes.tolist().index(0x01)] == 2.0 ** -9       # smallest subnormal
    assert vals[codes.tolist().index(0x08)] == 2.0 ** -6       # smallest normal
    assert vals[codes.tolist().index(0x41)] == 2.25            # 1.125 * 2^1


def test_e4m3_rounding_and_saturation():
    x = np.array([448.0, 449.0, 464.0, 1e6, -1e6, 2.0 ** -10, 2.0 ** -10 * 1.01,
                  3 * 2.0 ** -10, 1.0 + 1 / 16, 1.0 + 3 / 16, 0.0, -0.0], np.float32)
    got = E.e4m3_bits_from_f32(x).tolist()
    # 2^-10 is the midpoint of 0 and 2^-9: ties to even -> 0; just above -> 2^-9.
    # 3*2^-10 is the midpoint of 2^-9 and 2^-8: ties to even -> 2^-8 (code 2).
    # 1+1/16 is the midpoint of 1 and 1.125: -> 1.0 (0x38); 1+3/16 -> 1.25 (0x3A).
    assert got == [0x7E, 0x7E, 0x7E, 0x7E, 0xFE, 0x00, 0x01, 0x02, 0x38, 0x3A, 0x00, 0x80]


def test_e4m3_matches_torch_inside_range():
    x = _rand_f32(1_000_000, 4, -12, 9)
    x = x[np.abs(x) <= 448.0]
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(E.e4m3_bits_from_f32(x), ref)
