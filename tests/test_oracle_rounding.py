"""Pins for the oracle's rounding helpers (CPU only)."""
import json
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from oracle import bf16 as ob

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _edge_f32():
    vals = [0.0, -0.0, 1.0, -1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 1.0 + 2 ** -8 + 2 ** -23,
            3.3895313892515355e38, -3.3895313892515355e38, 1.1754943508222875e-38,
            2 ** -127, 2 ** -133, 2 ** -134, 2 ** -149, -2 ** -149, 65504.0, 1e-30]
    u = np.array([0x7F7FFFFF, 0x00000001, 0x007FFFFF, 0x00008000, 0x00018000, 0x3F808000,
                  0x3F818000, 0x3F7F8000, 0x7F7F0000, 0x7F7F7FFF], dtype=np.uint32)
    return np.concatenate([np.array(vals, dtype=np.float32), u.view(np.float32)])


def test_f32_to_bf16_matches_torch():
    g = np.random.default_rng(1)
    u = g.integers(0, 2 ** 32, size=1_000_000, dtype=np.uint64).astype(np.uint32)
    f = u.view(np.float32)
    f = f[np.isfinite(f)]
    # keep values whose bf16 rounding stays finite
    f = f[np.abs(f.astype(np.float64)) < 3.3895313892515355e38]
    f = np.concatenate([f, _edge_f32()])
    ref = torch.from_numpy(f.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(ob.f32_to_bf16_bits(f), ref)


def test_f64_to_bf16_exact():
    g = np.random.default_rng(2)
    x = np.concatenate([g.normal(0, 1, 3000) * np.exp2(g.integers(-140, 120, 3000)),
                        [0.0, -0.0, 1 + 2 ** -8, 1 + 3 * 2 ** -8, 1 + 2 ** -8 + 2 ** -40,
                         2 ** -133, 3 * 2 ** -134, 2 ** -134, 0.1, -0.1]])
    got = ob.f64_to_bf16_bits(x)
    want = np.array([ob.fraction_to_bf16_bits(Fraction(float(v))) for v in x], dtype=np.uint16)
    # fraction_to_bf16_bits drops the sign of zero; compare magnitudes for zeros
    nz = x != 0
    np.testing.assert_array_equal(got[nz], want[nz])
    assert got[x == 0].tolist() == [0x0000, 0x8000]


def test_f64_to_bf16_hand_values():
    # 0.1 -> 205/2048 (0x3DCD); 1+2^-8 ties to 1.0; 1+3*2^-8 ties to fraction 2;
    # 1+2^-8+2^-40 is above the tie -> fraction 1 (single rounding, no fp32 detour)
    got = ob.f64_to_bf16_bits([0.1, 1 + 2 ** -8, 1 + 3 * 2 ** -8, 1 + 2 ** -8 + 2 ** -40])
    assert [hex(v) for v in got] == ["0x3dcd", "0x3f80", "0x3f82", "0x3f81"]


def test_fraction_to_f32_against_numpy_cast():
    # for values exact in float64, numpy's float32 cast is IEEE nearest-even
    g = np.random.default_rng(3)
    x = g.normal(0, 1, 5000) * np.exp2(g.integers(-150, 100, 5000))
    want = x.astype(np.float32)
    got = np.array([ob.fraction_to_f32(Fraction(float(v))) for v in x], dtype=np.float32)
    np.testing.assert_array_equal(got.view(np.uint32), want.view(np.uint32))


def test_fma_golden_cases():
    d = json.load(open(os.path.join(GOLDEN, "fma_bf16_cases.json")))
    for a, l, b, want in d["cases"]:
        av, lv, bv = (ob.bf16_bits_to_f64([int(v, 16)]) for v in (a, l, b))
        got = ob.f32_to_bf16_bits(ob.fma_to_f32(av, lv, bv))[0]
        assert got == int(want, 16), (a, l, b, hex(got), want)


def _rand_bf16(g, n, lo, hi):
    mant = g.integers(0, 128, n)
    ex = g.integers(lo, hi, n)
    sign = g.integers(0, 2, n)
    v = (1 + mant / 128.0) * np.exp2(ex) * np.where(sign == 1, -1.0, 1.0)
    return v


def test_fma_against_exact_rationals():
    g = np.random.default_rng(4)
    n = 20000
    a = _rand_bf16(g, n, -12, 2)
    l = _rand_bf16(g, n, -10, 3)
    b = _rand_bf16(g, n, -40, 3)          # wide exponent gaps force the exact path
    got = ob.fma_to_f32(a, l, b)
    for i in range(0, n, 7):
        want = ob.fraction_to_f32(Fraction(float(a[i])) * Fraction(float(l[i])) + Fraction(float(b[i])))
        assert got[i].view(np.uint32) == want.view(np.uint32), i


def test_fma_nonexact_sum_path():
    # b far above the product: the float64 sum is inexact, TwoSum's error is
    # non-zero and the exact path decides the rounding.
    a = np.array([1.0, 1.0, -1.5])
    l = np.array([2.0 ** -60, -(2.0 ** -60), 2.0 ** -70])
    b = np.array([1.0 + 2 ** -7, 1.0 + 2 ** -7, -4.0])
    got = ob.fma_to_f32(a, l, b)
    for i in range(3):
        want = ob.fraction_to_f32(Fraction(a[i]) * Fraction(l[i]) + Fraction(b[i]))
        assert got[i] == want
    # the fp32 quantum in [1, 2) is 2^-23, so +/- 2^-60 rounds back to 1 + 2^-7
    assert got[0] == np.float32(1 + 2 ** -7) and got[1] == np.float32(1 + 2 ** -7)


def test_bf16_bits_roundtrip():
    bits = np.arange(0, 65536, dtype=np.uint32).astype(np.uint16)
    with np.errstate(invalid="ignore"):
        v = ob.bf16_bits_to_f64(bits)
    fin = np.isfinite(v)
    back = ob.f64_to_bf16_bits(v[fin])
    np.testing.assert_array_equal(back, bits[fin])
