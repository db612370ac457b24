"""CPU pins of the oracle's fixed-table formats (int4, NF4, FP4) and of the
b-bit (any3 / any2) generalization of the quantizer."""
import itertools

import numpy as np
import pytest

import oracle
import synth
from oracle import bf16 as ob


def test_fp4_table_is_e2m1():
    # E2M1: magnitudes 0, 0.5 (subnormal), 1, 1.5, 2, 3, 4, 6; bit 3 is the sign
    v = oracle.fp4_e2m1_values()
    assert list(v[:8]) == [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    assert list(v[8:]) == [-0.0, -0.5, -1.0, -1.5, -2.0, -3.0, -4.0, -6.0]
    bits = oracle.format_lut_bits("fp4")
    assert int(bits[8]) == 0x8000 and int(bits[0]) == 0          # +0 and -0
    assert int(bits[7]) == 0x40C0 and int(bits[15]) == 0xC0C0     # +-6 = 1.5 * 2^2


def test_int4_table_is_the_grid():
    bits = oracle.format_lut_bits("int4")
    np.testing.assert_array_equal(ob.bf16_bits_to_f64(bits), np.arange(-8.0, 8.0))


def test_nf4_levels_equal_published_values():
    # tests/golden/nf4_levels.json: the NF4 values as published with QLoRA
    import json
    import os
    gold = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "nf4_levels.json")))
    pub = np.array(gold["values"], dtype=np.float64)
    np.testing.assert_allclose(oracle.nf4_levels(), pub, rtol=0, atol=gold["abs_tolerance_float64"])
    np.testing.assert_array_equal(oracle.format_lut_bits("nf4"), oracle.f64_to_bf16_bits(pub))


def test_nf4_table_properties():
    v = ob.bf16_bits_to_f64(oracle.format_lut_bits("nf4"))
    assert np.all(np.diff(v) > 0) and v[0] == -1.0 and v[-1] == 1.0
    assert np.count_nonzero(v == 0.0) == 1 and np.count_nonzero(v > 0) == 8


@pytest.mark.parametrize("fmt", ["int4", "nf4", "fp4"])
def test_format_quantizer_picks_nearest_entry(fmt):
    w = synth.weights_bf16(6, 256, 3, layer="fmt")
    q = oracle.quantize_format(w, fmt, 64)
    table = ob.bf16_bits_to_f64(oracle.format_lut_bits(fmt))
    a = ob.bf16_bits_to_f64(q.alpha)
    b = ob.bf16_bits_to_f64(q.beta)
    wf = ob.bf16_bits_to_f64(w).reshape(6, 4, 64)
    idx = oracle.unpack_nibbles(q.idx_nib).reshape(6, 4, 64)
    for r, gi in itertools.product(range(6), range(4)):
        ws = (wf[r, gi] - b[r, gi]) / a[r, gi]
        d = np.abs(ws[:, None] - table[None, :])
        best = d.min(axis=1)
        # the chosen entry is a nearest one, and the lowest such index
        assert np.all(d[np.arange(64), idx[r, gi]] == best)
        assert np.all(idx[r, gi] == np.argmax(d == best[:, None], axis=1))
    if fmt != "int4":   # absmax scaling, no offset
        amax = np.abs(wf).max(axis=2)
        top = 1.0 if fmt == "nf4" else 6.0
        np.testing.assert_array_equal(q.alpha, ob.f64_to_bf16_bits(amax / top))
        assert np.all(q.beta == 0)


def test_group_scale_three_and_two_bits_hand_example():
    # one group [-1, 0, 0.5, 2.5]: 3 bits: alpha = 3.5/7 = 0.5, beta = -1 + 4*0.5 = 1
    #                              2 bits: alpha = 3.5/3 -> bf16, beta = -1 + 2*alpha
    w = ob.f64_to_bf16_bits(np.array([[-1.0, 0.0, 0.5, 2.5]]))
    a3, b3, ws3 = oracle.group_scale(w, 4, bits=3)
    assert ob.bf16_bits_to_f64(a3)[0, 0] == 0.5 and ob.bf16_bits_to_f64(b3)[0, 0] == 1.0
    np.testing.assert_array_equal(ws3[0], [-4.0, -2.0, -1.0, 3.0])
    a2, b2, ws2 = oracle.group_scale(w, 4, bits=2)
    alpha = ob.bf16_bits_to_f64(ob.f64_to_bf16_bits(np.array(3.5 / 3.0)))
    assert ob.bf16_bits_to_f64(a2)[0, 0] == alpha
    assert ob.bf16_bits_to_f64(b2)[0, 0] == ob.bf16_bits_to_f64(ob.f64_to_bf16_bits(np.array(-1.0 + 2 * alpha)))


@pytest.mark.parametrize("bits", [3, 2])
def test_b_bit_kmeans_invariants(bits):
    w = synth.weights_bf16(12, 256, 5, layer=f"any{bits}")
    ex = np.abs(np.random.default_rng(1).standard_normal(256)) + 0.1
    a, b, ws = oracle.group_scale(w, 128, bits)
    c = oracle.kmeans_weights(a, ex, 128)
    idx, lut_bits, hist = oracle.kmeans_rows(ws, c, 10, history=True, bits=bits)
    size = 1 << bits
    assert lut_bits.shape == (12, size) and idx.max() < size
    assert np.all(np.diff(hist, axis=1) <= 1e-12 * np.abs(hist[:, :-1]))   # J never increases
    grid = np.tile(oracle.int_grid(bits), (12, 1))
    j_int = oracle.objective(ws, c, oracle.e_step(ws, grid), grid)
    np.testing.assert_allclose(hist[:, 0], j_int, rtol=1e-15)             # iteration 0 = integer rounding
    q = oracle.quantize(w, ex, 128, bits=bits)
    assert q.bits == bits and oracle.unpack_nibbles(q.idx_nib).max() < size
    # the table is padded to 16 columns by repeating its last entry
    assert np.all(q.lut[:, size:] == q.lut[:, size - 1:size])


def test_b_bit_e_step_brute_force():
    rng = np.random.default_rng(7)
    lut = np.sort(rng.normal(size=(1, 8)), axis=1)
    ws = rng.normal(size=(1, 4)) * 2
    c = np.ones_like(ws)
    best = None
    for assign in itertools.product(range(8), repeat=4):
        j = oracle.objective(ws, c, np.array([assign]), lut)[0]
        if best is None or j < best[0]:
            best = (j, assign)
    idx = oracle.e_step(ws, lut)
    assert tuple(int(i) for i in idx[0]) == best[1]
