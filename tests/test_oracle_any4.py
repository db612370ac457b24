"""Pins for the oracle's quantizer, dequantization and linear layer (CPU only)."""
import itertools
from fractions import Fraction
import json
import os

import numpy as np
import pytest
import torch

import oracle
import synth
from oracle import bf16 as ob

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _bits(vals):
    return ob.f64_to_bf16_bits(np.asarray(vals, dtype=np.float64))


# ------------------------------------------------------------ group scaling

def test_group_scaling_golden():
    d = json.load(open(os.path.join(GOLDEN, "group_scaling.json")))
    w = _bits([d["w"]])
    a, b, ws = oracle.group_scale(w, d["group_size"])
    assert a[0, 0] == int(d["alpha_bits"], 16)
    assert b[0, 0] == int(d["beta_bits"], 16)
    want = np.array(d["ws_num"], dtype=np.float64) / d["ws_den"]
    np.testing.assert_allclose(ws[0], want, rtol=0, atol=4e-16)
    assert ws[0, 0] == -8.0


def test_group_scaling_range_and_constant_group():
    g = np.random.default_rng(5)
    w = _bits(g.normal(0, 0.02, (8, 256)))
    w[3, 128:] = _bits([0.125])[0]                       # a constant group
    a, b, ws = oracle.group_scale(w, 128)
    assert a[3, 1] == 0 and b[3, 1] == _bits([0.125])[0]
    assert np.all(ws[3, 128:] == 0.0)
    # min maps near -8 and max near 7 (alpha and beta are bf16-rounded)
    wsg = ws.reshape(8, 2, 128)
    mask = oracle.bf16_bits_to_f64(a) > 0
    assert np.all(np.abs(wsg.min(axis=2)[mask] + 8) < 0.1)
    assert np.all(np.abs(wsg.max(axis=2)[mask] - 7) < 0.1)


# ---------------------------------------------------------------- calibration

def test_calibration_closed_forms():
    x = np.array([[1.0, -2.0, 0.0], [-3.0, 4.0, 0.5]])
    np.testing.assert_array_equal(oracle.calibrate(x), [2.0, 3.0, 0.25])
    # E|z*s| = s*sqrt(2/pi) for z ~ N(0,1)
    s = np.array([0.5, 1.0, 3.0])
    xc = synth.rng(0, "t", "z").standard_normal((400_000, 3)) * s
    np.testing.assert_allclose(oracle.calibrate(xc), s * np.sqrt(2 / np.pi), rtol=5e-3)


# ------------------------------------------------------------------ k-means

def test_kmeans_step_golden():
    d = json.load(open(os.path.join(GOLDEN, "kmeans_step.json")))
    ws = np.array([d["ws"]])
    c = np.array([d["c"]])
    lut = np.array([d["lut_in"]], dtype=np.float64)
    idx = oracle.e_step(ws, lut)
    assert idx[0].tolist() == d["idx"]
    assert oracle.objective(ws, c, idx, lut)[0] == pytest.approx(d["J_before"], abs=1e-15)
    new = oracle.m_step(ws, c, idx, lut)
    np.testing.assert_allclose(new[0, :2], d["lut_out_01"], rtol=0, atol=1e-15)
    np.testing.assert_array_equal(new[0, 2:], lut[0, 2:])
    assert oracle.objective(ws, c, idx, new)[0] == pytest.approx(d["J_after"], abs=1e-15)


def test_kmeans_weights_are_alpha_times_ex():
    # the golden example's weights c = alpha * E|x| (M-step formula), built
    # from per-group alpha = [0.5, 2.0] (G = 3) and E|x| = [1, 1, 2, 1, 1, 3]
    d = json.load(open(os.path.join(GOLDEN, "kmeans_step.json")))
    c = oracle.kmeans_weights(_bits([[0.5, 2.0]]), np.array([1.0, 1, 2, 1, 1, 3]), 3)
    np.testing.assert_array_equal(c[0], d["c"])


def test_stored_indices_are_nearest_in_stored_table():
    w = synth.weights_bf16(12, 512, 3, layer="final")
    ex = np.abs(synth.rng(3, "final", "ex").normal(1, 0.3, 512))
    q = oracle.quantize(w, ex, g=128, iters=4)
    _, _, ws = oracle.group_scale(w, 128)
    want = oracle.e_step(ws, ob.bf16_bits_to_f64(q.lut))
    np.testing.assert_array_equal(oracle.unpack_nibbles(q.idx_nib), want)
    # row-chunked / row-subset quantization gives the same rows
    sub = oracle.quantize(w, ex, g=128, iters=4, rows=[2, 7])
    np.testing.assert_array_equal(sub.lut, q.lut[[2, 7]])
    np.testing.assert_array_equal(sub.idx_nib, q.idx_nib[[2, 7]])


def test_e_step_brute_force_optimal():
    g = np.random.default_rng(6)
    for trial in range(6):
        k = 4
        ws = g.uniform(-8, 7, (1, k))
        lut = np.sort(g.uniform(-8, 7, (1, 16)), axis=1)
        if trial % 2:
            lut[0, 5] = lut[0, 4]          # duplicate entry: ties must go to the lower index
            ws[0, 1] = lut[0, 4]
        c = g.uniform(0.1, 2, (1, k))
        idx = oracle.e_step(ws, lut)
        best, arg = np.inf, None
        for assign in itertools.product(range(16), repeat=k):   # all 16^4 joint assignments
            a = np.array(assign)
            j = float(np.sum(c[0] * (ws[0] - lut[0, a]) ** 2))
            if j < best - 1e-15:
                best, arg = j, a
        # J is separable, so the lexicographically first minimiser is the
        # elementwise lowest-index nearest entry
        assert idx[0].tolist() == arg.tolist()
        assert oracle.objective(ws, c, idx, lut)[0] == pytest.approx(best, rel=1e-12)


def test_m_step_is_optimal_for_fixed_assignment():
    g = np.random.default_rng(7)
    ws = g.normal(0, 3, (3, 200))
    c = g.uniform(0, 2, (3, 200))
    lut = np.sort(g.uniform(-8, 7, (3, 16)), axis=1)
    idx = oracle.e_step(ws, lut)
    new = oracle.m_step(ws, c, idx, lut)
    j0 = oracle.objective(ws, c, idx, new)
    for q in range(16):
        for eps in (1e-3, -1e-3, 0.1, -0.1):
            pert = new.copy()
            pert[:, q] += eps
            assert np.all(oracle.objective(ws, c, idx, pert) >= j0 - 1e-12 * (1 + j0))


def test_objective_non_increasing_and_beats_int4():
    w = synth.weights_bf16(16, 1024, 0, layer="mono")
    s = synth.channel_scale(1024, 0, layer="mono")
    ex = oracle.calibrate(synth.calibration_acts(512, s, 0, layer="mono"))
    a, b, ws = oracle.group_scale(w, 128)
    c = oracle.kmeans_weights(a, ex, 128)
    idx, lut_bits, hist = oracle.kmeans_rows(ws, c, iters=10, history=True)
    assert hist.shape == (16, 20)
    slack = 1e-12 * (1 + hist[:, :1])
    assert np.all(np.diff(hist, axis=1) <= slack)
    # iteration 0's E-step against the int4 grid is int4 rounding
    j_int4 = oracle.objective(ws, c, oracle.e_step(ws, np.tile(oracle.int4_grid(), (16, 1))),
                              np.tile(oracle.int4_grid(), (16, 1)))
    np.testing.assert_allclose(hist[:, 0], j_int4, rtol=1e-15)
    assert np.all(hist[:, -1] <= j_int4)
    assert np.mean(hist[:, -1]) < 0.95 * np.mean(j_int4)


def test_few_distinct_values_reproduced_exactly():
    g = np.random.default_rng(8)
    vals = g.normal(0, 0.02, 11)
    w = _bits(vals[g.integers(0, 11, (4, 256))])
    ex = g.uniform(0.5, 2, 256)
    a, b, ws = oracle.group_scale(w, 128)
    c = oracle.kmeans_weights(a, ex, 128)
    # two groups scale differently, so a row may hold up to 22 distinct values;
    # keep the rows that have at most 16
    rows = [r for r in range(4) if np.unique(ws[r]).size <= 16]
    assert rows
    idx, _, hist = oracle.kmeans_rows(ws[rows], c[rows], iters=3, history=True)
    assert np.all(hist == 0.0)


def test_integer_rows_dequantize_bit_exactly():
    # every group holds integers in [-8, 7] including -8 and 7: alpha = 1, beta = 0,
    # w_s = w, the table holds the integers and dequant returns W exactly
    g = np.random.default_rng(9)
    vals = g.integers(-8, 8, (6, 512)).astype(np.float64)
    vals[:, ::64] = -8.0
    vals[:, 1::64] = 7.0
    w = _bits(vals)
    ex = g.uniform(0.5, 2, 512)
    q = oracle.quantize(w, ex, g=64, iters=10)
    assert np.all(q.alpha == _bits([1.0])[0]) and np.all(q.beta == 0)
    np.testing.assert_array_equal(oracle.dequant(q), w)


# ----------------------------------------------------------------- reductions

def test_int4_reduction():
    g = np.random.default_rng(10)
    n, k, gs = 8, 256, 128
    qv = g.integers(-8, 8, (n, k))
    alpha = _bits(g.uniform(0.001, 0.05, (n, k // gs)))
    beta = _bits(g.normal(0, 0.01, (n, k // gs)))
    lut = np.tile(_bits(oracle.int4_grid()), (n, 1))
    t = oracle.Any4Tensors(oracle.pack_nibbles(qv + 8), lut, alpha, beta, gs)
    got = oracle.dequant(t)
    # independent: torch float32 a*q + b; a*q is exact in fp32 (8-bit x 4-bit
    # significands), so the separate multiply and add round once, like an fma
    af = torch.from_numpy(ob.bf16_bits_to_f64(alpha).astype(np.float32)).repeat_interleave(gs, 1)
    bf = torch.from_numpy(ob.bf16_bits_to_f64(beta).astype(np.float32)).repeat_interleave(gs, 1)
    want = (af * torch.from_numpy(qv.astype(np.float32)) + bf).to(torch.bfloat16)
    np.testing.assert_array_equal(got, want.view(torch.int16).numpy().view(np.uint16))


def test_int4_grid_e_step_is_round_to_nearest():
    g = np.random.default_rng(11)
    ws = g.uniform(-9, 8, (4, 4000))
    lut = np.tile(oracle.int4_grid(), (4, 1))
    idx = oracle.e_step(ws, lut).astype(np.int64) - 8
    want = np.clip(np.rint(ws), -8, 7)
    tie = np.abs(ws - np.floor(ws) - 0.5) < 1e-12
    np.testing.assert_array_equal(idx[~tie], want[~tie])


def test_nf4_reduction():
    g = np.random.default_rng(12)
    n, k, gs = 8, 256, 64
    idx = g.integers(0, 16, (n, k))
    absmax = _bits(g.uniform(0.01, 0.2, (n, k // gs)))
    lut = np.tile(oracle.nf4_bf16_bits(), (n, 1))
    t = oracle.Any4Tensors(oracle.pack_nibbles(idx), lut, absmax, np.zeros_like(absmax), gs)
    got = oracle.dequant(t)
    # NF4 dequant absmax * NF4[idx]: the product of two bf16 values is exact in fp32
    nf = torch.from_numpy(ob.bf16_bits_to_f64(oracle.nf4_bf16_bits()).astype(np.float32))
    am = torch.from_numpy(ob.bf16_bits_to_f64(absmax).astype(np.float32)).repeat_interleave(gs, 1)
    want = (am * nf[torch.from_numpy(idx)]).to(torch.bfloat16)
    np.testing.assert_array_equal(got, want.view(torch.int16).numpy().view(np.uint16))


def test_nf4_table_shape():
    v = oracle.nf4_levels()
    assert v.size == 16 and v[0] == -1.0 and v[-1] == 1.0 and v[7] == 0.0
    assert np.all(np.diff(v) > 0)
    assert np.sum(v > 0) == 8 and np.sum(v < 0) == 7


# ------------------------------------------------------------------- overhead

def test_lut_overhead_bits_per_weight():
    d = json.load(open(os.path.join(GOLDEN, "lut_overhead.json")))
    n, k = 4, d["columns"]
    q = oracle.Any4Tensors(np.zeros((n, k // 2), np.uint8), np.zeros((n, 16), np.uint16),
                           np.zeros((n, k // 128), np.uint16), np.zeros((n, k // 128), np.uint16), 128)
    bits = q.lut.nbytes * 8 / (n * k)
    assert bits == d["bits_per_weight"] == d["entries"] * d["bits_per_entry"] / d["columns"]
    assert q.idx_nib.nbytes * 8 / (n * k) == 4.0


# --------------------------------------------------------------------- linear

def test_linear_brute_force_tiny():
    g = np.random.default_rng(13)
    n, k, gs, m = 3, 8, 4, 2
    t = oracle.Any4Tensors(g.integers(0, 256, (n, k // 2), dtype=np.uint8),
                           _bits(g.uniform(-8, 7, (n, 16))), _bits(g.uniform(0.01, 0.1, (n, 2))),
                           _bits(g.normal(0, 0.01, (n, 2))), gs)
    x = _bits(g.normal(0, 1, (m, k)))
    y = oracle.linear(x, t)
    xv = ob.bf16_bits_to_f64(x)
    for mi in range(m):
        for ni in range(n):
            acc = 0.0
            for ki in range(k):
                byte = int(t.idx_nib[ni, ki // 2])
                q = (byte >> (4 * (ki % 2))) & 0xF
                a = ob.bf16_bits_to_f64([t.alpha[ni, ki // gs]])[0]
                b = ob.bf16_bits_to_f64([t.beta[ni, ki // gs]])[0]
                l = ob.bf16_bits_to_f64([t.lut[ni, q]])[0]
                f32 = ob.fraction_to_f32(Fraction(a) * Fraction(l) + Fraction(b))
                wv = float(ob.bf16_bits_to_f64(ob.f32_to_bf16_bits(np.array([f32])))[0])
                acc += xv[mi, ki] * wv
            assert y[mi, ni] == pytest.approx(acc, rel=1e-12, abs=1e-300)


def test_linear_unit_vectors_pick_columns():
    g = np.random.default_rng(14)
    n, k, gs = 5, 64, 32
    t = oracle.Any4Tensors(g.integers(0, 256, (n, k // 2), dtype=np.uint8),
                           _bits(g.uniform(-8, 7, (n, 16))), _bits(g.uniform(0.01, 0.1, (n, 2))),
                           _bits(g.normal(0, 0.01, (n, 2))), gs)
    x = _bits(np.eye(k))
    np.testing.assert_array_equal(oracle.linear(x, t), ob.bf16_bits_to_f64(oracle.dequant(t)).T)


def test_nibble_order_low_is_even():
    idx = np.array([[1, 2, 3, 4]], dtype=np.uint8)
    assert oracle.pack_nibbles(idx).tolist() == [[0x21, 0x43]]
    np.testing.assert_array_equal(oracle.unpack_nibbles(oracle.pack_nibbles(idx)), idx)


def test_algorithmic_bytes_table():
    # the per-call byte counts of the benchmark shapes
    assert oracle.algorithmic_bytes(1, 256, 512, 128) == 79_360
    assert oracle.algorithmic_bytes(1, 4096, 4096, 128) == 9_060_352
    assert oracle.algorithmic_bytes(16, 4096, 4096, 128) == 9_306_112
    assert oracle.algorithmic_bytes(1, 14336, 4096, 128) == 31_690_752
    assert oracle.algorithmic_bytes(1, 4096, 14336, 128) == 31_363_072
