"""Pins for the CPU oracle: each check ties it to something other than itself.

Sources of truth used here (never the oracle, never the CUDA path):
  * numpy's float16 cast and float32 division (IEEE library routines),
  * Python's exact rational arithmetic (fractions.Fraction, round-half-even round()),
  * numpy int64 matmul,
  * closed forms and invariances of Y = sum_g P_g * sa * sw,
  * the crossover table printed on the page "Why INT4 Weight-Only Quantization Doesn't
    Speed Up Prefill" (tests/golden/crossover_table.txt).
The method: "APEX4: Efficient Pure W4A4 LLM Inference via Intra-SM Compute
Rebalancing", abstract (pure INT4 W4A4 GEMM with 128-wide groups, INT4 products
dequantised per group on the CUDA cores).
"""
import os
from fractions import Fraction

import numpy as np
import pytest

from group_quantized_w4a4_b200 import roofline, synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ------------------------------------------------------------------ independent helpers

def np_unpack(packed: np.ndarray, K: int) -> np.ndarray:
    """Nibble unpack written from the byte formula (low nibble = even k)."""
    b = packed.astype(np.int16)
    lo = b & 0xF
    hi = (b >> 4) & 0xF
    lo = np.where(lo >= 8, lo - 16, lo)
    hi = np.where(hi >= 8, hi - 16, hi)
    q = np.empty((packed.shape[0], K), dtype=np.int64)
    q[:, 0::2] = lo
    q[:, 1::2] = hi
    return q


def np_pack(q: np.ndarray) -> np.ndarray:
    q = q.astype(np.int64)
    return ((q[:, 0::2] & 0xF) | ((q[:, 1::2] & 0xF) << 4)).astype(np.uint8)


def rational_quantize_row(xrow: np.ndarray, group: int):
    """Quantizer re-derived with exact rationals: s from an IEEE fp32 division rounded
    to fp16 by numpy, q = round_half_even(x / s) on the exact quotient, clamped."""
    K = xrow.size
    scales, qs = [], []
    for g in range(K // group):
        xs = xrow[g * group:(g + 1) * group]
        amax = np.max(np.abs(xs.astype(np.float32)))
        s = np.float16(np.float32(amax) / np.float32(7.0))
        scales.append(s)
        sf = Fraction(float(s))
        for v in xs:
            if sf == 0:
                qs.append(0)
            else:
                q = round(Fraction(float(v)) / sf)   # Python rounds halves to even
                qs.append(max(-8, min(7, q)))
    return np.array(scales, dtype=np.float16), np.array(qs, dtype=np.int64)


def dequant(q: np.ndarray, s: np.ndarray, group: int) -> np.ndarray:
    return q.astype(np.float64) * np.repeat(s.astype(np.float64), group, axis=1)


# ------------------------------------------------------------------ fp16 conversion

def test_f32_to_f16_matches_numpy(oracle_mod):
    rng = np.random.default_rng(7)
    edge = np.array([0.0, -0.0, 1.0, -1.0, 65504.0, 65519.99, 65520.0, 1e9, -1e9,
                     2.0 ** -14, 2.0 ** -24, 2.0 ** -25, 3 * 2.0 ** -26, 2.0 ** -26,
                     1.5 * 2.0 ** -24, 2.5 * 2.0 ** -24, (1 + 2 ** -11) * 1.0,
                     (1 + 3 * 2 ** -11), (1 + 2 ** -11 + 2 ** -20), 2.0 ** -14 * (1 - 2 ** -12),
                     np.inf, -np.inf], dtype=np.float32)
    bits = rng.integers(0, 2 ** 32, size=20000, dtype=np.uint64).astype(np.uint32)
    rand = bits.view(np.float32)
    rand = rand[np.isfinite(rand)]
    wide = (rng.standard_normal(5000) * 10.0 ** rng.uniform(-9, 5, 5000)).astype(np.float32)
    vals = np.concatenate([edge, rand, wide])
    got = oracle_mod.f32_to_f16(vals)
    with np.errstate(over="ignore"):
        want = vals.astype(np.float16).view(np.uint16)
    assert np.array_equal(got, want)
    nan = oracle_mod.f32_to_f16(np.array([np.nan], dtype=np.float32))
    assert np.isnan(nan.view(np.float16)[0])


# ------------------------------------------------------------------ quantizer

def _quant_inputs():
    rng = np.random.default_rng(11)
    rows = []
    rows.append(rng.standard_normal(512))
    rows.append(rng.standard_normal(512) * 0.02)
    r = rng.standard_normal(512)
    r[rng.choice(512, 6, replace=False)] *= 20.0
    rows.append(r)
    rows.append(rng.standard_t(4, 512) / np.sqrt(2))
    rows.append(rng.standard_normal(512) * 1e-5)          # subnormal-range scales
    r = np.zeros(512)
    r[128:256] = rng.standard_normal(128) * 3e-8           # scale underflows to 0
    r[256:384] = rng.integers(-7, 8, 128) * 0.5            # many exact halves
    rows.append(r)
    return np.array(rows).astype(np.float16)


def test_quantize_matches_exact_rationals(oracle_mod):
    x = _quant_inputs()
    packed, scales = oracle_mod.quantize_pack(x, 128)
    for r in range(x.shape[0]):
        s_ref, q_ref = rational_quantize_row(x[r], 128)
        assert np.array_equal(scales[r].view(np.uint16), s_ref.view(np.uint16)), r
        assert np.array_equal(packed[r], np_pack(q_ref[None, :])[0]), r


@pytest.mark.parametrize("group", [128, 512])
def test_quantize_random_groups_exact(oracle_mod, group):
    x = synth.activations(8, 1024, "outlier", 5)
    packed, scales = oracle_mod.quantize_pack(x, group)
    for r in range(x.shape[0]):
        s_ref, q_ref = rational_quantize_row(x[r], group)
        assert np.array_equal(scales[r].view(np.uint16), s_ref.view(np.uint16))
        assert np.array_equal(np_unpack(packed[r:r + 1], 1024)[0], q_ref)


def test_quantize_ties_round_half_even(oracle_mod):
    # absmax 7 gives s = 1 exactly, so q = round_half_even(x).
    halves = [0.5, 1.5, 2.5, -0.5, -1.5, -2.5, 3.5, 4.5, 5.5, 6.5, -6.5, 0.25, 0.75]
    want = [0, 2, 2, 0, -2, -2, 4, 4, 6, 6, -6, 0, 1]
    assert want == [round(Fraction(h)) for h in halves]   # textbook banker's rounding
    g = np.zeros(128)
    g[0] = 7.0
    g[1:1 + len(halves)] = halves
    packed, scales = oracle_mod.quantize_pack(g[None, :].astype(np.float16), 128)
    assert float(scales[0, 0]) == 1.0
    q = np_unpack(packed, 128)[0]
    assert q[0] == 7
    assert list(q[1:1 + len(halves)]) == want


def test_quantize_absmax_and_roundtrip_bound(oracle_mod):
    x = synth.activations(16, 2048, "student_t", 9)
    packed, scales = oracle_mod.quantize_pack(x, 128)
    q = np_unpack(packed, 2048)
    s = np.repeat(scales.astype(np.float64), 128, axis=1)
    xf = x.astype(np.float64)
    normal = s >= 2.0 ** -14
    assert normal.all()
    assert np.all(np.abs(xf - q * s) <= s / 2)
    for r in range(16):
        for g in range(16):
            sl = slice(g * 128, (g + 1) * 128)
            i = np.argmax(np.abs(xf[r, sl]))
            assert abs(q[r, sl][i]) == 7
    assert q.min() >= -7 and q.max() <= 7          # -8 is unreachable for this rule


def test_quantize_zero_and_underflow_groups(oracle_mod):
    x = np.zeros((2, 256), dtype=np.float16)
    x[1, 128:] = np.float16(2.0 ** -24)            # absmax/7 rounds to fp16 zero
    packed, scales = oracle_mod.quantize_pack(x, 128)
    assert np.all(scales.view(np.uint16) == 0)
    assert np.all(packed == 0)


# ------------------------------------------------------------------ pack / unpack

def test_unpack_explicit_byte_formula(oracle_mod):
    b = np.arange(256, dtype=np.uint8).reshape(2, 128)
    q = oracle_mod.unpack(b, 256)
    for byte in range(256):
        r, j = divmod(byte, 128)
        lo, hi = byte & 0xF, byte >> 4
        lo = lo - 16 if lo >= 8 else lo
        hi = hi - 16 if hi >= 8 else hi
        assert q[r, 2 * j] == lo and q[r, 2 * j + 1] == hi


def test_pack_unpack_roundtrip(oracle_mod):
    rng = np.random.default_rng(3)
    q = rng.integers(-8, 8, size=(5, 384))
    assert np.array_equal(oracle_mod.unpack(np_pack(q), 384).astype(np.int64), q)


# ------------------------------------------------------------------ integer partials

@pytest.mark.parametrize("ga,gw", [(128, 128), (128, 512), (128, 1024), (256, 128)])
def test_partials_equal_numpy_int_matmul(oracle_mod, ga, gw):
    rng = np.random.default_rng(ga + gw)
    M, N, K = 5, 7, 1024
    ap = rng.integers(0, 256, size=(M, K // 2), dtype=np.uint8)   # includes -8 nibbles
    wp = rng.integers(0, 256, size=(N, K // 2), dtype=np.uint8)
    P = oracle_mod.group_partials(ap, wp, M, N, K, ga, gw)
    qa, qw = np_unpack(ap, K), np_unpack(wp, K)
    ge = min(ga, gw)
    assert P.shape == (K // ge, M, N)
    for g in range(K // ge):
        sl = slice(g * ge, (g + 1) * ge)
        assert np.array_equal(P[g], qa[:, sl] @ qw[:, sl].T)
    assert np.array_equal(P.sum(axis=0), qa @ qw.T)
    rows = np.array([4, 0, 2])
    Pr = oracle_mod.group_partials(ap, wp, M, N, K, ga, gw, rows=rows)
    assert np.array_equal(Pr, P[:, rows, :])


def test_partials_extreme_values(oracle_mod):
    K = 256
    ap = np.full((2, K // 2), 0x88, dtype=np.uint8)               # all -8
    wp = np.stack([np.full(K // 2, 0x88, np.uint8), np.full(K // 2, 0x77, np.uint8)])
    P = oracle_mod.group_partials(ap, wp, 2, 2, K, 128, 128)
    assert np.all(P[:, :, 0] == 128 * 64)
    assert np.all(P[:, :, 1] == -128 * 56)


# ------------------------------------------------------------------ output

def _random_problem(rng, M, N, K, ga, gw):
    ap = rng.integers(0, 256, size=(M, K // 2), dtype=np.uint8)
    wp = rng.integers(0, 256, size=(N, K // 2), dtype=np.uint8)
    sa = (rng.uniform(0.05, 2.0, size=(M, K // ga))).astype(np.float16)
    sw = (rng.uniform(0.001, 0.02, size=(N, K // gw))).astype(np.float16)
    return ap, sa, wp, sw


@pytest.mark.parametrize("ga,gw", [(128, 128), (128, 512), (128, 1024), (512, 128)])
def test_gemm_brute_force_dequantised(oracle_mod, ga, gw):
    rng = np.random.default_rng(17 + gw)
    M, N, K = 6, 9, 1024
    ap, sa, wp, sw = _random_problem(rng, M, N, K, ga, gw)
    y = oracle_mod.gemm(ap, sa, wp, sw, M, N, K, ga, gw)
    ref = dequant(np_unpack(ap, K), sa, ga) @ dequant(np_unpack(wp, K), sw, gw).T
    assert np.max(np.abs(y - ref)) <= 1e-12 * np.max(np.abs(ref))


def test_gemm_from_quantized_fp16_inputs(oracle_mod):
    a = synth.activations(4, 512, "normal", 21)
    w = synth.weights(6, 512, 21)
    ap, sa = oracle_mod.quantize_pack(a, 128)
    wp, sw = oracle_mod.quantize_pack(w, 128)
    y = oracle_mod.gemm(ap, sa, wp, sw, 4, 6, 512, 128, 128)
    ref = dequant(np_unpack(ap, 512), sa, 128) @ dequant(np_unpack(wp, 512), sw, 128).T
    assert np.max(np.abs(y - ref)) <= 1e-12 * np.max(np.abs(ref))
    # and the quantized product approximates the fp16 product
    exact = a.astype(np.float64) @ w.astype(np.float64).T
    assert np.max(np.abs(y - exact)) < 0.2 * np.max(np.abs(exact))


def test_gemm_group_equals_k_closed_form(oracle_mod):
    rng = np.random.default_rng(23)
    M, N, K = 5, 6, 768
    ap, sa, wp, sw = _random_problem(rng, M, N, K, K, K)
    y = oracle_mod.gemm(ap, sa, wp, sw, M, N, K, K, K)
    I = np_unpack(ap, K) @ np_unpack(wp, K).T
    closed = sa.astype(np.float64)[:, :1] * sw.astype(np.float64)[:, 0][None, :] * I
    assert np.array_equal(y, closed)


def test_gemm_within_group_permutation_invariance(oracle_mod):
    rng = np.random.default_rng(29)
    M, N, K = 4, 5, 512
    ap, sa, wp, sw = _random_problem(rng, M, N, K, 128, 128)
    qa, qw = np_unpack(ap, K), np_unpack(wp, K)
    perm = np.concatenate([g * 128 + rng.permutation(128) for g in range(K // 128)])
    y0 = oracle_mod.gemm(ap, sa, wp, sw, M, N, K, 128, 128)
    y1 = oracle_mod.gemm(np_pack(qa[:, perm]), sa, np_pack(qw[:, perm]), sw, M, N, K, 128, 128)
    assert np.array_equal(y0, y1)
    # a permutation that crosses groups changes the answer (the pin is sensitive)
    cross = np.roll(np.arange(K), 64)
    y2 = oracle_mod.gemm(np_pack(qa[:, cross]), sa, np_pack(qw[:, cross]), sw, M, N, K, 128, 128)
    assert not np.array_equal(y0, y2)


def test_gemm_power_of_two_linearity(oracle_mod):
    rng = np.random.default_rng(31)
    M, N, K = 4, 6, 512
    ap, sa, wp, sw = _random_problem(rng, M, N, K, 128, 128)
    y0 = oracle_mod.gemm(ap, sa, wp, sw, M, N, K, 128, 128)
    sw2 = sw.copy()
    sw2[2] = (sw2[2].astype(np.float32) * 2).astype(np.float16)
    sa2 = sa.copy()
    sa2[1] = (sa2[1].astype(np.float32) * 0.5).astype(np.float16)
    y1 = oracle_mod.gemm(ap, sa2, wp, sw2, M, N, K, 128, 128)
    want = y0.copy()
    want[:, 2] *= 2
    want[1, :] *= 0.5
    assert np.array_equal(y1, want)


def test_gemm_row_subset(oracle_mod):
    rng = np.random.default_rng(37)
    M, N, K = 9, 5, 256
    ap, sa, wp, sw = _random_problem(rng, M, N, K, 128, 128)
    y = oracle_mod.gemm(ap, sa, wp, sw, M, N, K, 128, 128)
    rows = np.array([8, 3, 0])
    assert np.array_equal(oracle_mod.gemm(ap, sa, wp, sw, M, N, K, 128, 128, rows=rows), y[rows])


def test_brute_force_pin_catches_planted_mistakes(oracle_mod):
    """The brute-force pin must reject plausible oracle mistakes: swapped group sizes
    (wrong scale index), a wrong row index and a dropped group."""
    rng = np.random.default_rng(41)
    M, N, K = 6, 6, 1024
    ap, sa, wp, sw = _random_problem(rng, M, N, K, 128, 512)
    ref = dequant(np_unpack(ap, K), sa, 128) @ dequant(np_unpack(wp, K), sw, 512).T
    tol = 1e-12 * np.max(np.abs(ref))
    good = oracle_mod.gemm(ap, sa, wp, sw, M, N, K, 128, 512)
    assert np.max(np.abs(good - ref)) <= tol
    # wrong scale indexing: treat the weight scales as g128 (index g instead of g/4)
    sw_wrong = np.repeat(sw, 4, axis=1)[:, ::1][:, :K // 128]
    sw_wrong = np.ascontiguousarray(np.roll(sw_wrong, 1, axis=1))
    bad = oracle_mod.gemm(ap, sa, wp, sw_wrong, M, N, K, 128, 128)
    assert np.max(np.abs(bad - ref)) > tol
    # wrong weight-row index (rows read in reverse order)
    bad2 = oracle_mod.gemm(ap, sa, np.ascontiguousarray(wp[::-1]), sw, M, N, K, 128, 512)
    assert np.max(np.abs(bad2 - ref)) > tol
    # dropped last group (the g512 weight scales restated per 128-wide group)
    sw128 = np.repeat(sw, 4, axis=1)
    assert np.max(np.abs(oracle_mod.gemm(ap, sa, wp, sw128, M, N, K, 128, 128) - ref)) <= tol
    bad3 = oracle_mod.gemm(ap[:, :-64], sa[:, :-1], wp[:, :-64], sw128[:, :-1],
                           M, N, K - 128, 128, 128)
    assert bad3.shape == ref.shape and np.max(np.abs(bad3 - ref)) > tol


# ------------------------------------------------------------------ outlier dual path
# "OSC: Hardware Efficient W4A4 Quantization via Outlier Separation in Channel Dimension",
# abstract: fixed outlier channels go through a 16-bit branch GEMM, the rest through the
# 4-bit GEMM.


def _dual_inputs(rng, M, N, K, n_out, boost=20.0):
    ch = np.sort(rng.choice(K, size=n_out, replace=False))
    x = rng.standard_normal((M, K)).astype(np.float32)
    x[:, ch] *= np.float32(boost)
    w = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    return x.astype(np.float16), w.astype(np.float16), ch


def _dual_by_oracle(oracle_mod, x, w, ch, gw=128):
    M, K = x.shape
    N = w.shape[0]
    x_in, x_out = oracle_mod.split_outlier_channels(x, ch)
    ap, sa = oracle_mod.quantize_pack(x_in, 128)
    wp, sw = oracle_mod.quantize_pack(w, gw)
    y = oracle_mod.gemm_dual(ap, sa, wp, sw, x_out, np.ascontiguousarray(w[:, ch]),
                             M, N, K, 128, gw)
    return y, (ap, sa, wp, sw)


def _mixed_reference(x, w, ch, ops, gw=128):
    """Element-level restatement on full-width operands: channel k contributes
    x[m,k] w[n,k] (fp16 values) when it is an outlier channel, else the product of the
    dequantised int4 values; one fp64 matmul of the two mixed matrices."""
    ap, sa, wp, sw = ops
    K = x.shape[1]
    xd = dequant(np_unpack(ap, K), sa, 128)
    wd = dequant(np_unpack(wp, K), sw, gw)
    mask = np.zeros(K, dtype=bool)
    mask[ch] = True
    xm = np.where(mask[None, :], x.astype(np.float64), xd)
    wm = np.where(mask[None, :], w.astype(np.float64), wd)
    return xm @ wm.T


@pytest.mark.parametrize("gw", [128, 512])
def test_dual_path_matches_element_level_restatement(oracle_mod, gw):
    rng = np.random.default_rng(61)
    x, w, ch = _dual_inputs(rng, 7, 9, 1024, 11)
    y, ops = _dual_by_oracle(oracle_mod, x, w, ch, gw)
    ref = _mixed_reference(x, w, ch, ops, gw)
    assert np.max(np.abs(y - ref)) <= 1e-12 * np.max(np.abs(ref))
    # the 4-bit operands see the outlier channels as zeros
    assert not np.any(np_unpack(ops[0], 1024)[:, ch])


def test_dual_path_outlier_only_input_is_the_fp16_product(oracle_mod):
    rng = np.random.default_rng(62)
    x, w, ch = _dual_inputs(rng, 5, 6, 512, 9)
    only = np.zeros_like(x)
    only[:, ch] = x[:, ch]
    y, ops = _dual_by_oracle(oracle_mod, only, w, ch)
    assert not np.any(ops[1].astype(np.float32))       # every group scale is 0
    ref = only.astype(np.float64) @ w.astype(np.float64).T
    assert np.max(np.abs(y - ref)) <= 1e-12 * np.max(np.abs(ref))


def test_dual_path_without_outlier_channels_is_the_w4a4_gemm(oracle_mod):
    rng = np.random.default_rng(63)
    x, w, _ = _dual_inputs(rng, 4, 5, 384, 3)
    y, ops = _dual_by_oracle(oracle_mod, x, w, np.array([], dtype=np.int64))
    ap, sa, wp, sw = ops
    assert np.array_equal(y, oracle_mod.gemm(ap, sa, wp, sw, 4, 5, 384, 128, 128))


def test_dual_path_cuts_the_error_of_outlier_channels(oracle_mod):
    """What the dual path is for: on token-persistent outlier channels the error against
    the exact product of the fp16 operands drops well below the single 4-bit path's."""
    M, N, K = 8, 16, 2048
    x = synth.activations(M, K, "outlier", 5)
    w = synth.weights(N, K, 5)
    ch = synth.outlier_channels(K, 5 * 16 + 2)
    exact = x.astype(np.float64) @ w.astype(np.float64).T
    dual, _ = _dual_by_oracle(oracle_mod, x, w, ch)
    ap, sa = oracle_mod.quantize_pack(x, 128)
    wp, sw = oracle_mod.quantize_pack(w, 128)
    single = oracle_mod.gemm(ap, sa, wp, sw, M, N, K, 128, 128)
    e_dual = np.sqrt(np.mean((dual - exact) ** 2))
    e_single = np.sqrt(np.mean((single - exact) ** 2))
    assert e_dual < 0.5 * e_single


def test_dual_pin_catches_planted_mistakes(oracle_mod):
    """Plausible mistakes in the dual path, planted on the CPU, each fail the
    element-level restatement: outliers left in the 4-bit operands, the 16-bit branch
    dropped, and branch weights taken in the wrong channel order."""
    rng = np.random.default_rng(64)
    M, N, K = 6, 8, 1024
    x, w, ch = _dual_inputs(rng, M, N, K, 11)
    y, ops = _dual_by_oracle(oracle_mod, x, w, ch)
    ref = _mixed_reference(x, w, ch, ops)
    tol = 1e-12 * np.max(np.abs(ref))
    assert np.max(np.abs(y - ref)) <= tol
    ap, sa, wp, sw = ops
    x_out = np.ascontiguousarray(x[:, ch])
    w_out = np.ascontiguousarray(w[:, ch])
    # outliers not zeroed before quantizing (counted on both paths)
    ap_bad, sa_bad = oracle_mod.quantize_pack(x, 128)
    bad = oracle_mod.gemm_dual(ap_bad, sa_bad, wp, sw, x_out, w_out, M, N, K, 128, 128)
    assert np.max(np.abs(bad - ref)) > tol
    # the branch dropped
    assert np.max(np.abs(oracle_mod.gemm(ap, sa, wp, sw, M, N, K, 128, 128) - ref)) > tol
    # branch weights in reverse channel order
    bad = oracle_mod.gemm_dual(ap, sa, wp, sw, x_out, np.ascontiguousarray(w_out[:, ::-1]),
                               M, N, K, 128, 128)
    assert np.max(np.abs(bad - ref)) > tol


def test_split_outlier_channels_argument_rules(oracle_mod):
    x = np.zeros((2, 8), dtype=np.float16)
    with pytest.raises(ValueError):
        oracle_mod.split_outlier_channels(x, [1, 1])
    with pytest.raises(ValueError):
        oracle_mod.split_outlier_channels(x, [8])
    with pytest.raises(TypeError):
        oracle_mod.split_outlier_channels(x.astype(np.float32), [1])


def test_tolerance_rule():
    ok, _ = __import__("oracle").within_tolerance([1.0, 2.0], [1.0, 2.001])
    assert ok
    ok, _ = __import__("oracle").within_tolerance([1.0, 2.1], [1.0, 2.0])
    assert not ok


# ------------------------------------------------------------------ roofline helper

def test_crossover_table_from_page():
    rows = []
    with open(os.path.join(GOLDEN, "crossover_table.txt")) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                gpu, fl, bw, b, printed = line.split()
                rows.append((gpu, float(fl), float(bw), float(b), int(printed)))
    assert len(rows) == 5
    for gpu, fl, bw, b, printed in rows:
        got = roofline.crossover_tokens(fl, bw, b)
        assert int(round(got)) == printed, (gpu, b, got)


def test_bound_time():
    t, which = roofline.bound_time_s(2e12, 1e9, 1e15, 1e12)
    assert which == "tensor" and t == pytest.approx(2e-3)
    t, which = roofline.bound_time_s(1e9, 1e10, 1e15, 1e12)
    assert which == "hbm" and t == pytest.approx(1e-2)
