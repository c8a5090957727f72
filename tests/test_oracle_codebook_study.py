"""Pins for the oracle's codebook study: the code rule against exact nearest-level search, the zero-code
reading, statistics on inputs whose answer is known in closed form, Lloyd's algorithm on a discrete
uniform distribution (whose optimum is the equal-cell partition) and the pages' comparison figures."""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle as O
from oracle import codebook_study as CS
import synth

GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "page_figures.json")))
INT4 = np.arange(-7, 8, dtype=np.float32) / np.float32(7)
GRID16 = np.arange(-8, 8, dtype=np.float32) / np.float32(8)


def _exact_nearest(w: float, a: float, levels) -> int:
    """Index of the level q_j minimising |w - q_j a| in rational arithmetic, the lower one on a tie."""
    W, A = Fraction(w), Fraction(a)
    d = [abs(W - Fraction(float(q)) * A) for q in levels]
    return d.index(min(d))


@pytest.mark.parametrize("a", [1.0, 0.7, 3.0e-3])
def test_grid_codes_are_exact_nearest(a):
    """The {-8..7}/8 grid has exact fp32 midpoints, so the threshold rule is nearest-level with ties to
    the lower index for every bf16 value in [-a, a], a tie included."""
    a = float(np.float32(a))
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    v = O.bf16_bits_to_f32(bits)
    v = v[np.isfinite(v) & (np.abs(v) <= a)]
    v = np.concatenate([v, (CS.thresholds(GRID16) * np.float32(a)).astype(np.float32)])   # exact ties
    v = v[np.abs(v) <= a]
    c1 = np.full(-(-v.size // 64), np.float32(a), np.float32)
    got = CS.codes(v, c1, GRID16)
    for i, w in enumerate(v.tolist()):
        assert got[i] == _exact_nearest(w, a, GRID16), (w, a)


def test_int4_codes_follow_the_threshold_rule():
    """Symmetric int4 has 15 levels: codes 0..14, nearest level except in the sub-ulp band where the
    rounded midpoint and the true one disagree."""
    x = synth.normal_f32(64 * 512, 1.0, 3, 1)
    c1 = O.absmax_blocks(x)
    got = CS.codes(x, c1, INT4)
    assert got.max() <= 14
    T = CS.thresholds(INT4)
    for i in range(0, x.size, 7):
        w, a = float(x[i]), float(c1[i // 64])
        near = _exact_nearest(w, a, INT4)
        by_thr = sum(Fraction(w) > Fraction(float(t)) * Fraction(a) for t in T)
        assert got[i] == by_thr
        mid = [Fraction(float(INT4[j])) / 2 + Fraction(float(INT4[j + 1])) / 2 for j in range(14)]
        if all((Fraction(w) > m * Fraction(a)) == (Fraction(w) > Fraction(float(t)) * Fraction(a))
               for m, t in zip(mid, T)):
            assert got[i] == near


def test_codes_with_the_nf4_levels_reduce_to_the_nf4_rule():
    q, T = O.nf4_codebook()
    x = synth.normal_f32(64 * 300 + 17, 1.0, 4, 2)
    x[64:128] = 0.0                                      # an all-zero block
    c1 = O.absmax_blocks(x)
    assert np.array_equal(CS.codes(x, c1, q), O.nf4_codes(x, c1, T))
    assert np.array_equal(CS.thresholds(q), T)


def test_zero_code_reading():
    q, _ = O.nf4_codebook()
    assert CS.zero_code(q) == 7
    assert CS.zero_code(INT4) == 7
    assert CS.zero_code(GRID16) == 8
    assert CS.zero_code([-1.0, -0.5, 0.5, 1.0]) == 1           # tie on magnitude: the lower index
    x = np.zeros(130, np.float32)
    c = CS.codes(x, O.absmax_blocks(x), GRID16)
    assert np.all(c == 8)


def test_levels_are_validated():
    for bad in ([0.5], [0.0, 0.0], [0.5, -0.5], [-1.0, 1.5], [-1.0, np.nan], list(np.linspace(-1, 1, 17))):
        with pytest.raises(ValueError):
            CS.check_levels(bad)


def test_statistics_of_inputs_that_sit_on_the_levels():
    """Every block holds each of the 16 grid levels four times and absmax 1, so every element is
    recovered exactly: no error, 4 bits of entropy, each level its own centroid."""
    blk = np.repeat(GRID16, 4)
    x = np.concatenate([np.roll(blk, 3 * b) for b in range(40)]).astype(np.float32)
    packed, c1 = CS.quantize(x, GRID16)
    assert np.all(c1 == 1.0)
    st = CS.stats(x, packed, c1, GRID16)
    assert st["sse"] == 0.0 and st["rms"] == 0.0
    assert np.all(st["counts"] == 160)
    assert st["entropy_bits"] == 4.0
    assert np.array_equal(st["sums"], 160 * GRID16.astype(np.float64))
    assert np.array_equal(st["centroids"], GRID16)
    assert np.array_equal(CS.dequantize(packed, c1, x.size, GRID16), x)


def test_statistics_two_point_and_known_error():
    """Half the elements at -a (the level -1, exact) and half an eighth of a step off the level 1/2:
    1 bit of entropy and a known squared error."""
    a = np.float32(2.0)
    x = np.tile(np.array([-a, a * np.float32(0.5) + np.float32(1 / 32)], np.float32), 64 * 8)
    packed, c1 = CS.quantize(x, GRID16)
    st = CS.stats(x, packed, c1, GRID16)
    assert st["entropy_bits"] == 1.0
    # 0.5 * a + 1/32 = a * (0.5 + 1/64): nearest grid level 4/8, error 1/32 on half of the elements
    assert st["sse"] == (x.size // 2) * (1 / 32) ** 2
    assert math.isclose(st["rms"], math.sqrt(0.5) / 32, rel_tol=1e-15)


def test_lloyd_finds_the_equal_cell_partition_of_a_discrete_uniform():
    """64 equally spaced normalised values (odd multiples of 1/64 over absmax 63/64, so u runs from -1
    to 1 in steps of 2/63): the 4-level squared-error optimum splits them into four cells of 16, with
    levels at the cell means +-16/63 and +-48/63, a fixed point of the iteration."""
    blk = ((2 * np.arange(64) + 1 - 64) / 64).astype(np.float32)
    x = np.concatenate([np.roll(blk, 5 * b) for b in range(32)]).astype(np.float32)
    lv, hist = CS.lloyd(x, [-0.9, -0.1, 0.1, 0.9], 3)
    want = np.array([-48, -16, 16, 48], np.float64) / 63
    assert np.allclose(lv.astype(np.float64), want, rtol=0, atol=2 ** -24)
    st = CS.stats(x, CS.quantize(x, lv)[0], O.absmax_blocks(x), lv)
    assert np.all(st["counts"][:4] == 16 * 32)
    assert hist[1] <= hist[0] and abs(hist[-1] - hist[1]) <= 1e-12


def test_lloyd_never_increases_the_error_on_gaussian_data():
    x = synth.normal_f32(64 * 1024, 1.0, 5, 3)
    q, _ = O.nf4_codebook()
    _, hist = CS.lloyd(x, q, 8)
    for before, after in zip(hist, hist[1:]):
        assert after <= before * (1 + 1e-9)
    assert hist[-1] < hist[0]


def test_the_page_comparison_figures():
    """A Gaussian matrix in blocks of 64 with fp32 constants: NF4 3.88 bits of entropy against 3.50 for
    symmetric int4, RMS error about 15 % lower, the {-8..7}/8 grid in between, and Lloyd's codebook
    (started from NF4) about 5 % better than NF4."""
    x = synth.normal_f32((1024, 1024), 1.0, 0, 16).reshape(-1)
    q, _ = O.nf4_codebook()
    r = CS.study(x, q, lloyd_iters=30)
    assert abs(r["nf4"]["entropy_bits"] - GOLDEN["entropy_bits_nf4"]["value"]) < 0.02
    assert abs(r["int4_symmetric"]["entropy_bits"] - GOLDEN["entropy_bits_int4_symmetric"]["value"]) < 0.02
    red = 1 - r["nf4"]["rms"] / r["int4_symmetric"]["rms"]
    assert abs(red - GOLDEN["rms_reduction_nf4_vs_int4"]["value"]) < 0.03, red
    assert r["nf4"]["rms"] < r["grid_16"]["rms"] < r["int4_symmetric"]["rms"]
    gain = 1 - r["lloyd"]["rms"] / r["nf4"]["rms"]
    assert abs(gain - GOLDEN["lloyd_gain_over_nf4"]["value"]) < 0.03, gain
    assert np.all(np.diff(r["lloyd"]["levels"].astype(np.float64)) > 0)
