"""Pins for the NF4 codebook: the construction's invariants, an independent quantile routine, and the
bin masses a normal sample must land in."""
import json
import math
import os

import numpy as np
import scipy.special as sps

import oracle as O
import synth

GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "page_figures.json")))


def test_ppf_bisection_matches_scipy_ndtri():
    """Error bound from the conditioning of Phi: one ulp of p moves x by ulp(p)/phi(x)."""
    for p in list(np.linspace(0.5 + 1e-9, 0.999, 97)) + [O.OFFSET, 0.75, 0.99]:
        x = O.normal_ppf(float(p))
        phi = math.exp(-x * x / 2) / math.sqrt(2 * math.pi)
        assert abs(x - sps.ndtri(p)) <= 4 * np.spacing(p) / phi + 4 * np.spacing(abs(x)), p
        assert abs(O.normal_cdf(x) - p) <= 4 * np.spacing(p)


def test_codebook_shape_and_exact_points():
    q, T = O.nf4_codebook()
    assert q.dtype == np.float32 and q.shape == (16,) and T.shape == (15,)
    assert O.OFFSET == GOLDEN["nf4_offset_probability"]["value"]
    assert q[0] == -1.0 and q[15] == 1.0
    assert q[7] == 0.0 and not np.signbit(q[7])                 # exact +0
    assert np.all(np.diff(q) > 0)
    assert int((q > 0).sum()) == GOLDEN["nf4_positive_levels"]["value"]
    assert int((q < 0).sum()) == GOLDEN["nf4_negative_levels"]["value"]


def test_levels_are_normal_quantiles_of_evenly_spaced_probabilities():
    """Mapped back through Phi, the positive levels sit at evenly spaced probabilities from 0.9677 to
    0.5 (step (0.9677-0.5)/8) and the negative ones at step (0.9677-0.5)/7."""
    q64 = O.nf4_levels_f64()
    z = sps.ndtri(O.OFFSET)
    pos = np.sort(q64[q64 > 0])[::-1]
    neg = np.sort(-q64[q64 < 0])[::-1]
    p_pos = sps.ndtr(pos * z)
    p_neg = sps.ndtr(neg * z)
    assert np.allclose(p_pos, O.OFFSET - np.arange(8) * (O.OFFSET - 0.5) / 8, atol=1e-13)
    assert np.allclose(p_neg, O.OFFSET - np.arange(7) * (O.OFFSET - 0.5) / 7, atol=1e-13)


def test_denser_near_zero_and_finer_positive_side():
    q = O.nf4_codebook()[0].astype(np.float64)
    pos_steps = np.diff(q[7:])          # 0 -> q8 -> ... -> 1
    neg_steps = np.diff(q[:8])[::-1]    # 0 -> q6 -> ... -> -1 (magnitudes)
    assert np.all(np.diff(pos_steps) > 0) and np.all(np.diff(neg_steps) > 0)
    assert np.all(pos_steps[:7] < neg_steps)       # the side with one more level has finer steps


def test_thresholds_are_rounded_midpoints():
    q, T = O.nf4_codebook()
    mid = (q[:-1].astype(np.float64) + q[1:]) / 2
    assert np.all(np.abs(T.astype(np.float64) - mid) <= np.spacing(np.abs(T)) / 2)
    assert np.all((q[:-1] < T) & (T < q[1:]))


def test_bin_masses_of_normal_samples():
    """N(0,1) samples divided by z* (the scale the levels were built for; no absmax) land in bin j with
    probability Phi(z* T_j) - Phi(z* T_{j-1}); the bins hold roughly equal mass (1/16 each)."""
    q, T = O.nf4_codebook()
    z = O.normal_ppf(O.OFFSET)
    n = 10_000_000
    x = (synth.rng(0, 11).standard_normal(n) / z).astype(np.float32)
    codes = O.nf4_codes(x, np.ones(-(-n // 64), np.float32), T)
    freq = np.bincount(codes, minlength=16) / n
    edges = np.concatenate([[-np.inf], T.astype(np.float64) * z, [np.inf]])
    expect = np.array([O.normal_cdf(edges[j + 1]) - O.normal_cdf(edges[j]) if np.isfinite(edges[j + 1])
                       else 1 - O.normal_cdf(edges[j]) for j in range(16)])
    expect[0] = O.normal_cdf(edges[1])
    sigma = np.sqrt(expect * (1 - expect) / n)
    assert np.all(np.abs(freq - expect) <= 5 * sigma), (freq, expect)
    assert np.all((freq[1:15] > 0.045) & (freq[1:15] < 0.085)), freq
    assert abs(expect.sum() - 1) < 1e-12
