"""The NF4 codebook: 16 levels from normal quantiles with an exact zero, and its decision thresholds.

Test infrastructure (see the package docstring).

Source: PEFT page (zerotofrontier.app/sft/peft), section "NF4, derived from normal quantiles".
The page builds the levels from the normal quantile function Phi^-1 evaluated at evenly spaced
probabilities, 8 on the positive side and 7 on the negative side, adds an exact 0, and rescales so the
largest magnitude is 1; the probabilities run from p = 0.9677 down to 0.5, which keeps clear of the
infinite Phi^-1(1).  The arXiv abstract (mlsanity.com, "QLoRA: Efficient Finetuning of Quantized
LLMs") and the QLoRA explainer (prism.theerrors.in, "The three innovations") name the goal: levels
used about equally often for normally distributed weights.

Readings (the page's formula was lost in extraction; the recipe in words is followed):
  * 0.9677 is taken literally.  The page remarks that it "equals" the mean of 1-1/30 and 1-1/32,
    which is 0.96770833...; that remark explains the constant and does not replace it.
  * Positive side: Phi^-1(p_i)/z* for the 9 evenly spaced probabilities from 0.9677 to 0.5 with the
    0.5 end dropped (8 levels).  Negative side: -Phi^-1(p_i)/z* for the 8 evenly spaced probabilities
    from 0.9677 to 0.5 with the 0.5 end dropped (7 levels).  z* = Phi^-1(0.9677), so both ends are
    exactly +-1.  Computed in fp64, then rounded once to fp32.
  * Decision thresholds T_j (j = 0..14) are the exact midpoints (q_j + q_{j+1})/2 of adjacent fp32
    levels, rounded once to fp32.  The pages say only "index of the nearest level"; how the codec uses
    T_j (strict comparison, ties to the lower index) is stated in codec.py.

Phi^-1 here is plain bisection on Phi(x) = erfc(-x/sqrt 2)/2 (the C library's erfc) down to adjacent
doubles; the CUDA library builds its copy of the table with a different method.
"""
from __future__ import annotations

import math

import numpy as np

OFFSET = 0.9677


def normal_cdf(x: float) -> float:
    return 0.5 * math.erfc(-x / math.sqrt(2.0))


def normal_ppf(p: float) -> float:
    """Smallest double x (to within one ulp) with Phi(x) >= p, by bisection.  0 < p < 1."""
    if not (0.0 < p < 1.0):
        raise ValueError("normal_ppf: p must lie in (0, 1)")
    lo, hi = -40.0, 40.0
    while True:
        mid = 0.5 * (lo + hi)
        if mid <= lo or mid >= hi:
            return hi
        if normal_cdf(mid) < p:
            lo = mid
        else:
            hi = mid


def nf4_levels_f64() -> np.ndarray:
    """The 16 NF4 levels in fp64, ascending: 7 negative, an exact 0, 8 positive; ends at -1 and +1."""
    z = normal_ppf(OFFSET)
    pos_p = np.linspace(OFFSET, 0.5, 9)[:-1]
    neg_p = np.linspace(OFFSET, 0.5, 8)[:-1]
    pos = [normal_ppf(float(p)) / z for p in pos_p]
    neg = [-normal_ppf(float(p)) / z for p in neg_p]
    levels = np.array(sorted(neg + [0.0] + pos), dtype=np.float64)
    return levels


def nf4_codebook():
    """(levels fp32[16], thresholds fp32[15]) as the codec uses them."""
    q = nf4_levels_f64().astype(np.float32)
    mid = (q[:-1].astype(np.float64) + q[1:].astype(np.float64)) / 2.0   # exact in fp64
    t = mid.astype(np.float32)
    return q, t
