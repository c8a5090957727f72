"""The codebook comparison: blockwise absmax quantization with fp32 block constants under any sorted
codebook of 2 to 16 levels, the statistics of the codes it produces, and Lloyd's algorithm.

Test infrastructure (see the package docstring).

Sources:
  PEFT page (zerotofrontier.app/sft/peft), "NF4, derived from normal quantiles": a large matrix of
    Gaussian weights is quantized in blocks of 64 with three codebooks (the symmetric int4 grid
    {-7..7}/7, the 16-level grid {-8..7}/8 and NF4) and with the codebook of least squared error, found
    by Lloyd's algorithm (k-means in one dimension). NF4's RMS error is about 15 % below symmetric int4,
    its codes carry 3.88 bits of entropy against 3.50, and the Lloyd codebook is about 5 % better again.
  "Block-wise quantization in one page": blocks of consecutive values, one absmax constant each, the
    index of the nearest level, and the value recovered as level times constant.

Readings where the pages leave a step open:
  R-cb-thr   the decision thresholds are the level midpoints (q_j + q_{j+1}) / 2, the sum formed in
             fp64 and the half rounded once to fp32; the code of w in a block with absmax a > 0 is
             #{j : w > T_j * a} in exact arithmetic (the NF4 codec's tie rule), so it never exceeds
             nlev - 1.
  R-cb-zero  a block whose absmax is 0 codes every element as the index of the level of least
             magnitude (the lower index on a tie); for NF4 that is 7, its exact zero.
  R-cb-u     the normalised value of an element is u = w / a in fp64, correctly rounded; u = 0 in a
             block with a = 0.
  R-cb-err   the error of an element is w_hat - w in fp64, w_hat = RN32(q[code] * a) being the fp32
             value the dequantizer writes; RMS = sqrt(sum of squared errors / n).
  R-cb-ent   code entropy = -sum_j p_j log2 p_j over the code frequencies p_j, with 0 log 0 = 0.
  R-cb-lloyd one Lloyd step: assign every element by the code rule above with the current fp32 levels,
             then replace each level by the fp64 mean of the u values assigned to it, rounded to fp32;
             a level that received no element keeps its value. The study starts it from NF4.
"""
from __future__ import annotations

import math

import numpy as np

from .codec import BLOCK, absmax_blocks, as_f32_values, num_blocks, pack_codes, unpack_codes
from .lowp import rn32_mul, bf16_rne_bits

_CHUNK = 1 << 22          # a multiple of BLOCK


def check_levels(levels) -> np.ndarray:
    """The levels as fp32, after checking they are 2..16 finite values in [-1, 1], strictly ascending."""
    q = np.asarray(levels, dtype=np.float32).reshape(-1)
    if not 2 <= q.size <= 16 or not np.all(np.isfinite(q)) or np.any(np.abs(q) > 1):
        raise ValueError("levels: 2 to 16 finite values in [-1, 1]")
    if np.any(np.diff(q.astype(np.float64)) <= 0):
        raise ValueError("levels: strictly ascending")
    return q


def thresholds(levels) -> np.ndarray:
    """T_j = RN32((q_j + q_{j+1}) / 2) with the sum in fp64 (reading R-cb-thr)."""
    q = check_levels(levels).astype(np.float64)
    return ((q[:-1] + q[1:]) / 2).astype(np.float32)


def zero_code(levels) -> int:
    """Index of the level of least magnitude, the lower on a tie (reading R-cb-zero)."""
    q = np.abs(check_levels(levels).astype(np.float64))
    return int(np.argmin(q))          # argmin returns the first minimum


def codes(w32: np.ndarray, c1: np.ndarray, levels) -> np.ndarray:
    """One code per element (unpacked uint8) per readings R-cb-thr and R-cb-zero."""
    w32 = np.asarray(w32, dtype=np.float32).reshape(-1)
    T64 = thresholds(levels).astype(np.float64)
    z = zero_code(levels)
    out = np.empty(w32.size, dtype=np.uint8)
    for s in range(0, w32.size, _CHUNK):
        w = w32[s:s + _CHUNK].astype(np.float64)
        a = np.repeat(c1[s // BLOCK:(s + w.size + BLOCK - 1) // BLOCK].astype(np.float64), BLOCK)[:w.size]
        cnt = np.zeros(w.size, dtype=np.int64)
        for t in T64:
            cnt += w > t * a                 # t * a: a product of two fp32 values, exact in fp64
        out[s:s + w.size] = np.where(a == 0.0, z, cnt)
    return out


def quantize(w, levels):
    """Packed codes (two per byte, even element in the high nibble) and the fp32 block absmax."""
    w32 = as_f32_values(w)
    c1 = absmax_blocks(w32)
    return pack_codes(codes(w32, c1, levels)), c1


def dequantize(packed: np.ndarray, c1: np.ndarray, n: int, levels, out: str = "f32") -> np.ndarray:
    """w_hat = RN32(q[code] * c1_b); bf16 output as uint16 bit patterns (round to nearest even)."""
    q = np.zeros(16, dtype=np.float32)
    lv = check_levels(levels)
    q[:lv.size] = lv
    c = unpack_codes(packed, n)
    w = np.empty(n, dtype=np.float32)
    for s in range(0, n, _CHUNK):
        m = min(_CHUNK, n - s)
        a = np.repeat(np.asarray(c1, np.float32)[s // BLOCK:(s + m + BLOCK - 1) // BLOCK], BLOCK)[:m]
        w[s:s + m] = rn32_mul(q[c[s:s + m]], a)
    if out == "f32":
        return w
    if out == "bf16":
        return bf16_rne_bits(w)
    raise ValueError(out)


def entropy_bits(counts) -> float:
    """Reading R-cb-ent."""
    c = np.asarray(counts, dtype=np.float64)
    p = c[c > 0] / c.sum()
    return float(-(p * np.log2(p)).sum())


def stats(w, packed: np.ndarray, c1: np.ndarray, levels) -> dict:
    """Per level: how many elements took it and the fp64 sum of their u; over all elements the sum of
    squared errors; from these the entropy, the RMS error and the Lloyd update of the levels."""
    w32 = as_f32_values(w)
    n = w32.size
    lv = check_levels(levels)
    nl = lv.size
    c = unpack_codes(packed, n).astype(np.int64)
    counts = np.zeros(16, dtype=np.int64)
    sums = np.zeros(16, dtype=np.float64)
    sse = 0.0
    for s in range(0, n, _CHUNK):
        m = min(_CHUNK, n - s)
        x = w32[s:s + m].astype(np.float64)
        a = np.repeat(np.asarray(c1, np.float64)[s // BLOCK:(s + m + BLOCK - 1) // BLOCK], BLOCK)[:m]
        u = np.divide(x, a, out=np.zeros_like(x), where=a != 0.0)           # R-cb-u
        cs = c[s:s + m]
        counts += np.bincount(cs, minlength=16)
        sums += np.bincount(cs, weights=u, minlength=16)
        wh = rn32_mul(lv[cs], np.asarray(a, np.float32)).astype(np.float64)  # R-cb-err
        sse += float(((wh - x) ** 2).sum())
    cent = lv.copy()
    for j in range(nl):
        if counts[j] > 0:
            cent[j] = np.float32(sums[j] / counts[j])                        # R-cb-lloyd
    return {"counts": counts, "sums": sums, "sse": sse, "n": n,
            "entropy_bits": entropy_bits(counts), "rms": math.sqrt(sse / n), "centroids": cent}


def lloyd(w, levels, iters: int):
    """Lloyd's algorithm on the normalised values, `iters` steps from `levels` (reading R-cb-lloyd).
    Returns the final fp32 levels and the RMS error before each step and after the last."""
    w32 = as_f32_values(w)
    c1 = absmax_blocks(w32)
    lv = check_levels(levels)
    history = []
    for _ in range(iters):
        st = stats(w32, pack_codes(codes(w32, c1, lv)), c1, lv)
        history.append(st["rms"])
        lv = st["centroids"][:lv.size]
    history.append(stats(w32, pack_codes(codes(w32, c1, lv)), c1, lv)["rms"])
    return lv, history


def study(w, nf4_levels, lloyd_iters: int):
    """The page's comparison on one tensor: entropy and RMS error for symmetric int4, the {-8..7}/8
    grid, NF4 and the Lloyd codebook started from NF4."""
    w32 = as_f32_values(w)
    c1 = absmax_blocks(w32)
    books = {"int4_symmetric": np.arange(-7, 8, dtype=np.float32) / np.float32(7),
             "grid_16": np.arange(-8, 8, dtype=np.float32) / np.float32(8),
             "nf4": check_levels(nf4_levels)}
    books["lloyd"], _ = lloyd(w32, books["nf4"], lloyd_iters)
    out = {}
    for name, lv in books.items():
        st = stats(w32, pack_codes(codes(w32, c1, lv)), c1, lv)
        out[name] = {"levels": lv, "entropy_bits": st["entropy_bits"], "rms": st["rms"]}
    return out


def storage_bytes(n: int) -> dict:
    return {"codes": -(-n // 2), "absmax": 4 * num_blocks(n)}
