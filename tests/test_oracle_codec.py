"""Pins for the oracle's codec: brute-force nearest-level checks in exact arithmetic, hand-built
packing and summation cases, the double-quantization error bound, the pages' storage figures and the
pages' codebook statistics."""
import json
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle as O
import synth

GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "page_figures.json")))
S = 320   # every value below is a multiple of 2^-S, so x * 2^S is an exact integer


def _int(x) -> int:
    n, d = float(x).as_integer_ratio()
    assert (1 << S) % d == 0
    return n * ((1 << S) // d)


def _check_rule(w32: np.ndarray, a: np.float32):
    """Code of every w (|w| <= a) against exact nearest-level search, and against the threshold rule
    where the rounded threshold and the true midpoint disagree."""
    q, T = O.nf4_codebook()
    codes = O.nf4_codes(w32, np.full(-(-w32.size // 64), a, np.float32), T)
    A = _int(a)
    Q = [_int(v) for v in q]
    TT = [_int(v) for v in T]
    for i, w in enumerate(w32.tolist()):
        W = _int(w) << S                                  # w * 2^(2S)
        P = [qj * A for qj in Q]                          # q_j * a * 2^(2S), exact
        dist = [abs(W - p) for p in P]
        nearest = dist.index(min(dist))                   # first minimum: ties to the lower index
        by_mid = [2 * W > P[j] + P[j + 1] for j in range(15)]
        by_thr = [W > TT[j] * A for j in range(15)]
        if by_mid == by_thr:
            assert codes[i] == nearest, (w, a, codes[i], nearest)
            assert nearest == sum(by_mid)
        else:
            assert codes[i] == sum(by_thr), (w, a)


def _bf16_patterns_upto(a: float) -> np.ndarray:
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    v = O.bf16_bits_to_f32(bits)
    keep = np.isfinite(v) & (np.abs(v) <= a)
    return v[keep]


@pytest.mark.parametrize("a", [1.0, 0.02, 3.7e-3, 2.0 ** -100, 448.0, 1e-40, 3e38])
def test_codes_exhaustive_bf16_against_exact_nearest(a):
    a = np.float32(a)
    w = _bf16_patterns_upto(float(a))
    _check_rule(w, a)


def test_codes_fp32_near_thresholds_against_exact_nearest():
    rng = np.random.default_rng(5)
    q, T = O.nf4_codebook()
    for a in [np.float32(1.0), np.float32(0.0173), np.float32(2.3e-30), np.float32(5.5e5)]:
        base = (T.astype(np.float64) * float(a)).astype(np.float32)
        near = [np.nextafter(base, np.float32(np.inf)), base, np.nextafter(base, np.float32(-np.inf))]
        w = np.concatenate(near + [(rng.uniform(-1, 1, 300) * float(a)).astype(np.float32)])
        w = w[np.abs(w) <= a]
        _check_rule(w, a)


def test_exact_ties_go_to_lower_index_and_special_cases():
    q, T = O.nf4_codebook()
    one = np.ones(1, np.float32)
    assert list(O.nf4_codes(T, one, T)) == list(range(15))          # w = T_j * 1 exactly -> j
    assert list(O.nf4_codes(q, one, T)) == list(range(16))          # each level codes to itself
    assert list(O.nf4_codes(np.float32([-0.0, 0.0]), one, T)) == [7, 7]
    assert list(O.nf4_codes(np.zeros(64, np.float32), np.zeros(1, np.float32), T)) == [7] * 64
    w = synth.normal_f32(64, 1.0, 0, 9)
    c1 = O.absmax_blocks(w)
    codes = O.nf4_codes(w, c1, T)
    assert codes[np.argmax(w)] == 15 or codes[np.argmin(w)] == 0    # the absmax element hits an end
    assert codes[np.argmax(np.abs(w))] in (0, 15)


def test_nonfinite_input_is_rejected():
    w = np.zeros(130, np.float32)
    for bad in (np.inf, -np.inf, np.nan):
        w[70] = bad
        with pytest.raises(ValueError):
            O.absmax_blocks(w)


def test_partial_last_block_absmax():
    w = np.float32([1, -2, 3] + [0.5] * 61 + [-7.0, 0.25])      # 66 elements: blocks of 64 and 2
    assert list(O.absmax_blocks(w)) == [3.0, 7.0]
    assert O.num_blocks(66) == 2 and O.num_groups(66) == 1


def test_packing_hand_built():
    assert list(O.pack_codes(np.uint8([0x3, 0xA]))) == [0x3A]
    assert list(O.pack_codes(np.uint8([0x3, 0xA, 0xF]))) == [0x3A, 0xF0]
    assert list(O.unpack_codes(np.uint8([0x3A, 0xF0]), 3)) == [0x3, 0xA, 0xF]
    rng = np.random.default_rng(6)
    c = rng.integers(0, 16, 1001).astype(np.uint8)
    assert np.array_equal(O.unpack_codes(O.pack_codes(c), c.size), c)


def test_pairwise_tree_order_hand_computed():
    e = 2.0 ** -53
    # ((1 + e) + (0 + e)) : 1 + e rounds to 1 (tie to even), then 1 + e rounds to 1 again
    assert O.pairwise_tree_sum([1.0, e, 0.0, e]) == 1.0
    # ((1 + 0) + (e + e)) = 1 + 2e exactly
    assert O.pairwise_tree_sum([1.0, 0.0, e, e]) == 1.0 + 2 * e
    c1 = np.zeros(300, np.float32)
    c1[:4] = [1.0, e, 0.0, e]
    # 300 constants pad to 512 leaves; the first four form the leftmost subtree as above
    assert O.block_mean(c1) == np.float32(1.0 / 300)


def test_block_mean_equal_constants_and_exact_sum():
    for nb in (1, 3, 255, 256, 257, 1000, 4099):
        v = np.float32(0.0173)
        assert O.block_mean(np.full(nb, v, np.float32)) == v
    rng = np.random.default_rng(7)
    c1 = np.abs(rng.normal(0, 0.05, 100_000)).astype(np.float32)
    mu = O.block_mean(c1)
    exact = sum(Fraction(float(x)) for x in c1) / len(c1)
    assert abs(Fraction(float(mu)) - exact) <= Fraction(float(np.spacing(mu)))


def test_double_quantization_error_bound_and_full_range():
    w = synth.sweep_f32(64 * 256 * 5 + 300, seed=0, tensor_id=12)
    c1 = O.absmax_blocks(w)
    e, s2, mu = O.double_quantize(c1)
    chat = O.double_dequantize(e, s2, mu).astype(np.float64)
    nb = c1.size
    g = np.arange(nb) // 256
    d = O.rn32_sub(c1, mu).astype(np.float64)
    t = d / s2[g]
    dec = O.e4m3_decode(e)
    # half an E4M3 step at |t| (subnormal step 2^-9 below 2^-6), plus the fp32 roundings
    step = np.where(np.abs(dec) < 2 ** -6, 2.0 ** -9, np.exp2(np.floor(np.log2(np.maximum(np.abs(dec), 2 ** -6))) - 3))
    step = np.maximum(step, np.where(np.abs(t) >= 2 ** -6, np.exp2(np.floor(np.log2(np.abs(t) + 1e-300)) - 3), 2.0 ** -9))
    bound = s2[g] * (step / 2 + np.spacing(np.abs(t).astype(np.float32))) + np.spacing(np.abs(d).astype(np.float32)) \
        + np.spacing(np.abs(chat).astype(np.float32))
    assert np.all(np.abs(chat - c1) <= bound)
    for gi in range(s2.size):        # each group's largest |d| maps to the E4M3 end point 448
        sl = slice(256 * gi, min(nb, 256 * gi + 256))
        assert np.max(np.abs(dec[sl])) == 448.0


def test_storage_overhead_matches_page_figures():
    n = 64 * 256 * 1000
    sb = O.storage_bytes(n)
    bits_total = 8.0 * sum(sb.values()) / n
    overhead = 8.0 * (sb["absmax"] + sb["scale2"]) / n
    assert overhead == pytest.approx(8 / 64 + 32 / (64 * 256), abs=1e-6)
    assert round(overhead, 3) == GOLDEN["overhead_bits_after_dq"]["value"]
    assert round(GOLDEN["overhead_bits_before_dq"]["value"] - overhead, 3) == GOLDEN["overhead_saving_bits"]["value"]
    assert round(bits_total, 3) == GOLDEN["bits_per_weight_total"]["value"]
    assert round(bits_total / 8, 3) == GOLDEN["bytes_per_weight_total"]["value"]
    p65 = GOLDEN["base_65b_gb"]["params"]
    assert round(p65 * (4 + overhead) / 8 / 1e9, 1) == GOLDEN["base_65b_gb"]["value"]
    assert round(p65 * (0.5 - overhead) / 8 / 1e9) == GOLDEN["saving_65b_gb"]["value"]


def test_dequant_special_cases():
    w = np.zeros(200, np.float32)
    w[64:128] = synth.normal_f32(64, 0.02, 0, 13)
    t = O.quantize(w)
    wd = O.dequantize(t, "f32")
    assert np.all(wd[:64] == 0) and np.all(wd[128:] == 0)           # all-zero blocks stay exactly zero
    codes = O.unpack_codes(t.codes, t.n)
    assert np.all(codes[:64] == 7) and np.all(codes[128:] == 7)
    bits = O.dequantize(t, "bf16")
    assert np.array_equal(bits, O.bf16_rne_bits(wd))


def test_quantization_error_without_double_quant_is_bounded():
    """Without the second level (fp32 c1) every weight lies within half the widest level gap of its
    level, times its block's absmax."""
    q, T = O.nf4_codebook()
    w = synth.weight_f32(128, 256, seed=0, tensor_id=14)
    c1 = O.absmax_blocks(w)
    codes = O.nf4_codes(w.reshape(-1), c1, T)
    rec = q[codes].astype(np.float64) * np.repeat(c1, 64)
    gap = np.max(np.diff(q.astype(np.float64))) / 2
    assert np.all(np.abs(rec - w.reshape(-1)) <= np.repeat(c1, 64) * gap * (1 + 1e-6))


def test_codebook_statistics_match_the_page():
    """Large Gaussian matrix, blocks of 64, fp32 constants: entropy 3.88 vs 3.50 bits, RMS error about
    15 % below symmetric int4, and an MSE-optimal (Lloyd) codebook about 5 % better than NF4."""
    x = synth.normal_f32((2048, 2048), 1.0, 0, 15).reshape(-1)
    c1 = O.absmax_blocks(x)
    a = np.repeat(c1.astype(np.float64), 64)

    def run(levels):
        lv = np.asarray(levels, np.float32)
        Tm = ((lv[:-1].astype(np.float64) + lv[1:]) / 2).astype(np.float32)
        codes = O.nf4_codes(x, c1, Tm)
        h = np.bincount(codes, minlength=lv.size) / codes.size
        ent = float(-(h[h > 0] * np.log2(h[h > 0])).sum())
        rms = float(np.sqrt(np.mean((lv[codes].astype(np.float64) * a - x) ** 2)))
        return ent, rms

    q, _ = O.nf4_codebook()
    ent_nf4, rms_nf4 = run(q)
    ent_i4, rms_i4 = run(np.arange(-7, 8) / 7.0)
    _, rms_i8 = run(np.arange(-8, 8) / 8.0)
    assert abs(ent_nf4 - GOLDEN["entropy_bits_nf4"]["value"]) < 0.02
    assert abs(ent_i4 - GOLDEN["entropy_bits_int4_symmetric"]["value"]) < 0.02
    assert abs((1 - rms_nf4 / rms_i4) - GOLDEN["rms_reduction_nf4_vs_int4"]["value"]) < 0.03
    assert rms_nf4 < rms_i8 < rms_i4
    # Lloyd (1-D k-means) on the normalised values, started from NF4
    u = (x.astype(np.float64) / a)[::4]
    lv = q.astype(np.float64)
    for _ in range(60):
        mid = (lv[:-1] + lv[1:]) / 2
        idx = np.searchsorted(mid, u)
        lv = np.array([u[idx == j].mean() if np.any(idx == j) else lv[j] for j in range(16)])
    _, rms_lloyd = run(lv)
    gain = 1 - rms_lloyd / rms_nf4
    assert abs(gain - GOLDEN["lloyd_gain_over_nf4"]["value"]) < 0.03, gain


# ---- the variant without double quantization ---------------------------------------------------

def test_single_variant_overhead_is_half_a_bit_per_weight():
    """PEFT page, 'Double quantization': fp32 constants per block of 64 cost 32/64 = 0.5 bits/param."""
    n = 64 * 4096
    sb = O.storage_bytes_single(n)
    assert 8.0 * sb["absmax"] / n == GOLDEN["overhead_bits_before_dq"]["value"]
    assert sb["codes"] == n // 2


def test_single_variant_shares_codes_and_dequantizes_by_definition():
    x = synth.sweep_f32(64 * 300 + 17, seed=5, tensor_id=12)
    s = O.quantize_single(x)
    d = O.quantize(x)
    assert np.array_equal(s.codes, d.codes)                        # the first level is unchanged
    assert np.array_equal(s.absmax.view(np.uint32), O.absmax_blocks(x).view(np.uint32))
    q, _ = O.nf4_codebook()
    codes = O.unpack_codes(s.codes, s.n)
    want = (q[codes].astype(np.float64) * np.repeat(s.absmax, 64)[:s.n].astype(np.float64)).astype(np.float32)
    assert np.array_equal(O.dequantize_single(s, "f32").view(np.uint32), want.view(np.uint32))


def test_single_and_double_agree_when_the_second_level_is_exact():
    """All block constants equal: s2 = 0 and c1_hat = mu = c1 exactly, so both variants dequantize alike."""
    rng = np.random.default_rng(3)
    x = (rng.standard_normal(64 * 512) * 0.01).astype(np.float32)
    x.reshape(-1, 64)[:, 0] = np.float32(0.25)                       # every block's absmax is 0.25
    s, d = O.quantize_single(x), O.quantize(x)
    assert np.all(d.scale2 == 0)
    assert np.array_equal(O.dequantize_single(s, "bf16"), O.dequantize(d, "bf16"))


def test_single_variant_error_bound():
    """|w - w_hat| <= a * max_j (T_j - q_j) + fp32 rounding, per block (nearest-level quantization)."""
    x = synth.sweep_f32(64 * 2000, seed=6, tensor_id=13)
    s = O.quantize_single(x)
    q, T = O.nf4_codebook()
    half_gap = float(np.max(np.maximum(T - q[:-1], q[1:] - T)))
    a = np.repeat(s.absmax, 64)[:s.n].astype(np.float64)
    err = np.abs(O.dequantize_single(s, "f32").astype(np.float64) - x.astype(np.float64))
    assert np.all(err <= a * half_gap * (1 + 1e-6) + 1e-30)
