"""GPU parity of the NF4 codec against the oracle: codes, E4M3 constants, second-level scales, the mean
and dequantized values must be bit-identical on the same seeded inputs."""
import numpy as np
import pytest
import torch

import oracle as O
import synth

pytestmark = pytest.mark.gpu


def run_quantize(lib, w_np=None, w_t=None):
    w = w_t if w_t is not None else torch.from_numpy(w_np).cuda()
    q = lib.quantize(w)
    st = lib.get_status()
    return q, st


def assert_same_as_oracle(q, ref):
    n = ref.n
    assert np.array_equal(q.codes.cpu().numpy(), ref.codes), "codes"
    assert np.array_equal(q.absmax_e4m3.cpu().numpy(), ref.absmax_e4m3), "E4M3 constants"
    assert np.array_equal(q.scale2.cpu().numpy().view(np.uint32), ref.scale2.view(np.uint32)), "scale2"
    assert q.offset.cpu().numpy().view(np.uint32)[0] == np.float32(ref.offset).view(np.uint32), "mean"
    assert q.codes.numel() == -(-n // 2)


def assert_dequant_same(lib, q, ref, shape):
    got16 = lib.dequantize(q, torch.bfloat16).cpu().view(torch.int16).numpy().view(np.uint16).reshape(-1)
    assert np.array_equal(got16, O.dequantize(ref, "bf16").reshape(-1)), "bf16 dequant"
    got32 = lib.dequantize(q, torch.float32).cpu().numpy().reshape(-1)
    assert np.array_equal(got32.view(np.uint32), O.dequantize(ref, "f32").reshape(-1).view(np.uint32)), "fp32 dequant"


def test_tiny_config_fp32(lib):
    W = synth.weight_f32(256, 256, sigma=0.02, outlier_p=0.0, seed=0, tensor_id=1)
    q, st = run_quantize(lib, W)
    assert st == 0
    ref = O.quantize(W)
    assert_same_as_oracle(q, ref)
    assert_dequant_same(lib, q, ref, W.shape)


@pytest.mark.parametrize("n", [1, 2, 3, 63, 64, 65, 255, 257, 4097, 16383, 16384, 16385,
                               3 * 16384 + 77, 100_003, 64 * 256 * 37 + 5])
def test_ragged_sizes_fp32_and_bf16(lib, n):
    x = synth.sweep_f32(n, seed=1, tensor_id=n % 1000)
    q, st = run_quantize(lib, x.reshape(1, n))
    assert st == 0
    ref = O.quantize(x)
    assert_same_as_oracle(q, ref)
    assert_dequant_same(lib, q, ref, (1, n))
    xb = synth.to_bf16(x)
    qb, st = run_quantize(lib, w_t=xb.reshape(1, n).cuda())
    refb = O.quantize(synth.bf16_bits(xb))
    assert st == 0
    assert_same_as_oracle(qb, refb)
    qw, _ = run_quantize(lib, w_t=xb.float().reshape(1, n).cuda())   # bf16 input == its fp32 widening
    assert torch.equal(qw.codes, qb.codes) and torch.equal(qw.absmax_e4m3, qb.absmax_e4m3)
    assert torch.equal(qw.scale2, qb.scale2) and torch.equal(qw.offset, qb.offset)


def test_many_groups_mean_tree(lib):
    """ng = 1500 groups: the mean's fp64 tree spans several levels of the reduction kernel."""
    n = 16384 * 1500 - 333
    x = synth.sweep_f32(n, seed=2, tensor_id=5)
    q, st = run_quantize(lib, x)
    assert st == 0
    ref = O.quantize(x)
    assert_same_as_oracle(q, ref)


def test_special_values(lib):
    q_, T = O.nf4_codebook()
    parts = [np.zeros(64 * 3, np.float32),                                  # all-zero blocks
             np.full(64 * 256, 0.0173, np.float32),                         # equal constants: s2 = 0 group
             (T.astype(np.float64) * 1.0).astype(np.float32),               # exact ties at a = 1
             np.float32([1.0] + [-1.0] * 63),
             np.float32([1e-40, -3e-39, 2e-45] + [0.0] * 61),               # subnormal block
             np.float32([3e38, -1e38] + [1e30] * 62),                       # huge block
             np.float32([-0.0] * 64),
             synth.normal_f32(64 * 300 + 17, 0.02, 0, 31)]
    x = np.concatenate(parts).astype(np.float32)
    q, st = run_quantize(lib, x)
    assert st == 0
    ref = O.quantize(x)
    assert_same_as_oracle(q, ref)
    assert_dequant_same(lib, q, ref, x.shape)


def test_constant_tensor_gives_zero_second_level_scale(lib):
    x = np.full(64 * 512, -0.5, np.float32)
    q, _ = run_quantize(lib, x)
    ref = O.quantize(x)
    assert_same_as_oracle(q, ref)
    assert np.all(ref.scale2 == 0) and np.all(ref.absmax_e4m3 == 0)
    assert_dequant_same(lib, q, ref, x.shape)


@pytest.mark.parametrize("bad", [np.nan, np.inf, -np.inf])
def test_nonfinite_input_sets_status(lib, bad):
    x = synth.normal_f32(64 * 40, 0.02, 0, 41)
    x[1000] = bad
    lib.quantize(torch.from_numpy(x).cuda())
    assert lib.get_status() & lib.STATUS_NONFINITE
    assert lib.get_status() == 0          # reading clears it


def test_full_size_7b_weight(lib):
    """The 11008 x 4096 LLaMA-7B-shaped weight (N(0, 0.02^2) with 0.1 % x10 outliers), fp32 input."""
    W = synth.weight_f32(11008, 4096, seed=0, tensor_id=1)
    q, st = run_quantize(lib, W)
    assert st == 0
    ref = O.quantize(W)
    assert_same_as_oracle(q, ref)
    got = lib.dequantize(q, torch.bfloat16).cpu().view(torch.int16).numpy().view(np.uint16).reshape(-1)
    assert np.array_equal(got, O.dequantize(ref, "bf16").reshape(-1))


def test_sweep_size_sampled(lib):
    """A 2^26-element sweep tensor: exact on every per-block quantity; dequant checked on a sample."""
    n = 1 << 26
    x = synth.sweep_f32(n, seed=0, tensor_id=3)
    q, st = run_quantize(lib, x)
    assert st == 0
    ref = O.quantize(x)
    assert_same_as_oracle(q, ref)
    deq = lib.dequantize(q, torch.bfloat16).view(-1)
    idx = torch.from_numpy(np.random.default_rng(0).integers(0, n, 200_000)).cuda()
    got = deq[idx].cpu().view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, O.dequantize(ref, "bf16").reshape(-1)[idx.cpu().numpy()])


def test_deterministic(lib):
    x = synth.sweep_f32(1_000_003, seed=4, tensor_id=9)
    a = lib.quantize(torch.from_numpy(x).cuda())
    b = lib.quantize(torch.from_numpy(x).cuda())
    for f in ("codes", "absmax_e4m3", "scale2", "offset"):
        assert torch.equal(getattr(a, f), getattr(b, f))


def _rd_f32(p):
    """fp32 rounding toward -inf of the exactly representable fp64 values p."""
    f = p.astype(np.float32)
    down = f.astype(np.float64) > p
    f[down] = np.nextafter(f[down], np.float32(-np.inf))
    return f


ABSMAX = [1.0, 0.02, 3.7e-3, 0.5, 448.0, 2.0 ** -100, 2.0 ** -126, 1e-39, 3e38]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_codes_over_every_bf16_value(lib, dtype):
    """For absmax values a from subnormal to near the fp32 maximum, every finite bf16 value w with
    |w| <= a, in blocks led by +a or -a (so a is the block absmax): codes, constants and the dequantized
    values equal the oracle's exact threshold rule. With fp32 input, also the 7 fp32 values around each
    decision point RD(T_j a) for every threshold j. Covers every bucket of the table-assisted code search,
    the scaled path for absmax below 2^-120, and reciprocals that are subnormal (a near 3e38)."""
    _, T = O.nf4_codebook()
    allv = (np.arange(65536, dtype=np.uint32) << 16).view(np.float32)
    allv = allv[np.isfinite(allv)]
    blocks = []
    for a0 in ABSMAX:
        a = np.float32(a0)
        if dtype == "bf16":
            a = synth.bf16_values(synth.to_bf16(np.array([a], np.float32)))[0]
        vals = allv[np.abs(allv) <= a]
        if dtype == "f32":
            P = _rd_f32(T.astype(np.float64) * np.float64(a))
            near = [P]
            up, dn = P.copy(), P.copy()
            for _ in range(3):
                up = np.nextafter(up, np.float32(np.inf))
                dn = np.nextafter(dn, np.float32(-np.inf))
                near += [up.copy(), dn.copy()]
            near = np.concatenate(near)
            vals = np.concatenate([vals, near[np.abs(near) <= a]])
        for sign in (1.0, -1.0):
            pad = (-len(vals)) % 63
            body = np.concatenate([vals, np.zeros(pad, np.float32)]).reshape(-1, 63)
            lead = np.full((body.shape[0], 1), np.float32(sign) * a, np.float32)
            blocks.append(np.concatenate([lead, body], axis=1).reshape(-1))
    x = np.concatenate(blocks).astype(np.float32)
    if dtype == "f32":
        q, st = run_quantize(lib, x)
        ref = O.quantize(x)
    else:
        xb = synth.to_bf16(x)
        assert np.array_equal(synth.bf16_values(xb), x)          # every value is bf16-exact
        q, st = run_quantize(lib, w_t=xb.cuda())
        ref = O.quantize(synth.bf16_bits(xb))
    assert st == 0
    assert_same_as_oracle(q, ref)
    assert_dequant_same(lib, q, ref, x.shape)


# ---- the variant without double quantization --------------------------------------------------

def _assert_single_same(lib, x_dev, ref, n):
    qs = lib.quantize_single(x_dev)
    assert lib.get_status() == 0
    assert np.array_equal(qs.codes.cpu().numpy(), ref.codes), "codes"
    assert np.array_equal(qs.absmax.cpu().numpy().view(np.uint32), ref.absmax.view(np.uint32)), "fp32 constants"
    got16 = lib.dequantize_single(qs, torch.bfloat16).cpu().view(torch.int16).numpy().view(np.uint16).reshape(-1)
    assert np.array_equal(got16, O.dequantize_single(ref, "bf16").reshape(-1)), "bf16 dequant"
    got32 = lib.dequantize_single(qs, torch.float32).cpu().numpy().reshape(-1)
    assert np.array_equal(got32.view(np.uint32), O.dequantize_single(ref, "f32").reshape(-1).view(np.uint32))
    return qs


@pytest.mark.parametrize("n", [1, 63, 65, 4097, 16383, 16385, 3 * 16384 + 77, 64 * 256 * 37 + 5])
def test_single_variant_ragged_sizes(lib, n):
    x = synth.sweep_f32(n, seed=7, tensor_id=n % 997)
    _assert_single_same(lib, torch.from_numpy(x.reshape(1, n)).cuda(), O.quantize_single(x), n)
    xb = synth.to_bf16(x)
    _assert_single_same(lib, xb.reshape(1, n).cuda(), O.quantize_single(synth.bf16_bits(xb)), n)


def test_single_variant_codes_match_the_double_quantized_path(lib):
    W = synth.weight_f32(1024, 4096, seed=3, tensor_id=2)
    d = lib.quantize(torch.from_numpy(W).cuda())
    s = _assert_single_same(lib, torch.from_numpy(W).cuda(), O.quantize_single(W), W.size)
    assert torch.equal(d.codes, s.codes)


def test_single_variant_special_values(lib):
    x = np.concatenate([np.zeros(128, np.float32), np.float32([1e-40, -3e-39] + [0.0] * 62),
                        np.float32([3e38, -1e38] + [1e30] * 62), synth.normal_f32(64 * 50 + 3, 0.02, 0, 77)])
    _assert_single_same(lib, torch.from_numpy(x).cuda(), O.quantize_single(x), x.size)


def test_largest_sweep_size_2_31(lib):
    """The top of the quantize/dequantize size sweep, 2^31 elements (eight 2^28-element sweep tensors,
    drawn as the benchmark draws them; indices past 2^31 - 1 exercise 64-bit addressing): every block
    constant's E4M3 value, every group scale and the mean exact against the oracle, and the codes and
    dequantized bf16 values of 4096 sampled blocks."""
    n, chunk = 1 << 31, 1 << 28
    dev = torch.device("cuda", 0)
    x = torch.empty(n, dtype=torch.float32, device=dev)
    c1 = np.empty(n // 64, np.float32)
    sb = np.sort(np.random.default_rng(1).choice(n // 64, 4096, replace=False))
    sv = np.empty((sb.size, 64), np.float32)
    for c in range(0, n, chunk):
        xc = synth.sweep_f32(chunk, seed=50, tensor_id=c // chunk)
        x[c:c + chunk] = torch.from_numpy(xc).to(dev)
        c1[c // 64:(c + chunk) // 64] = O.absmax_blocks(xc)
        for i in np.nonzero((sb >= c // 64) & (sb < (c + chunk) // 64))[0]:
            off = int(sb[i]) * 64 - c
            sv[i] = xc[off:off + 64]
        del xc
    q = lib.quantize(x)
    assert lib.get_status() == 0
    e, s2, mu = O.double_quantize(c1)
    assert q.offset.cpu().numpy().view(np.uint32)[0] == np.float32(mu).view(np.uint32), "mean"
    assert np.array_equal(q.scale2.cpu().numpy().view(np.uint32), s2.view(np.uint32)), "group scales"
    assert np.array_equal(q.absmax_e4m3.cpu().numpy(), e), "E4M3 constants"
    levels, T = O.nf4_codebook()
    ref_codes = O.nf4_codes(sv.reshape(-1), c1[sb], T).reshape(sb.size, 64)
    byte_idx = torch.from_numpy((sb[:, None] * 32 + np.arange(32)[None, :]).reshape(-1)).to(dev)
    got = q.codes[byte_idx].cpu().numpy().reshape(sb.size, 32)
    assert np.array_equal(got, O.pack_codes(ref_codes.reshape(-1)).reshape(sb.size, 32)), "codes"
    del x
    deq = lib.dequantize(q, torch.bfloat16).view(-1)
    elem_idx = torch.from_numpy((sb[:, None] * 64 + np.arange(64)[None, :]).reshape(-1)).to(dev)
    got16 = deq[elem_idx].cpu().view(torch.int16).numpy().view(np.uint16).reshape(sb.size, 64)
    chat = O.fma32(O.e4m3_decode(e[sb]).astype(np.float32), s2[sb // 256], np.float32(mu))
    ref16 = O.bf16_rne_bits(O.rn32_mul(levels[ref_codes], np.repeat(chat, 64).reshape(sb.size, 64)))
    assert np.array_equal(got16, ref16), "dequantized bf16"
