"""The C ABI without a GPU: the library loads, exports every declared entry point, builds the same
codebook as the oracle (by an independent method), sizes buffers by the closed forms, and rejects bad
arguments on the host before touching CUDA."""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def q():
    from bit_nf4_quantized_14_b200 import build
    build.build()
    import bit_nf4_quantized_14_b200 as mod
    return mod


def declared_functions():
    text = open(os.path.join(ROOT, "include", "qlora_nf4.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:int|int64_t|const char\*)\s+(qlora_\w+)\s*\(", text, flags=re.M)))


def test_every_declared_symbol_is_exported(q):
    names = declared_functions()
    assert len(names) >= 12
    for n in names:
        assert hasattr(q.lib, n), n


def test_codebook_identical_to_oracle(q):
    lv, th = q.codebook()
    ql, qt = O.nf4_codebook()
    assert np.array_equal(lv.view(np.uint32), ql.view(np.uint32))
    assert np.array_equal(th.view(np.uint32), qt.view(np.uint32))


@pytest.mark.parametrize("n", [1, 2, 63, 64, 65, 16383, 16384, 16385, 1 << 31, 65_000_000_000])
def test_storage_bytes_closed_form(q, n):
    assert q.storage_bytes(n) == O.storage_bytes(n)
    nb, ng = -(-n // 64), -(-n // 16384)
    assert q.quantize_workspace_bytes(n) >= 4 * nb + 8 * ng


def test_workspace_queries_and_shape_rules(q):
    assert q.linear_workspace_bytes(8192, 4096, 4096, 64) > 8192 * 64 * 2
    for bad in [(0, 64, 64, 8), (16, 64, 100, 8), (16, 60, 64, 8)]:
        with pytest.raises(q.QLoRAError) as e:
            q.linear_workspace_bytes(*bad)
        assert e.value.code == -2
    for r in (0, 4, 12, 264):
        with pytest.raises(q.QLoRAError) as e:
            q.linear_workspace_bytes(16, 64, 64, r)
        assert e.value.code == -1


def _nf4(rows, cols, base=0x100000):
    return q_struct(base, rows, cols)


def q_struct(base, rows, cols):
    import bit_nf4_quantized_14_b200 as mod
    return mod._NF4Struct(base, base + 0x10000, base + 0x20000, base + 0x30000, rows, cols)


V = ctypes.c_void_p


def test_quantize_argument_errors_before_any_cuda_call(q):
    L = q.lib
    st = q_struct(0x100000, 4, 64)
    ws = V(0x200000)
    assert L.qlora_nf4_quantize(None, 0, 4, 64, ctypes.byref(st), ws, 1 << 20, None) == -1
    assert L.qlora_nf4_quantize(V(0x300000), 7, 4, 64, ctypes.byref(st), ws, 1 << 20, None) == -1
    assert L.qlora_nf4_quantize(V(0x300000), 0, 0, 64, ctypes.byref(st), ws, 1 << 20, None) == -2
    assert L.qlora_nf4_quantize(V(0x300000), 0, 4, 65, ctypes.byref(st), ws, 1 << 20, None) == -2   # shape mismatch
    assert L.qlora_nf4_quantize(V(0x300008), 0, 4, 64, ctypes.byref(st), ws, 1 << 20, None) == -3
    assert L.qlora_nf4_quantize(V(0x300000), 0, 4, 64, ctypes.byref(st), ws, 8, None) == -4
    assert L.qlora_nf4_quantize(V(0x300000), 0, 4, 64, None, ws, 1 << 20, None) == -1
    bad = q_struct(0x100000, 4, 64)
    bad.scale2 = 0x100004
    assert L.qlora_nf4_quantize(V(0x300000), 0, 4, 64, ctypes.byref(bad), ws, 1 << 20, None) == -3


def test_valid_call_without_a_gpu_reports_cuda_error_not_a_fallback(q):
    import torch
    if torch.cuda.is_available():
        pytest.skip("this box has a GPU")
    st = q_struct(0x100000, 4, 64)
    rc = q.lib.qlora_nf4_quantize(V(0x300000), 0, 4, 64, ctypes.byref(st), V(0x200000), 1 << 20, None)
    assert rc in (-5, -8)
    assert q.lib.qlora_nf4_dequantize(ctypes.byref(st), V(0x300000), 1, None) in (-5, -8)


def test_linear_argument_errors(q):
    L = q.lib
    W = q_struct(0x100000, 64, 128)
    X, A, B, Y, ws = V(0x300000), V(0x310000), V(0x320000), V(0x330000), V(0x400000)
    big = 1 << 30
    f = L.qlora_linear_fwd
    assert f(None, 16, ctypes.byref(W), A, B, 8, 16.0, Y, None, ws, big, None) == -1
    assert f(X, 16, ctypes.byref(W), A, B, 12, 16.0, Y, None, ws, big, None) == -1       # r % 8
    assert f(X, 16, ctypes.byref(W), A, B, 8, float("nan"), Y, None, ws, big, None) == -1
    assert f(X, 0, ctypes.byref(W), A, B, 8, 16.0, Y, None, ws, big, None) == -2
    W2 = q_struct(0x100000, 64, 96)                                                        # K % 64
    assert f(X, 16, ctypes.byref(W2), A, B, 8, 16.0, Y, None, ws, big, None) == -2
    W3 = q_struct(0x100000, 60, 128)                                                       # N % 8
    assert f(X, 16, ctypes.byref(W3), A, B, 8, 16.0, Y, None, ws, big, None) == -2
    assert f(V(0x300002), 16, ctypes.byref(W), A, B, 8, 16.0, Y, None, ws, big, None) == -3
    assert f(X, 16, ctypes.byref(W), A, B, 8, 16.0, Y, None, ws, 16, None) == -4
    b = L.qlora_linear_bwd
    assert b(X, X, 16, ctypes.byref(W), A, B, 8, 16.0, None, None, None, V(0x340000), ws, big, None) == -1
    assert b(X, X, 16, ctypes.byref(W), A, B, 8, 16.0, V(0x350001), None, V(0x360000), V(0x370000), ws, big,
             None) == -3


def test_error_strings(q):
    for c in range(-9, 1):
        assert len(q.lib.qlora_error_string(c)) > 0
    assert q.lib.qlora_error_string(-99) == b"unknown error code"


def test_codebook_calls_reject_bad_codebooks_before_any_cuda_call(q):
    """Unsorted, out-of-range, non-finite, too few or too many levels, and two thresholds closer than
    one bucket (1/15 in w / a) all return QLORA_ERR_CODEBOOK; the oracle rejects the same level lists."""
    from oracle import codebook_study as CS
    L = q.lib
    F = ctypes.c_float
    W, C, A, OUT, WS = V(0x300000), V(0x310000), V(0x320000), V(0x330000), V(0x340000)
    bad = [[0.5], [0.0, 0.0], [0.5, -0.5], [-1.0, 1.5], [-1.0, float("nan")], list(np.linspace(-1, 1, 17))]
    dense = [-1.0, -0.02, 0.0, 0.02, 1.0]            # midpoints -0.01 and 0.01 share a bucket
    for lv in bad + [dense]:
        arr = (F * len(lv))(*lv)
        assert L.qlora_codebook_quantize(W, 0, 4096, arr, len(lv), C, A, None) == -10, lv
        assert L.qlora_codebook_dequantize(C, A, 4096, arr, len(lv), OUT, 1, None) == -10, lv
        assert L.qlora_codebook_stats(W, 0, C, A, 4096, arr, len(lv), OUT, WS, 1 << 20, None) == -10, lv
        if lv is not dense:
            with pytest.raises(ValueError):
                CS.check_levels(lv)
    good = (F * 15)(*(np.arange(-7, 8, dtype=np.float32) / np.float32(7)).tolist())
    assert L.qlora_codebook_quantize(W, 0, 0, good, 15, C, A, None) == -2
    assert L.qlora_codebook_quantize(W, 5, 64, good, 15, C, A, None) == -1
    assert L.qlora_codebook_quantize(V(0x300004), 0, 64, good, 15, C, A, None) == -3
    assert L.qlora_codebook_stats(W, 0, C, A, 64, good, 15, OUT, WS, 0, None) == -4
    assert L.qlora_codebook_stats(W, 0, C, A, 64, good, 15, OUT, None, 1 << 20, None) == -4
    b = ctypes.c_size_t()
    assert L.qlora_codebook_stats_workspace(1 << 30, ctypes.byref(b)) == 0 and b.value >= 33 * 8
    assert L.qlora_codebook_stats_workspace(0, ctypes.byref(b)) == -2


def test_adamw_and_paged_calls_reject_bad_arguments_before_any_cuda_call(q):
    L = q.lib
    P, G, M, Vv = V(0x300000), V(0x310000), V(0x320000), V(0x330000)
    ok = dict(step=1, lr=2e-4, b1=0.9, b2=0.999, eps=1e-8, wd=0.0)

    def call(p=P, n=64, **kw):
        a = dict(ok, **kw)
        return L.qlora_adamw_step(p, G, M, Vv, None, n, a["step"], a["lr"], a["b1"], a["b2"], a["eps"], a["wd"], None)

    assert call(p=None) == -1
    assert call(step=0) == -1
    assert call(lr=float("nan")) == -1 and call(lr=-1.0) == -1 and call(lr=float("inf")) == -1
    assert call(b1=1.0) == -1 and call(b2=-0.1) == -1
    assert call(eps=0.0) == -1 and call(wd=-0.5) == -1
    assert call(n=0) == -2
    assert call(p=V(0x300004)) == -3
    assert L.qlora_paged_alloc(0, ctypes.byref(V())) == -1
    assert L.qlora_paged_alloc(64, None) == -1
    assert L.qlora_paged_prefetch(None, 64, 1, None) == -1
    assert L.qlora_paged_free(None) == 0


def test_codebook_density_rule(q):
    """Any codebook whose thresholds are more than one widened bucket (1/15 + 2^-17 in w / a) apart is
    accepted; two thresholds inside one bucket are rejected. Accepted calls go on to the device check and
    fail there without a GPU (or succeed with one), never with QLORA_ERR_CODEBOOK."""
    from oracle import codebook_study as CS
    import torch
    L = q.lib
    F = ctypes.c_float
    W, C, A = V(0x300000), V(0x310000), V(0x320000)
    rng = np.random.default_rng(7)
    gap = 1 / 15 + 2.0 ** -17
    if torch.cuda.is_available():
        pytest.skip("the accepted calls would run on the device")
    for _ in range(200):
        nl = int(rng.integers(2, 17))
        # levels whose midpoints are at least `gap` apart: spread the levels by more than that
        steps = rng.uniform(gap * 1.01, 2.0 / max(nl - 1, 1), size=nl - 1)
        lv = np.concatenate([[0.0], np.cumsum(steps)])
        lv = lv - lv[-1] / 2
        if np.abs(lv).max() > 1:
            lv = lv / np.abs(lv).max()
        lv = lv.astype(np.float32)
        th = CS.thresholds(lv).astype(np.float64)
        if len(th) > 1 and np.diff(th).min() <= gap:
            continue
        arr = (F * nl)(*lv.tolist())
        assert L.qlora_codebook_quantize(W, 0, 4096, arr, nl, C, A, None) != -10, lv
    rejected = 0
    for centre in np.linspace(-0.9, 0.9, 19):
        # two thresholds 0.01 apart around the centre b of a bucket (buckets are 1/15 wide): levels
        # l0 = m0 - d, l1 = m0 + d, l2 = 2 m1 - l1 have midpoints m0 and m1
        b = round(centre * 15) / 15
        m0, m1, d = b - 0.005, b + 0.005, 0.004
        lv = np.array([m0 - d, m0 + d, 2 * m1 - (m0 + d)], np.float32)
        assert np.all(np.diff(lv) > 0) and np.abs(lv).max() <= 1
        arr = (F * 3)(*lv.tolist())
        assert L.qlora_codebook_quantize(W, 0, 4096, arr, 3, C, A, None) == -10, lv
        rejected += 1
    assert rejected == 19


def test_fault_injection_fails_the_chosen_call_on_the_host():
    """QLORA_FAULT_INJECT=<entry>:<k> fails exactly the k-th call of that entry point, after its argument
    checks (a call with a bad argument is not counted) and before any CUDA call; QLORA_DEBUG reports it.
    Run in a child process so the variables apply from the library's first call."""
    import subprocess
    import sys
    code = r"""
import ctypes, sys
sys.path.insert(0, ROOT)
import bit_nf4_quantized_14_b200 as q
L = q.lib
st = q._NF4Struct(0x100000, 0x110000, 0x120000, 0x130000, 4, 64)
V = ctypes.c_void_p
call = lambda w: L.qlora_nf4_quantize(V(w), 0, 4, 64, ctypes.byref(st), V(0x200000), 1 << 20, None)
print("RC", call(0x300008), call(0x300000), call(0x300000), call(0x300000), flush=True)
print("WL", L.qlora_set_wait_limit(10), L.qlora_set_wait_limit(1 << 40), L.qlora_selftest_wait(9, None), flush=True)
"""
    env = dict(os.environ, QLORA_FAULT_INJECT="qlora_nf4_quantize:2", QLORA_DEBUG="1", CUDA_VISIBLE_DEVICES="")
    r = subprocess.run([sys.executable, "-c", f"ROOT = {ROOT!r}\n" + code], capture_output=True, text=True,
                       env=env, timeout=300)
    assert r.returncode == 0, r.stderr
    rc = [int(v) for v in next(l for l in r.stdout.splitlines() if l.startswith("RC")).split()[1:]]
    assert rc[0] == -3                       # misaligned: rejected before the injection point, not counted
    assert rc[1] in (-5, -8) and rc[3] in (-5, -8)   # no GPU in the child: the device check fails
    assert rc[2] == -5
    injected = [l for l in r.stderr.splitlines() if "injected launch failure" in l]
    assert injected == ["qlora: injected launch failure in qlora_nf4_quantize (call 2)"]
    wl = [int(v) for v in next(l for l in r.stdout.splitlines() if l.startswith("WL")).split()[1:]]
    assert wl == [-1, -1, -1]
