"""The no-allocation quantize entry point against the regular one.

qlora_nf4_quantize_noalloc serves callers that cannot allocate device memory at the point of the call
(a framework's caching allocator that must not be bypassed, plugin interfaces that pass only inputs and
outputs, loops that forbid allocation after start-up). It keeps its intermediates in a fixed scratch
array inside the library instead of a caller workspace. Its results must equal qlora_nf4_quantize's
exactly (the codec's tolerance is bit-exactness), on consecutive calls that reuse the shared scratch.
This file is collected last so that a stopping run has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu


def _noalloc(lib, w, out):
    rows, cols = (w.shape[0], w.shape[1]) if w.dim() == 2 else (1, w.numel())
    st = out.struct()
    rc = lib.load().qlora_nf4_quantize_noalloc(ctypes.c_void_p(w.data_ptr()),
                                               0 if w.dtype == torch.float32 else 1, rows, cols,
                                               ctypes.byref(st), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return rc


def _same(a, b):
    for f in ("codes", "absmax_e4m3", "scale2", "offset"):
        x, y = getattr(a, f), getattr(b, f)
        assert torch.equal(x, y), f


def test_noalloc_matches_workspace_entry_point_on_consecutive_calls(lib):
    # two calls in a row on different inputs (the second overwrites the first's scratch contents),
    # then the first input again: each must equal the workspace entry point's result exactly
    cases = [synth.weight_f32(4096, 4096, seed=0, tensor_id=61),
             synth.sweep_f32(3 * 16384 * 7 + 129, seed=0, tensor_id=62).reshape(1, -1)]
    cases.append(cases[0])
    for i, W in enumerate(cases):
        w = torch.from_numpy(W).cuda()
        ref = lib.quantize(w)
        got = lib.NF4Weight.empty(w.shape[0], w.shape[1], w.device)
        assert _noalloc(lib, w, got) == 0, f"call {i}"
        assert lib.get_status() == 0
        _same(got, ref)
    wb = synth.to_bf16(cases[1]).cuda()
    got = lib.NF4Weight.empty(wb.shape[0], wb.shape[1], wb.device)
    assert _noalloc(lib, wb, got) == 0
    _same(got, lib.quantize(wb))


def test_noalloc_back_to_back_on_one_stream(lib):
    """Stream order is what makes the shared scratch safe: two calls enqueued one after the other on one
    non-default stream, with no synchronization between them, each equal the workspace entry point's
    result bit for bit."""
    W1 = torch.from_numpy(synth.weight_f32(2048, 3072, seed=0, tensor_id=64)).cuda()
    W2 = torch.from_numpy(synth.sweep_f32(5 * 16384 + 4097, seed=0, tensor_id=65).reshape(1, -1)).cuda()
    refs = [lib.quantize(W1), lib.quantize(W2)]
    torch.cuda.synchronize()
    side = torch.cuda.Stream()
    outs = [lib.NF4Weight.empty(w.shape[0], w.shape[1], w.device) for w in (W1, W2)]
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        for w, o in zip((W1, W2), outs):
            assert _noalloc(lib, w, o) == 0
    side.synchronize()
    assert lib.get_status(side) == 0
    for o, ref in zip(outs, refs):
        _same(o, ref)


def test_noalloc_rejects_inputs_beyond_its_scratch(lib):
    n = lib.NOALLOC_MAX_NUMEL
    fake = lib.NF4Weight.empty(1, 64, "cuda")
    st = lib._NF4Struct(fake.codes.data_ptr(), fake.absmax_e4m3.data_ptr(), fake.scale2.data_ptr(),
                        fake.offset.data_ptr(), 2, n // 2 + 64)
    w = torch.zeros(64, device="cuda")
    rc = lib.load().qlora_nf4_quantize_noalloc(ctypes.c_void_p(w.data_ptr()), 0, 2, n // 2 + 64,
                                               ctypes.byref(st), None)
    assert rc == -9
    assert b"scratch" in lib.load().qlora_error_string(rc)
    # exactly at the limit is accepted
    W = torch.from_numpy(synth.sweep_f32(n, seed=0, tensor_id=63)).cuda().reshape(1, n)
    got = lib.NF4Weight.empty(1, n, W.device)
    assert _noalloc(lib, W, got) == 0
    _same(got, lib.quantize(W))
