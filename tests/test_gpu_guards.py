"""Bounds evidence without a sanitizer: every output buffer of the codec and of the linear layer sits
between guard regions filled with a canary byte, and after each call the guards must be untouched. The
sizes are ragged (odd element counts, partial blocks and groups, token, row and rank tails of every
tile shape), so a kernel that writes one element, one vector or one tile past its end is caught here.
The outputs themselves are also compared with the oracle (codec bit for bit, linear within 5e-3)."""
import numpy as np
import pytest
import torch

import oracle as O
import synth

pytestmark = pytest.mark.gpu
CANARY = 0xA5
GUARD = 4096          # bytes before and after each output; a multiple of 256 keeps every view aligned
TOL = 5e-3


class Guarded:
    """A device buffer of `numel` elements of `dtype` with GUARD canary bytes on both sides."""

    def __init__(self, numel, dtype, device="cuda"):
        esz = torch.empty(0, dtype=dtype).element_size()
        self.nbytes = numel * esz
        body = (self.nbytes + 255) // 256 * 256
        self.raw = torch.full((GUARD + body + GUARD,), CANARY, dtype=torch.uint8, device=device)
        self.tail = GUARD + self.nbytes
        self.t = self.raw[GUARD:GUARD + self.nbytes].view(dtype) if numel else self.raw[GUARD:GUARD].view(dtype)

    def intact(self):
        raw = self.raw.cpu().numpy()
        return bool(np.all(raw[:GUARD] == CANARY) and np.all(raw[self.tail:] == CANARY))


def guarded_nf4(lib, rows, cols):
    sb = lib.storage_bytes(rows * cols)
    parts = [Guarded(sb["codes"], torch.uint8), Guarded(sb["absmax"], torch.uint8),
             Guarded(sb["scale2"] // 4, torch.float32), Guarded(1, torch.float32)]
    q = lib.NF4Weight(parts[0].t, parts[1].t, parts[2].t, parts[3].t, rows, cols)
    return q, parts


@pytest.mark.parametrize("n", [1, 3, 63, 65, 127, 4095, 4097, 16385, 16384 * 3 + 7, 64 * 256 * 11 + 33, 606_213])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_codec_outputs_stay_inside_their_buffers(lib, n, dtype):
    x = synth.sweep_f32(n, seed=5, tensor_id=n % 997)
    w = torch.from_numpy(x).cuda() if dtype == "f32" else synth.to_bf16(x).cuda()
    ref = O.quantize(x if dtype == "f32" else synth.bf16_bits(synth.to_bf16(x)))
    ws = Guarded(lib.quantize_workspace_bytes(n), torch.uint8)
    q, parts = guarded_nf4(lib, 1, n)
    lib.quantize(w.reshape(1, n), out=q, workspace=ws.t)
    assert lib.get_status() == 0
    assert all(p.intact() for p in parts) and ws.intact()
    assert np.array_equal(q.codes.cpu().numpy(), ref.codes)
    assert np.array_equal(q.absmax_e4m3.cpu().numpy(), ref.absmax_e4m3)
    for out_dtype, tag in ((torch.bfloat16, "bf16"), (torch.float32, "f32")):
        o = Guarded(n, out_dtype)
        lib.dequantize(q, out_dtype, out=o.t.reshape(1, n))
        assert o.intact(), tag
        got = o.t.cpu().view(torch.int16 if tag == "bf16" else torch.int32).numpy().view(
            np.uint16 if tag == "bf16" else np.uint32)
        assert np.array_equal(got, O.dequantize(ref, tag).reshape(-1).view(got.dtype)), tag


@pytest.mark.parametrize("n", [1, 65, 4097, 100_003])
def test_single_and_noalloc_outputs_stay_inside_their_buffers(lib, n):
    x = synth.sweep_f32(n, seed=6, tensor_id=n % 991)
    w = torch.from_numpy(x).cuda().reshape(1, n)
    codes, absmax = Guarded(-(-n // 2), torch.uint8), Guarded(-(-n // 64), torch.float32)
    qs = lib.NF4SingleWeight(codes.t, absmax.t, 1, n)
    lib.quantize_single(w, out=qs)
    o = Guarded(n, torch.bfloat16)
    lib.dequantize_single(qs, torch.bfloat16, out=o.t.reshape(1, n))
    q, parts = guarded_nf4(lib, 1, n)
    lib.quantize_noalloc(w, q)
    assert lib.get_status() == 0
    assert codes.intact() and absmax.intact() and o.intact() and all(p.intact() for p in parts)
    ref = O.quantize(x)
    assert np.array_equal(q.codes.cpu().numpy(), ref.codes)


@pytest.mark.parametrize("T,N,K,r", [(1, 264, 192, 8), (3, 1000, 320, 24), (9, 8, 64, 8), (17, 520, 704, 64),
                                     (33, 136, 1088, 136), (64, 1032, 128, 16), (65, 392, 320, 24),
                                     (12, 200, 640, 136), (2, 11848, 128, 16),
                                     (129, 520, 128, 64), (300, 8, 576, 256)])
def test_linear_outputs_stay_inside_their_buffers(lib, T, N, K, r):
    """Both the small-token path (T <= 64) and the fused GEMM path, with tails in every tile dimension."""
    case = synth.linear_case(T=T, N=N, K=K, r=r, alpha=16.0, seed=7)
    W = case["W"]
    q = lib.quantize(torch.from_numpy(W).cuda())
    d = {k: case[k].cuda() for k in ("X", "A", "B", "dY")}
    ws = Guarded(lib.linear_workspace_bytes(T, N, K, r), torch.uint8)
    Y, U = Guarded(T * N, torch.bfloat16), Guarded(T * r, torch.bfloat16)
    lib.linear_fwd(d["X"], q, d["A"], d["B"], 16.0, out=Y.t.view(T, N), U_out=U.t.view(T, r), workspace=ws.t)
    dX, dA, dB = Guarded(T * K, torch.bfloat16), Guarded(r * K, torch.float32), Guarded(N * r, torch.float32)
    lib.linear_bwd(d["dY"], d["X"], q, d["A"], d["B"], 16.0, U=U.t.view(T, r), dX=dX.t.view(T, K),
                   dA=dA.t.view(r, K), dB=dB.t.view(N, r), workspace=ws.t)
    # the backward again with U recomputed in the workspace
    dX2 = Guarded(T * K, torch.bfloat16)
    lib.linear_bwd(d["dY"], d["X"], q, d["A"], d["B"], 16.0, U=None, dX=dX2.t.view(T, K), dA=dA.t.view(r, K),
                   dB=dB.t.view(N, r), workspace=ws.t)
    assert lib.get_status() == 0
    for name, g in (("Y", Y), ("U", U), ("dX", dX), ("dA", dA), ("dB", dB), ("dX2", dX2), ("workspace", ws)):
        assert g.intact(), name
    Wt = O.bf16_bits_to_f32(O.dequantize(O.quantize(W), "bf16")).reshape(W.shape)
    h = {k: synth.bf16_values(case[k]) for k in ("X", "A", "B", "dY")}
    Yr, _ = O.linear_fwd(h["X"], Wt, h["A"], h["B"], 16.0)
    dXr, dAr, dBr = O.linear_bwd(h["dY"], h["X"], Wt, h["A"], h["B"], 16.0)

    def rel(a, b):
        a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
        return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))

    assert rel(Y.t.view(T, N).float().cpu(), Yr) <= TOL
    assert rel(dX.t.view(T, K).float().cpu(), dXr) <= TOL
    assert torch.equal(dX.t, dX2.t)
    assert rel(dA.t.view(r, K).cpu(), dAr) <= TOL and rel(dB.t.view(N, r).cpu(), dBr) <= TOL
