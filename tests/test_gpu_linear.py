"""GPU parity of the QLoRA linear layer against the fp64 oracle: Y, U, dX, dA, dB within a normwise
relative error of 5e-3 (bf16 inputs, fp32 accumulation), including adapter-only and base-only cases,
ragged tile tails, and sampled outputs at the LLaMA-7B-shaped size."""
import numpy as np
import pytest
import torch

import oracle as O
import synth

pytestmark = pytest.mark.gpu
TOL = 5e-3


def rel(got, ref):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    return float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300))


def setup(lib, case):
    W = case["W"]
    q = lib.quantize(torch.from_numpy(W).cuda())
    Wt = O.bf16_bits_to_f32(O.dequantize(O.quantize(W), "bf16")).reshape(W.shape)
    dev = {k: case[k].cuda() for k in ("X", "A", "B", "dY")}
    host = {k: synth.bf16_values(case[k]) for k in ("X", "A", "B", "dY")}
    return q, Wt, dev, host


def run_and_check(lib, case, check_u=True):
    q, Wt, d, h = setup(lib, case)
    alpha, r = case["alpha"], case["r"]
    Y, U = lib.linear_fwd(d["X"], q, d["A"], d["B"], alpha)
    dX, dA, dB = lib.linear_bwd(d["dY"], d["X"], q, d["A"], d["B"], alpha, U=U)
    assert lib.get_status() == 0
    Yr, Ur = O.linear_fwd(h["X"], Wt, h["A"], h["B"], alpha)
    dXr, dAr, dBr = O.linear_bwd(h["dY"], h["X"], Wt, h["A"], h["B"], alpha)
    errs = dict(Y=rel(Y.float().cpu(), Yr), dX=rel(dX.float().cpu(), dXr), dA=rel(dA.cpu(), dAr),
                dB=rel(dB.cpu(), dBr))
    if check_u:
        errs["U"] = rel(U.float().cpu(), (alpha / r) * Ur)
    for k, e in errs.items():
        assert e <= TOL, (k, e, errs)
    return errs, (Y, U, dX, dA, dB), q, d


def test_tiny_config(lib):
    case = synth.linear_case(**synth.TINY, seed=0)
    errs, *_ = run_and_check(lib, case)


def test_adapter_only_when_weight_is_zero(lib):
    """W = 0 quantizes to code 7 everywhere, so Y and dX are the LoRA terms alone."""
    case = synth.linear_case(T=200, N=264, K=192, r=16, alpha=16.0, seed=1, zero_w=True)
    errs, (Y, U, dX, dA, dB), *_ = run_and_check(lib, case)
    assert float(Y.float().abs().max()) > 0


@pytest.mark.parametrize("zero", ["a", "b"])
def test_base_only_when_adapter_is_zero(lib, zero):
    case = synth.linear_case(T=130, N=256, K=320, r=8, alpha=16.0, seed=2, zero_a=(zero == "a"),
                             zero_b=(zero == "b"))
    q, Wt, d, h = setup(lib, case)
    Y, U = lib.linear_fwd(d["X"], q, d["A"], d["B"], 16.0)
    Yr = h["X"].astype(np.float64) @ Wt.T.astype(np.float64)
    assert rel(Y.float().cpu(), Yr) <= TOL
    dX, dA, dB = lib.linear_bwd(d["dY"], d["X"], q, d["A"], d["B"], 16.0, U=U)
    dXr, dAr, dBr = O.linear_bwd(h["dY"], h["X"], Wt, h["A"], h["B"], 16.0)
    assert rel(dX.float().cpu(), dXr) <= TOL
    if zero == "a":
        assert rel(dA.cpu(), dAr) <= TOL and float(dB.abs().max()) == 0.0
    else:
        assert float(dA.abs().max()) == 0.0 and rel(dB.cpu(), dBr) <= TOL


@pytest.mark.parametrize("T,N,K,r", [(300, 392, 320, 24), (129, 520, 128, 64), (1, 256, 64, 8),
                                     (17, 8, 576, 256), (515, 1032, 704, 136)])
def test_ragged_tiles(lib, T, N, K, r):
    """Tails in every tiled dimension: tokens (128-row tiles), outputs (256-wide tiles), the 64-deep
    contraction of the backward, and adapter ranks that are not multiples of 64."""
    case = synth.linear_case(T=T, N=N, K=K, r=r, alpha=16.0, seed=3)
    run_and_check(lib, case)


def test_bwd_recomputes_u_identically(lib):
    case = synth.linear_case(T=257, N=512, K=384, r=64, alpha=16.0, seed=4)
    errs, (Y, U, dX, dA, dB), q, d = run_and_check(lib, case)
    dX2, dA2, dB2 = lib.linear_bwd(d["dY"], d["X"], q, d["A"], d["B"], 16.0, U=None)
    assert torch.equal(dX, dX2) and torch.equal(dA, dA2) and torch.equal(dB, dB2)
    _, dA3, dB3 = lib.linear_bwd(d["dY"], d["X"], q, d["A"], d["B"], 16.0, U=U, need_dx=False)
    assert torch.equal(dA, dA3) and torch.equal(dB, dB3)


def test_deterministic(lib):
    case = synth.linear_case(T=384, N=768, K=512, r=64, alpha=16.0, seed=5)
    q, Wt, d, h = setup(lib, case)
    outs = [lib.linear_fwd(d["X"], q, d["A"], d["B"], 16.0) for _ in range(2)]
    assert torch.equal(outs[0][0], outs[1][0]) and torch.equal(outs[0][1], outs[1][1])
    g = [lib.linear_bwd(d["dY"], d["X"], q, d["A"], d["B"], 16.0) for _ in range(2)]
    for a, b in zip(g[0], g[1]):
        assert torch.equal(a, b)


@pytest.mark.parametrize("N,K", synth.LLAMA7B_SHAPES)
def test_llama7b_shapes_sampled(lib, N, K):
    """The bench workload (T = 16 x 512 tokens, r = 64, alpha = 16) in the same launch configuration:
    Y and dX on 48 sampled token rows against the oracle, dA and dB in full (fp64 GEMMs over all T)."""
    T, r, alpha = synth.LLAMA7B_TOKENS, synth.LLAMA7B_R, synth.LLAMA7B_ALPHA
    case = synth.linear_case(T=T, N=N, K=K, r=r, alpha=alpha, seed=0)
    q, Wt, d, h = setup(lib, case)
    Y, U = lib.linear_fwd(d["X"], q, d["A"], d["B"], alpha)
    dX, dA, dB = lib.linear_bwd(d["dY"], d["X"], q, d["A"], d["B"], alpha, U=U)
    assert lib.get_status() == 0
    rows = np.sort(np.random.default_rng(7).choice(T, 48, replace=False))
    Yr, _ = O.linear_fwd(h["X"][rows], Wt, h["A"], h["B"], alpha)
    assert rel(Y.float().cpu().numpy()[rows], Yr) <= TOL
    s = alpha / r
    X64, dY64 = h["X"].astype(np.float64), h["dY"].astype(np.float64)
    V = dY64[rows] @ h["B"].astype(np.float64)
    dXr = dY64[rows] @ Wt.astype(np.float64) + s * V @ h["A"].astype(np.float64)
    assert rel(dX.float().cpu().numpy()[rows], dXr) <= TOL
    Vall = dY64 @ h["B"].astype(np.float64)
    assert rel(dA.cpu(), s * Vall.T @ X64) <= TOL
    assert rel(dB.cpu(), s * dY64.T @ (X64 @ h["A"].astype(np.float64).T)) <= TOL


@pytest.mark.parametrize("N,K", [(4096, 256), (256, 4096)])
def test_persistent_tiles_full_compare(lib, N, K):
    """More output tiles than SMs (4096 features x 4096 tokens = 32 x 16 tiles, in the forward for the
    first shape and in the backward for the second): each persistent CTA runs several tiles through the
    shared-memory ring and both tensor-memory accumulators. Every output is compared."""
    case = synth.linear_case(T=4096, N=N, K=K, r=64, alpha=16.0, seed=6)
    run_and_check(lib, case)


# ---- small token counts (decode shapes): the stream-K GEMV path serves T <= 64 --------------------

@pytest.mark.parametrize("T", [1, 2, 4, 7, 8, 9, 16, 17, 32, 33, 64])
@pytest.mark.parametrize("N,K,r", [(520, 704, 24), (1000, 320, 64)])
def test_small_token_forward(lib, T, N, K, r):
    """T <= 64 runs the small-token kernels: tails in rows (partial row tiles), in the contraction
    (partial stages), in tokens (8-wide MMA tiles) and in r (16-deep MMA steps). Y and U against the oracle; the backward
    (GEMM path) against the oracle as well, with U from this forward and recomputed."""
    case = synth.linear_case(T=T, N=N, K=K, r=r, alpha=16.0, seed=11 + T)
    errs, (Y, U, dX, dA, dB), q, d = run_and_check(lib, case)
    dX2, dA2, dB2 = lib.linear_bwd(d["dY"], d["X"], q, d["A"], d["B"], 16.0, U=None)
    assert torch.equal(dA, dA2) and torch.equal(dB, dB2)


@pytest.mark.parametrize("T", [1, 16])
def test_small_token_adapter_only_and_base_only(lib, T):
    case = synth.linear_case(T=T, N=496, K=448, r=16, alpha=16.0, seed=21, zero_w=True)
    errs, (Y, U, dX, dA, dB), *_ = run_and_check(lib, case)
    assert float(Y.float().abs().max()) > 0
    case = synth.linear_case(T=T, N=496, K=448, r=16, alpha=16.0, seed=22, zero_b=True)
    q, Wt, d, h = setup(lib, case)
    Y, U = lib.linear_fwd(d["X"], q, d["A"], d["B"], 16.0)
    Yr = h["X"].astype(np.float64) @ Wt.T.astype(np.float64)
    assert rel(Y.float().cpu(), Yr) <= TOL


def test_small_token_deterministic(lib):
    case = synth.linear_case(T=5, N=2048, K=4096, r=64, alpha=16.0, seed=23)
    q, Wt, d, h = setup(lib, case)
    outs = [lib.linear_fwd(d["X"], q, d["A"], d["B"], 16.0) for _ in range(3)]
    for o in outs[1:]:
        assert torch.equal(outs[0][0], o[0]) and torch.equal(outs[0][1], o[1])


@pytest.mark.parametrize("T", [64, 65])
def test_gemv_and_gemm_paths_at_the_boundary(lib, T):
    """T = 64 is the last GEMV size, T = 65 the first fused-GEMM size: both meet the oracle's tolerance on
    the same layer, so the two paths agree with each other to twice it."""
    case = synth.linear_case(T=T, N=1024, K=1024, r=64, alpha=16.0, seed=24)
    run_and_check(lib, case)


@pytest.mark.parametrize("N,K,Ts", [(8192, 8192, (1, 4, 16)), (22016, 8192, (1, 4, 16)), (8192, 22016, (1, 4, 16)),
                                    (4096, 11008, (16,))])
def test_decode_shapes(lib, N, K, Ts):
    """The decode-shaped layers of a 65B model (attention 8192 x 8192, gate/up 22016 x 8192, down
    8192 x 22016) at the decode token counts, plus the wide contraction of a 7B down projection: every
    output of Y and U against the oracle (fp64 GEMM over the oracle's exact W_hat). The 22016-row and
    22016-deep layers are the ones whose row and contraction counts leave partial tiles and stages."""
    case = synth.linear_case(T=max(Ts), N=N, K=K, r=64, alpha=16.0, seed=25)
    q, Wt, d, h = setup(lib, case)
    for T in Ts:
        X = d["X"][:T].contiguous()
        Y, U = lib.linear_fwd(X, q, d["A"], d["B"], 16.0)
        assert lib.get_status() == 0
        Yr, Ur = O.linear_fwd(h["X"][:T], Wt, h["A"], h["B"], 16.0)
        assert rel(Y.float().cpu(), Yr) <= TOL, T
        assert rel(U.float().cpu(), (16.0 / 64) * Ur) <= TOL, T


def test_small_token_and_gemm_paths_agree(lib):
    """The same 64 tokens through the small-token path (T = 64) and, as the first 64 of 65 tokens,
    through the fused GEMM path: the two results agree with each other within the oracle tolerance."""
    case = synth.linear_case(T=65, N=2048, K=1536, r=64, alpha=16.0, seed=26)
    q, Wt, d, h = setup(lib, case)
    Y64, U64 = lib.linear_fwd(d["X"][:64].contiguous(), q, d["A"], d["B"], 16.0)
    Y65, U65 = lib.linear_fwd(d["X"], q, d["A"], d["B"], 16.0)
    assert lib.get_status() == 0
    assert rel(Y64.float().cpu(), Y65[:64].float().cpu()) <= TOL
    assert rel(U64.float().cpu(), U65[:64].float().cpu()) <= TOL


@pytest.mark.parametrize("T,N,K,r", [(2, 11848, 128, 16),     # ~10 row units per CTA: two passes
                                     (16, 45056, 64, 8),      # per-CTA results kept in the workspace
                                     (12, 200, 640, 136),     # r > 64: several adapter column boxes
                                     (4, 64, 256, 256),       # the largest rank
                                     (7, 96, 1088, 64),       # 17 blocks: a last stage with one block
                                     (16, 8, 64, 8)])         # one row unit: a one-CTA grid
def test_decode_path_structure(lib, T, N, K, r):
    """The decode-sized path (T <= 16) in the configurations its structure depends on; Y and U against
    the oracle, and the backward's recomputed U bit-identical to the forward's."""
    case = synth.linear_case(T=T, N=N, K=K, r=r, alpha=16.0, seed=27)
    errs, (Y, U, dX, dA, dB), q, d = run_and_check(lib, case)
    dX2, dA2, dB2 = lib.linear_bwd(d["dY"], d["X"], q, d["A"], d["B"], 16.0, U=None)
    assert torch.equal(dA, dA2) and torch.equal(dB, dB2) and torch.equal(dX, dX2)
    Y2, U2 = lib.linear_fwd(d["X"], q, d["A"], d["B"], 16.0)
    assert torch.equal(Y, Y2) and torch.equal(U, U2)
