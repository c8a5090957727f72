"""Pins for the oracle's QLoRA linear layer: PyTorch's own linear for the base term and for the merged
LoRA weight, the alpha/r scaling, and adjoint identities tying the backward to the forward."""
import numpy as np
import torch
import torch.nn.functional as F

import oracle as O
import synth


def _case(T=5, N=12, K=128, r=4, alpha=16.0, seed=3):
    c = synth.linear_case(T, N, K, r, alpha, seed=seed)
    t = O.quantize(c["W"])
    Wt = O.bf16_bits_to_f32(O.dequantize(t, "bf16")).reshape(N, K)
    X, A, B, dY = (synth.bf16_values(c[k]) for k in ("X", "A", "B", "dY"))
    return X, Wt, A, B, dY, alpha, r


def _t(x):
    return torch.from_numpy(np.asarray(x, np.float64))


def test_base_term_is_pytorch_linear_with_out_by_in_weight():
    X, Wt, A, B, dY, alpha, r = _case()
    Y, _ = O.linear_fwd(X, Wt, np.zeros_like(A), B, alpha)
    assert np.allclose(Y, F.linear(_t(X), _t(Wt)).numpy(), rtol=1e-13, atol=1e-13)


def test_lora_term_equals_merged_weight():
    """Y = X (W~ + (alpha/r) B A)^T: the adapter merges into the out x in weight."""
    X, Wt, A, B, dY, alpha, r = _case()
    Y, U = O.linear_fwd(X, Wt, A, B, alpha)
    merged = _t(Wt) + (alpha / r) * (_t(B) @ _t(A))
    assert np.allclose(Y, F.linear(_t(X), merged).numpy(), rtol=1e-12, atol=1e-12)
    assert np.allclose(U, F.linear(_t(X), _t(A)).numpy(), rtol=1e-13, atol=1e-13)


def test_scale_is_alpha_over_r():
    """Doubling alpha doubles the adapter term; doubling r by zero-padding the adapter halves it."""
    X, Wt, A, B, dY, alpha, r = _case()
    base, _ = O.linear_fwd(X, Wt, np.zeros_like(A), B, alpha)
    y1, _ = O.linear_fwd(X, Wt, A, B, alpha)
    y2, _ = O.linear_fwd(X, Wt, A, B, 2 * alpha)
    assert np.allclose(y2 - base, 2 * (y1 - base), rtol=1e-10, atol=1e-12)
    A2 = np.concatenate([A, np.zeros_like(A)], 0)
    B2 = np.concatenate([B, np.zeros_like(B)], 1)
    y3, _ = O.linear_fwd(X, Wt, A2, B2, alpha)
    assert np.allclose(y3 - base, 0.5 * (y1 - base), rtol=1e-10, atol=1e-12)


def test_backward_adjoint_identities():
    """Y is affine in each of X, A, B, so <dY, Y(P+E) - Y(P)> = <dP, E> up to fp64 rounding."""
    X, Wt, A, B, dY, alpha, r = _case(T=7, N=24, K=192, r=8)
    rng = np.random.default_rng(8)
    dX, dA, dB = O.linear_bwd(dY, X, Wt, A, B, alpha)
    Y0, _ = O.linear_fwd(X, Wt, A, B, alpha)
    for name, P, G in (("X", X, dX), ("A", A, dA), ("B", B, dB)):
        E = rng.normal(0, 1, P.shape)
        args = dict(X=X, A=A, B=B)
        args[name] = P + E
        Y1, _ = O.linear_fwd(args["X"], Wt, args["A"], args["B"], alpha)
        lhs = float(np.sum(dY * (Y1 - Y0)))
        rhs = float(np.sum(G * E))
        assert abs(lhs - rhs) <= 1e-10 * (abs(lhs) + 1.0), name


def test_no_gradient_path_to_the_frozen_weight_and_torch_autograd():
    """Autograd through the same expression gives the same dX, dA, dB; W~ is a constant."""
    X, Wt, A, B, dY, alpha, r = _case(T=6, N=16, K=64, r=4)
    tX, tA, tB = (_t(v).requires_grad_(True) for v in (X, A, B))
    Y = F.linear(tX, _t(Wt)) + (alpha / r) * F.linear(F.linear(tX, tA), tB)
    Y.backward(_t(dY))
    dX, dA, dB = O.linear_bwd(dY, X, Wt, A, B, alpha)
    for got, ref in ((dX, tX.grad), (dA, tA.grad), (dB, tB.grad)):
        assert np.allclose(got, ref.numpy(), rtol=1e-12, atol=1e-12)


def test_brute_force_loops_tiny():
    X, Wt, A, B, dY, alpha, r = _case(T=2, N=3, K=64, r=2)
    s = alpha / r
    Y, _ = O.linear_fwd(X, Wt, A, B, alpha)
    for t in range(2):
        for n in range(3):
            acc = sum(float(X[t, k]) * float(Wt[n, k]) for k in range(64))
            for j in range(r):
                acc += s * sum(float(X[t, k]) * float(A[j, k]) for k in range(64)) * float(B[n, j])
            assert abs(acc - Y[t, n]) <= 1e-12 * (1 + abs(acc))
