"""The QLoRA linear layer, forward and backward, in fp64.

Test infrastructure (see the package docstring).

Sources:
  QLoRA explainer (prism.theerrors.in), "Putting it together": Y = X . dequant(W_4bit) + X . L1 . L2
    (the simplified Eq. 5); storage type 4-bit, compute type bf16; gradients flow only into L1, L2,
    never into the 4-bit weights.
  PEFT page (zerotofrontier.app/sft/peft), "Paged optimizers, and QLoRA end to end": each frozen
    matrix is dequantized to bf16 on the fly and multiplied in 16-bit precision, a bf16 LoRA adapter
    is added to its output, gradients flow backward through the dequantized weights to reach earlier
    layers, and the 4-bit weights are constants; r = 64, alpha = 16.
  arXiv abstract (mlsanity.com): QLoRA backpropagates through the frozen 4-bit model into LoRA.

Reading: W is out x in (PyTorch layout, as the PEFT page's IA3/DoRA paragraphs use), so
  Y  = X W~^T + s (X A^T) B^T                with s = alpha / r (LoRA's scaling), A: r x in, B: out x r
  dX = dY W~ + s (dY B) A
  dA = s (dY B)^T X
  dB = s dY^T (X A^T)
No bias (LLaMA-style linears have none) and no dropout (the pages mention neither); no dW.
The explainer's L1, L2 are A^T and s B^T.  Inputs are the exact bf16 values; W~ is the bit-exact
dequantized weight from codec.dequantize; everything after that is fp64 with no intermediate rounding.
"""
from __future__ import annotations

import numpy as np


def _f64(x):
    return np.asarray(x, dtype=np.float64)


def linear_fwd(X, Wt, A, B, alpha: float):
    """Y (T x N) and U = X A^T (T x r), in fp64."""
    X, Wt, A, B = map(_f64, (X, Wt, A, B))
    s = float(alpha) / A.shape[0]
    U = X @ A.T
    Y = X @ Wt.T + s * (U @ B.T)
    return Y, U


def linear_bwd(dY, X, Wt, A, B, alpha: float):
    """(dX, dA, dB) in fp64; the frozen weight gets no gradient."""
    dY, X, Wt, A, B = map(_f64, (dY, X, Wt, A, B))
    s = float(alpha) / A.shape[0]
    U = X @ A.T
    V = dY @ B
    dX = dY @ Wt + s * (V @ A)
    dA = s * (V.T @ X)
    dB = s * (dY.T @ U)
    return dX, dA, dB
