"""Seeded synthetic inputs shared by the tests, the smoke check and the benchmark.

This module only draws random numbers and shapes them into the workloads the QLoRA pages describe
(LLaMA-shaped weight matrices with a few large outliers, normal activations, small LoRA adapters).
It holds none of the method's arithmetic: no quantization, no codebook, no matrix products.

Recipe (stated once, used everywhere):
  * generator: numpy's Philox4x64-10 counter-based bit generator, keyed by (seed, tensor_id), so every
    tensor of a workload has its own independent stream and can be regenerated alone;
  * normals: numpy's standard_normal on that stream, scaled by the requested sigma, rounded once to fp32;
  * outliers (weights only): an independent Bernoulli(p) stream (tensor_id + 2**20) marks elements whose
    value is multiplied by 10 (the "0.1 % outliers x10" of the LLaMA-shaped configurations);
  * bf16 tensors: the fp32 draw rounded to nearest-even bf16 by torch's CPU conversion.
"""
from __future__ import annotations

import numpy as np
import torch

OUTLIER_STREAM = 1 << 20
SIGMA_STREAM = 1 << 21


def rng(seed: int, tensor_id: int) -> np.random.Generator:
    return np.random.Generator(np.random.Philox(key=[int(seed), int(tensor_id)]))


def normal_f32(shape, sigma: float = 1.0, seed: int = 0, tensor_id: int = 0) -> np.ndarray:
    """N(0, sigma^2) samples drawn in fp64 and rounded once to fp32."""
    x = rng(seed, tensor_id).standard_normal(size=shape)
    return (x * sigma).astype(np.float32)


def weight_f32(rows: int, cols: int, sigma: float = 0.02, outlier_p: float = 0.001,
               seed: int = 0, tensor_id: int = 0) -> np.ndarray:
    """An out x in weight, N(0, sigma^2), with a fraction outlier_p of entries scaled by 10."""
    w = rng(seed, tensor_id).standard_normal(size=(rows, cols)) * sigma
    if outlier_p > 0:
        mask = rng(seed, tensor_id + OUTLIER_STREAM).random(size=(rows, cols)) < outlier_p
        w = np.where(mask, w * 10.0, w)
    return w.astype(np.float32)


def sweep_f32(n: int, row: int = 4096, sigma_lo: float = 0.005, sigma_hi: float = 0.05,
              outlier_p: float = 0.001, seed: int = 0, tensor_id: int = 0) -> np.ndarray:
    """A flat tensor of n values in rows of `row` elements, each row N(0, s^2) with
    s ~ U(sigma_lo, sigma_hi), plus outliers as in weight_f32 (the quantize/dequant sweep workload)."""
    nrows = -(-n // row)
    sig = rng(seed, tensor_id + SIGMA_STREAM).uniform(sigma_lo, sigma_hi, size=nrows)
    x = rng(seed, tensor_id).standard_normal(size=n)
    x *= np.repeat(sig, row)[:n]
    if outlier_p > 0:
        mask = rng(seed, tensor_id + OUTLIER_STREAM).random(size=n) < outlier_p
        x = np.where(mask, x * 10.0, x)
    return x.astype(np.float32)


def to_bf16(x: np.ndarray) -> torch.Tensor:
    """fp32 numpy -> bf16 torch tensor (round to nearest even, torch's CPU conversion)."""
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)


def bf16_values(t: torch.Tensor) -> np.ndarray:
    """The exact values of a bf16 tensor as fp32 numpy (widening is exact)."""
    return t.detach().to("cpu").to(torch.float32).numpy()


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """The raw 16-bit patterns of a bf16 tensor."""
    return t.detach().to("cpu").contiguous().view(torch.int16).numpy().view(np.uint16)


# ---- the workloads of the QLoRA linear and codec configurations ---------------------------------

def linear_case(T: int, N: int, K: int, r: int, alpha: float, seed: int = 0,
                w_sigma: float = 0.02, outlier_p: float = 0.001, ab_sigma: float = 0.01,
                zero_w: bool = False, zero_a: bool = False, zero_b: bool = False) -> dict:
    """Inputs of one QLoRA linear layer: W (N x K fp32, to be quantized), X (T x K bf16),
    A (r x K bf16), B (N x r bf16), dY (T x N bf16); all N(0, .) as in the configurations."""
    W = np.zeros((N, K), np.float32) if zero_w else weight_f32(N, K, w_sigma, outlier_p, seed, 1)
    X = to_bf16(normal_f32((T, K), 1.0, seed, 2))
    A = to_bf16(np.zeros((r, K), np.float32) if zero_a else normal_f32((r, K), ab_sigma, seed, 3))
    B = to_bf16(np.zeros((N, r), np.float32) if zero_b else normal_f32((N, r), ab_sigma, seed, 4))
    dY = to_bf16(normal_f32((T, N), 1.0, seed, 5))
    return dict(W=W, X=X, A=A, B=B, dY=dY, T=T, N=N, K=K, r=r, alpha=float(alpha))


TINY = dict(T=16, N=256, K=256, r=8, alpha=16.0)                 # the small correctness case
LLAMA7B_SHAPES = [(4096, 4096), (11008, 4096), (4096, 11008)]   # (N, K) = (out, in)
LLAMA7B_TOKENS = 16 * 512
LLAMA7B_R, LLAMA7B_ALPHA = 64, 16.0
LLAMA65B_SHAPES = [(8192, 8192), (22016, 8192), (8192, 22016)]  # decode-shaped linears
