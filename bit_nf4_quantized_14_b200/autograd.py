"""PyTorch autograd glue for the QLoRA linear layer: the frozen NF4 weight and the trainable LoRA adapters
as one torch.autograd.Function and an nn.Module around it.

The adapters are fp32 parameters (the pages keep the adapters in full precision for training: PEFT page,
zerotofrontier.app/sft/peft, "Paged optimizers, and QLoRA end to end"); each call hands bf16 copies to the
library, which computes Y = X W_hat^T + (alpha/r) (X A^T) B^T in its kernels and returns fp32 gradients of
A and B (written straight into the parameters' .grad by autograd). The frozen weight gets no gradient
(QLoRA explainer, prism.theerrors.in, "Putting it together"). No arithmetic of the layer happens here.
"""
from __future__ import annotations

import math

import torch

from . import NF4Weight, linear_bwd, linear_fwd, quantize


class QLoRALinearFn(torch.autograd.Function):
    """y = x W_hat^T + (alpha / r) (x A^T) B^T for x of shape (..., K); returns (..., N) bf16."""

    @staticmethod
    def forward(ctx, x: torch.Tensor, A: torch.Tensor, B: torch.Tensor, w: NF4Weight, alpha: float):
        K = x.shape[-1]
        x2 = x.reshape(-1, K).to(torch.bfloat16).contiguous()
        a16 = A.detach().to(torch.bfloat16).contiguous()
        b16 = B.detach().to(torch.bfloat16).contiguous()
        y, u = linear_fwd(x2, w, a16, b16, alpha)
        ctx.save_for_backward(x2, a16, b16, u)
        ctx.w, ctx.alpha, ctx.in_shape = w, alpha, x.shape
        return y.view(*x.shape[:-1], w.rows)

    @staticmethod
    def backward(ctx, dy: torch.Tensor):
        x2, a16, b16, u = ctx.saved_tensors
        dy2 = dy.reshape(-1, ctx.w.rows).to(torch.bfloat16).contiguous()
        need_dx = ctx.needs_input_grad[0]
        dx, dA, dB = linear_bwd(dy2, x2, ctx.w, a16, b16, ctx.alpha, U=u, need_dx=need_dx)
        dx = dx.view(ctx.in_shape) if need_dx else None
        return dx, dA, dB, None, None


class QLoRALinear(torch.nn.Module):
    """A frozen weight (N x K, out x in) stored as NF4 with double-quantized constants, plus a LoRA adapter
    of rank r: A (r x K) initialised like a Kaiming-uniform linear, B (N x r) at zero, so the layer starts
    as the quantized base layer."""

    def __init__(self, weight: torch.Tensor, r: int = 64, alpha: float = 16.0,
                 generator: torch.Generator | None = None):
        super().__init__()
        if weight.dim() != 2 or not weight.is_cuda:
            raise ValueError("QLoRALinear: weight must be a 2-D CUDA tensor (out x in)")
        N, K = weight.shape
        self.w = quantize(weight.contiguous())
        self.r, self.alpha = r, float(alpha)
        bound = 1.0 / math.sqrt(K)
        a = torch.empty(r, K, device=weight.device, dtype=torch.float32).uniform_(-bound, bound, generator=generator)
        self.A = torch.nn.Parameter(a)
        self.B = torch.nn.Parameter(torch.zeros(N, r, device=weight.device, dtype=torch.float32))

    @property
    def in_features(self) -> int:
        return self.w.cols

    @property
    def out_features(self) -> int:
        return self.w.rows

    def forward(self, x: torch.Tensor) -> torch.Tensor:
        return QLoRALinearFn.apply(x, self.A, self.B, self.w, self.alpha)
