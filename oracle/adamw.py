"""AdamW, the optimizer whose states the paged optimizer keeps in unified memory.

Test infrastructure (see the package docstring).

Sources:
  PEFT page (zerotofrontier.app/sft/peft), "Paged optimizers, and QLoRA end to end": the optimizer
    states live in unified memory that the driver pages between GPU and CPU; with LoRA they are small;
    learning rate 2e-4 (1e-4 for the largest models).
  QLoRA explainer (prism.theerrors.in), "The three innovations": paged optimizers absorb the memory
    spikes of gradient checkpointing.
  The update itself is not written on the pages; it is the standard AdamW step (Adam with decoupled
  weight decay, Loshchilov & Hutter, "Decoupled Weight Decay Regularization", 2019, Algorithm 2).

Reading R-adamw (one step t = 1, 2, ... for parameter p, gradient g, first and second moments m, v):
    p <- p * (1 - lr * wd)
    m <- beta1 * m + (1 - beta1) * g
    v <- beta2 * v + (1 - beta2) * g^2
    p <- p - lr * (m / (1 - beta1^t)) / (sqrt(v / (1 - beta2^t)) + eps)
  in fp64 here; the states and parameters are fp32 on the GPU. Defaults beta1 = 0.9, beta2 = 0.999,
  eps = 1e-8, wd = 0 (the pages give only the learning rate).
"""
from __future__ import annotations

import numpy as np


def adamw_step(p, g, m, v, t: int, lr: float, beta1: float = 0.9, beta2: float = 0.999, eps: float = 1e-8,
               wd: float = 0.0):
    """One AdamW step (reading R-adamw) in fp64; returns the new (p, m, v) as fp64 arrays."""
    if t < 1:
        raise ValueError("step count t starts at 1")
    p = np.asarray(p, np.float64) * (1.0 - lr * wd)
    g = np.asarray(g, np.float64)
    m = beta1 * np.asarray(m, np.float64) + (1.0 - beta1) * g
    v = beta2 * np.asarray(v, np.float64) + (1.0 - beta2) * g * g
    mhat = m / (1.0 - beta1 ** t)
    vhat = v / (1.0 - beta2 ** t)
    p = p - lr * mhat / (np.sqrt(vhat) + eps)
    return p, m, v
