"""The paged optimizer: AdamW over the trainable LoRA parameters with its moment states in unified memory.

PEFT page (zerotofrontier.app/sft/peft), "Paged optimizers, and QLoRA end to end": the optimizer states
are allocated in NVIDIA unified memory, evicted to host RAM when the GPU runs short and paged back when
the optimizer step touches them. The parameters (and their gradients) are gathered into one flat fp32
buffer each, so one launch of the library's fused AdamW kernel updates every adapter; the moments m and v
live in managed memory from qlora_paged_alloc (or in device memory with paged=False, for comparison).
Argument marshalling and buffer bookkeeping only: the update runs in the library's kernel.
"""
from __future__ import annotations

import threading

import torch

from . import adamw_step, paged_empty, paged_prefetch


class PagedAdamW:
    def __init__(self, params, lr: float = 2e-4, betas=(0.9, 0.999), eps: float = 1e-8, weight_decay: float = 0.0,
                 paged: bool = True):
        self.params = [p for p in params]
        if not self.params:
            raise ValueError("PagedAdamW: no parameters")
        dev = self.params[0].device
        for p in self.params:
            if p.dtype != torch.float32 or not p.is_cuda or p.device != dev:
                raise ValueError("PagedAdamW: parameters must be float32 CUDA tensors on one device")
        self.lr, self.betas, self.eps, self.weight_decay = lr, tuple(betas), eps, weight_decay
        self.paged = paged
        n = sum(p.numel() for p in self.params)
        self.n = n
        self.flat_p = torch.empty(n, dtype=torch.float32, device=dev)
        self.flat_g = torch.zeros(n, dtype=torch.float32, device=dev)
        off = 0
        for p in self.params:          # parameters and gradients become views of the flat buffers
            k = p.numel()
            self.flat_p[off:off + k].copy_(p.detach().reshape(-1))
            p.data = self.flat_p[off:off + k].view_as(p)
            p.grad = self.flat_g[off:off + k].view_as(p)
            off += k
        if paged:
            self.m, self.v = paged_empty(n, dev), paged_empty(n, dev)
        else:
            self.m = torch.empty(n, dtype=torch.float32, device=dev)
            self.v = torch.empty(n, dtype=torch.float32, device=dev)
        self.m.zero_()
        self.v.zero_()
        self.t = 0
        self._side = None
        self._ready = None
        self._thread = None

    def zero_grad(self) -> None:
        """Zero the gradients in place (they are views of one flat buffer that autograd adds into)."""
        self.flat_g.zero_()

    def step(self, stream=None) -> None:
        if self._ready is not None:            # moments still on their way back: wait on the device
            self._thread.join()
            (stream if stream is not None else torch.cuda.current_stream()).wait_event(self._ready)
            self._ready = None
            self._thread = None
        self.t += 1
        adamw_step(self.flat_p, self.flat_g, self.m, self.v, self.t, self.lr, self.betas, self.eps,
                   self.weight_decay, stream=stream)

    def evict_states(self, stream=None) -> None:
        """Move the moment states to host memory, as the driver does under GPU memory pressure."""
        if not self.paged:
            raise RuntimeError("PagedAdamW: states are in device memory (paged=False)")
        paged_prefetch(self.m, False, stream)
        paged_prefetch(self.v, False, stream)

    def prefetch_states(self, stream=None) -> None:
        """Bring the moment states back to the GPU ahead of the step."""
        if not self.paged:
            return
        paged_prefetch(self.m, True, stream)
        paged_prefetch(self.v, True, stream)

    def side_stream(self) -> torch.cuda.Stream:
        if self._side is None:
            self._side = torch.cuda.Stream(device=self.flat_p.device)
        return self._side

    def prefetch_states_async(self, evict_first: bool = False) -> None:
        """Bring the moments back to the GPU on a side stream, issued from a worker thread (a migration
        call can hold the calling thread while the driver moves pages), so that it overlaps whatever the
        current stream runs next -- the forward and backward passes; the next step() waits for it.
        evict_first moves them to the host first, as the driver does under a memory spike (to measure
        the cost of paging)."""
        if not self.paged:
            return
        side = self.side_stream()
        side.wait_stream(torch.cuda.current_stream())
        ready = torch.cuda.Event()
        dev = self.flat_p.device

        def work():
            torch.cuda.set_device(dev)
            if evict_first:
                paged_prefetch(self.m, False, side)
                paged_prefetch(self.v, False, side)
            paged_prefetch(self.m, True, side)
            paged_prefetch(self.v, True, side)
            ready.record(side)

        self._thread = threading.Thread(target=work, daemon=True)
        self._thread.start()
        self._ready = ready

    def state_bytes(self) -> int:
        return 8 * self.n
