"""Python binding of libqlora_nf4.so, the B200 (sm_100a) QLoRA NF4 library.

Argument marshalling only: every step of the codec and of the linear layer runs in the library's CUDA
kernels. PyTorch provides device memory and the current stream. The names follow the C ABI in
include/qlora_nf4.h:

    quantize(w)                      -> NF4Weight     (qlora_nf4_quantize)
    dequantize(q, dtype)             -> tensor        (qlora_nf4_dequantize)
    linear_fwd(X, q, A, B, alpha)    -> (Y, U)        (qlora_linear_fwd)
    linear_bwd(dY, X, q, A, B, alpha, U) -> (dX, dA, dB)   (qlora_linear_bwd)
    codebook_quantize / codebook_dequantize / codebook_stats   (qlora_codebook_*)
    adamw_step, paged_empty, paged_prefetch   (qlora_adamw_step, qlora_paged_*; optim.PagedAdamW)

The shared library is loaded on first use (so that the build step, a submodule of this package, can run
before it exists); a call made while it is not built raises ImportError. There is no fallback
implementation.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libqlora_nf4.so")

QLORA_F32, QLORA_BF16 = 0, 1
STATUS_NONFINITE, STATUS_TIMEOUT = 1, 2
PROF_NAMES = ("quantize", "dequantize", "fwd_gemm", "bwd_gemm", "lora")


class _NF4Struct(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("absmax_e4m3", ctypes.c_void_p),
                ("scale2", ctypes.c_void_p), ("offset", ctypes.c_void_p),
                ("rows", ctypes.c_int64), ("cols", ctypes.c_int64)]


_LIB = None


def load() -> ctypes.CDLL:
    """The loaded library (loads it on the first call)."""
    global _LIB
    if _LIB is None:
        _LIB = _open()
    return _LIB


def __getattr__(name):          # `bit_nf4_quantized_14_b200.lib` is the loaded CDLL
    if name == "lib":
        return load()
    raise AttributeError(name)


def _open() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is not built; run `python -m bit_nf4_quantized_14_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i64, sz, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t, ctypes.c_int
    P = ctypes.POINTER
    sig = {
        "qlora_nf4_codebook": [P(ctypes.c_float), P(ctypes.c_float)],
        "qlora_nf4_storage_bytes": [i64, P(sz), P(sz), P(sz), P(sz)],
        "qlora_nf4_quantize_workspace": [i64, P(sz)],
        "qlora_nf4_quantize": [vp, i32, i64, i64, P(_NF4Struct), vp, sz, vp],
        "qlora_nf4_quantize_noalloc": [vp, i32, i64, i64, P(_NF4Struct), vp],
        "qlora_nf4_dequantize": [P(_NF4Struct), vp, i32, vp],
        "qlora_nf4_quantize_single": [vp, i32, i64, i64, vp, vp, vp],
        "qlora_nf4_dequantize_single": [vp, vp, i64, i64, vp, i32, vp],
        "qlora_codebook_quantize": [vp, i32, i64, P(ctypes.c_float), i32, vp, vp, vp],
        "qlora_codebook_dequantize": [vp, vp, i64, P(ctypes.c_float), i32, vp, i32, vp],
        "qlora_codebook_stats_workspace": [i64, P(sz)],
        "qlora_codebook_stats": [vp, i32, vp, vp, i64, P(ctypes.c_float), i32, vp, vp, sz, vp],
        "qlora_adamw_step": [vp, vp, vp, vp, vp, i64, i64, ctypes.c_float, ctypes.c_float, ctypes.c_float,
                             ctypes.c_float, ctypes.c_float, vp],
        "qlora_paged_alloc": [sz, P(vp)],
        "qlora_paged_free": [vp],
        "qlora_paged_prefetch": [vp, sz, i32, vp],
        "qlora_linear_workspace": [i64, i64, i64, i32, P(sz)],
        "qlora_linear_fwd": [vp, i64, P(_NF4Struct), vp, vp, i32, ctypes.c_float, vp, vp, vp, sz, vp],
        "qlora_linear_bwd": [vp, vp, i64, P(_NF4Struct), vp, vp, i32, ctypes.c_float, vp, vp, vp, vp,
                             vp, sz, vp],
        "qlora_get_status": [P(i32), vp],
        "qlora_set_wait_limit": [ctypes.c_uint64],
        "qlora_selftest_wait": [i32, vp],
        "qlora_error_string": [i32],
        "qlora_profile_enable": [i32],
        "qlora_profile_read": [P(i64), P(ctypes.c_double)],
        "qlora_kernel_launches": [],
    }
    for name, args in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = {"qlora_error_string": ctypes.c_char_p, "qlora_kernel_launches": i64}.get(name, i32)
    return lib


class QLoRAError(RuntimeError):
    def __init__(self, code: int, where: str = ""):
        self.code = code
        super().__init__(f"{where}: {load().qlora_error_string(code).decode()} (code {code})")


def _check(rc: int, where: str) -> None:
    if rc != 0:
        raise QLoRAError(rc, where)


def _stream(stream) -> ctypes.c_void_p:
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t) -> ctypes.c_void_p:
    return ctypes.c_void_p(0 if t is None else t.data_ptr())


def _need(t: torch.Tensor, dtype, name: str) -> None:
    if not t.is_cuda or t.dtype != dtype or not t.is_contiguous():
        raise ValueError(f"{name}: expected a contiguous CUDA tensor of {dtype}, got {t.dtype} on {t.device}")


# ---- host-only queries --------------------------------------------------------------------------

def codebook():
    """(levels float32[16], thresholds float32[15]) as the library uses them."""
    lv = (ctypes.c_float * 16)()
    th = (ctypes.c_float * 15)()
    _check(load().qlora_nf4_codebook(lv, th), "qlora_nf4_codebook")
    return np.array(lv, np.float32), np.array(th, np.float32)


def storage_bytes(n: int) -> dict:
    out = [ctypes.c_size_t() for _ in range(4)]
    _check(load().qlora_nf4_storage_bytes(n, *[ctypes.byref(o) for o in out]), "qlora_nf4_storage_bytes")
    return dict(codes=out[0].value, absmax=out[1].value, scale2=out[2].value, offset=out[3].value)


def quantize_workspace_bytes(n: int) -> int:
    b = ctypes.c_size_t()
    _check(load().qlora_nf4_quantize_workspace(n, ctypes.byref(b)), "qlora_nf4_quantize_workspace")
    return b.value


def linear_workspace_bytes(T: int, N: int, K: int, r: int) -> int:
    b = ctypes.c_size_t()
    _check(load().qlora_linear_workspace(T, N, K, r, ctypes.byref(b)), "qlora_linear_workspace")
    return b.value


# ---- the NF4 tensor -----------------------------------------------------------------------------

@dataclass
class NF4Weight:
    """Device buffers of an NF4 tensor with double-quantized constants (see qlora_nf4_tensor)."""
    codes: torch.Tensor        # uint8 [ceil(n/2)]
    absmax_e4m3: torch.Tensor  # uint8 [nb]
    scale2: torch.Tensor       # float32 [ng]
    offset: torch.Tensor       # float32 [1]
    rows: int
    cols: int

    @classmethod
    def empty(cls, rows: int, cols: int, device) -> "NF4Weight":
        sb = storage_bytes(rows * cols)
        u8 = dict(dtype=torch.uint8, device=device)
        return cls(torch.empty(sb["codes"], **u8), torch.empty(sb["absmax"], **u8),
                   torch.empty(sb["scale2"] // 4, dtype=torch.float32, device=device),
                   torch.empty(1, dtype=torch.float32, device=device), rows, cols)

    def struct(self) -> _NF4Struct:
        return _NF4Struct(self.codes.data_ptr(), self.absmax_e4m3.data_ptr(), self.scale2.data_ptr(),
                          self.offset.data_ptr(), self.rows, self.cols)

    @property
    def nbytes(self) -> int:
        return sum(t.numel() * t.element_size() for t in (self.codes, self.absmax_e4m3, self.scale2, self.offset))


def quantize(w: torch.Tensor, out: NF4Weight | None = None, workspace: torch.Tensor | None = None,
             stream=None) -> NF4Weight:
    """NF4 + double quantization of a CUDA fp32 or bf16 tensor (1-D or 2-D, contiguous)."""
    if w.dtype not in (torch.float32, torch.bfloat16):
        raise ValueError("quantize: w must be float32 or bfloat16")
    _need(w, w.dtype, "w")
    rows, cols = (w.shape[0], w.shape[1]) if w.dim() == 2 else (1, w.numel())
    q = out if out is not None else NF4Weight.empty(rows, cols, w.device)
    need = quantize_workspace_bytes(rows * cols)
    ws = workspace if workspace is not None else torch.empty(need, dtype=torch.uint8, device=w.device)
    st = q.struct()
    _check(load().qlora_nf4_quantize(_ptr(w), QLORA_F32 if w.dtype == torch.float32 else QLORA_BF16, rows, cols,
                                  ctypes.byref(st), _ptr(ws), ws.numel(), _stream(stream)), "qlora_nf4_quantize")
    return q


@dataclass
class NF4SingleWeight:
    """NF4 codes with the fp32 block constants kept per block of 64 (no double quantization)."""
    codes: torch.Tensor      # uint8[ceil(n/2)]
    absmax: torch.Tensor     # float32[ceil(n/64)]
    rows: int
    cols: int

    @classmethod
    def empty(cls, rows: int, cols: int, device) -> "NF4SingleWeight":
        n = rows * cols
        return cls(torch.empty(-(-n // 2), dtype=torch.uint8, device=device),
                   torch.empty(-(-n // 64), dtype=torch.float32, device=device), rows, cols)


def quantize_single(w: torch.Tensor, out: NF4SingleWeight | None = None, stream=None) -> NF4SingleWeight:
    """NF4 codes + fp32 block constants of a CUDA fp32 or bf16 tensor (1-D or 2-D, contiguous)."""
    if w.dtype not in (torch.float32, torch.bfloat16):
        raise ValueError("quantize_single: w must be float32 or bfloat16")
    _need(w, w.dtype, "w")
    rows, cols = (w.shape[0], w.shape[1]) if w.dim() == 2 else (1, w.numel())
    q = out if out is not None else NF4SingleWeight.empty(rows, cols, w.device)
    _check(load().qlora_nf4_quantize_single(_ptr(w), QLORA_F32 if w.dtype == torch.float32 else QLORA_BF16, rows,
                                            cols, _ptr(q.codes), _ptr(q.absmax), _stream(stream)),
           "qlora_nf4_quantize_single")
    return q


def dequantize_single(q: NF4SingleWeight, dtype=torch.bfloat16, out: torch.Tensor | None = None,
                      stream=None) -> torch.Tensor:
    if dtype not in (torch.float32, torch.bfloat16):
        raise ValueError("dequantize_single: dtype must be float32 or bfloat16")
    o = out if out is not None else torch.empty(q.rows, q.cols, dtype=dtype, device=q.codes.device)
    _need(o, dtype, "out")
    _check(load().qlora_nf4_dequantize_single(_ptr(q.codes), _ptr(q.absmax), q.rows, q.cols, _ptr(o),
                                              QLORA_F32 if dtype == torch.float32 else QLORA_BF16, _stream(stream)),
           "qlora_nf4_dequantize_single")
    return o


# ---- codebook comparison: any sorted codebook of 2..16 levels, fp32 block constants -------------------

CODEBOOK_STATS_LEN = 51


def _levels(levels):
    lv = np.ascontiguousarray(np.asarray(levels, dtype=np.float32).reshape(-1))
    return (ctypes.c_float * lv.size)(*lv.tolist()), int(lv.size)


def codebook_quantize(w: torch.Tensor, levels, codes: torch.Tensor | None = None,
                      absmax: torch.Tensor | None = None, stream=None):
    """(codes uint8[ceil(n/2)], absmax float32[ceil(n/64)]) of a contiguous CUDA fp32/bf16 tensor under
    `levels` (qlora_codebook_quantize)."""
    if w.dtype not in (torch.float32, torch.bfloat16):
        raise ValueError("codebook_quantize: w must be float32 or bfloat16")
    _need(w, w.dtype, "w")
    n = w.numel()
    c = codes if codes is not None else torch.empty(-(-n // 2), dtype=torch.uint8, device=w.device)
    a = absmax if absmax is not None else torch.empty(-(-n // 64), dtype=torch.float32, device=w.device)
    lv, nl = _levels(levels)
    _check(load().qlora_codebook_quantize(_ptr(w), QLORA_F32 if w.dtype == torch.float32 else QLORA_BF16, n, lv, nl,
                                          _ptr(c), _ptr(a), _stream(stream)), "qlora_codebook_quantize")
    return c, a


def codebook_dequantize(codes: torch.Tensor, absmax: torch.Tensor, n: int, levels, dtype=torch.float32,
                        out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    if dtype not in (torch.float32, torch.bfloat16):
        raise ValueError("codebook_dequantize: dtype must be float32 or bfloat16")
    o = out if out is not None else torch.empty(n, dtype=dtype, device=codes.device)
    _need(o, dtype, "out")
    lv, nl = _levels(levels)
    _check(load().qlora_codebook_dequantize(_ptr(codes), _ptr(absmax), n, lv, nl, _ptr(o),
                                            QLORA_F32 if dtype == torch.float32 else QLORA_BF16, _stream(stream)),
           "qlora_codebook_dequantize")
    return o


def codebook_stats_workspace_bytes(n: int) -> int:
    b = ctypes.c_size_t()
    _check(load().qlora_codebook_stats_workspace(n, ctypes.byref(b)), "qlora_codebook_stats_workspace")
    return b.value


def codebook_stats(w: torch.Tensor, codes: torch.Tensor, absmax: torch.Tensor, levels,
                   out: torch.Tensor | None = None, workspace: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """The CODEBOOK_STATS_LEN float64 values of qlora_codebook_stats, on the device."""
    _need(w, w.dtype, "w")
    n = w.numel()
    o = out if out is not None else torch.empty(CODEBOOK_STATS_LEN, dtype=torch.float64, device=w.device)
    _need(o, torch.float64, "out")
    ws = workspace if workspace is not None else torch.empty(codebook_stats_workspace_bytes(n), dtype=torch.uint8,
                                                             device=w.device)
    lv, nl = _levels(levels)
    _check(load().qlora_codebook_stats(_ptr(w), QLORA_F32 if w.dtype == torch.float32 else QLORA_BF16, _ptr(codes),
                                       _ptr(absmax), n, lv, nl, _ptr(o), _ptr(ws), ws.numel(), _stream(stream)),
           "qlora_codebook_stats")
    return o


def stats_dict(stats: torch.Tensor, nlevels: int) -> dict:
    """The fields of a qlora_codebook_stats result, copied to the host."""
    v = stats.detach().cpu().numpy()
    return {"counts": v[0:16].astype(np.int64), "sums": v[16:32].copy(), "sse": float(v[32]),
            "entropy_bits": float(v[33]), "rms": float(v[34]), "centroids": v[35:35 + nlevels].astype(np.float32)}


def lloyd(w: torch.Tensor, levels, iters: int, stream=None):
    """Lloyd's algorithm on the device: `iters` rounds of codebook_quantize + codebook_stats, each taking
    the kernel's updated levels. Returns the final levels (numpy fp32) and the RMS error before each step
    and after the last."""
    lv = np.asarray(levels, dtype=np.float32).copy()
    n = w.numel()
    codes = torch.empty(-(-n // 2), dtype=torch.uint8, device=w.device)
    absmax = torch.empty(-(-n // 64), dtype=torch.float32, device=w.device)
    ws = torch.empty(codebook_stats_workspace_bytes(n), dtype=torch.uint8, device=w.device)
    st = torch.empty(CODEBOOK_STATS_LEN, dtype=torch.float64, device=w.device)
    hist = []
    for k in range(iters + 1):
        codebook_quantize(w, lv, codes, absmax, stream)
        d = stats_dict(codebook_stats(w, codes, absmax, lv, st, ws, stream), lv.size)
        hist.append(d["rms"])
        if k < iters:
            lv = d["centroids"]
    return lv, hist


# ---- paged optimizer: AdamW step and managed-memory buffers ------------------------------------------

def adamw_step(p: torch.Tensor, g: torch.Tensor, m: torch.Tensor, v: torch.Tensor, step: int, lr: float,
               betas=(0.9, 0.999), eps: float = 1e-8, weight_decay: float = 0.0,
               p_bf16: torch.Tensor | None = None, stream=None) -> None:
    """qlora_adamw_step on contiguous fp32 CUDA tensors of equal size (device or managed memory)."""
    n = p.numel()
    for t, name in ((p, "p"), (g, "g"), (m, "m"), (v, "v")):
        if t.dtype != torch.float32 or not t.is_contiguous() or t.numel() != n:
            raise ValueError(f"adamw_step: {name} must be a contiguous float32 tensor of {n} elements")
    if p_bf16 is not None and (p_bf16.dtype != torch.bfloat16 or p_bf16.numel() != n or not p_bf16.is_contiguous()):
        raise ValueError("adamw_step: p_bf16 must be a contiguous bfloat16 tensor of the same size")
    _check(load().qlora_adamw_step(_ptr(p), _ptr(g), _ptr(m), _ptr(v), _ptr(p_bf16), n, int(step), lr, betas[0],
                                   betas[1], eps, weight_decay, _stream(stream)), "qlora_adamw_step")


class PagedBuffer:
    """Managed memory from qlora_paged_alloc, freed with qlora_paged_free when the last tensor viewing it
    goes away; exposes __cuda_array_interface__ so torch.as_tensor can wrap it without a copy."""

    def __init__(self, n: int, device=None):
        dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
        self.device = dev
        self.n = int(n)
        self.nbytes = 4 * self.n
        self.ptr = ctypes.c_void_p()
        with torch.cuda.device(dev):
            _check(load().qlora_paged_alloc(self.nbytes, ctypes.byref(self.ptr)), "qlora_paged_alloc")
        self.__cuda_array_interface__ = {"shape": (self.n,), "typestr": "<f4", "data": (self.ptr.value, False),
                                         "version": 3, "strides": None}

    def __del__(self):
        if getattr(self, "ptr", None) is not None and self.ptr.value:
            load().qlora_paged_free(self.ptr)
            self.ptr = ctypes.c_void_p()


def paged_empty(n: int, device=None) -> torch.Tensor:
    """An n-element float32 tensor in managed (unified) memory; uninitialised."""
    buf = PagedBuffer(n, device)
    with torch.cuda.device(buf.device):
        return torch.as_tensor(buf, device=buf.device)


def paged_prefetch(t: torch.Tensor, to_device: bool = True, stream=None) -> None:
    """Migrate a managed-memory tensor's pages to the GPU, or to host memory (an eviction)."""
    _check(load().qlora_paged_prefetch(_ptr(t), t.numel() * t.element_size(), 1 if to_device else 0, _stream(stream)),
           "qlora_paged_prefetch")


NOALLOC_MAX_NUMEL = 1 << 26


def quantize_noalloc(w: torch.Tensor, out: NF4Weight, stream=None) -> NF4Weight:
    """qlora_nf4_quantize_noalloc: like quantize() but with the library's fixed internal scratch instead
    of a workspace, for callers that cannot allocate device memory at the call (at most 2^26 elements;
    calls that overlap on the GPU race on the shared scratch). `out` must be preallocated."""
    if w.dtype not in (torch.float32, torch.bfloat16):
        raise ValueError("quantize_noalloc: w must be float32 or bfloat16")
    _need(w, w.dtype, "w")
    rows, cols = (w.shape[0], w.shape[1]) if w.dim() == 2 else (1, w.numel())
    st = out.struct()
    _check(load().qlora_nf4_quantize_noalloc(_ptr(w), QLORA_F32 if w.dtype == torch.float32 else QLORA_BF16,
                                             rows, cols, ctypes.byref(st), _stream(stream)),
           "qlora_nf4_quantize_noalloc")
    return out


def dequantize(q: NF4Weight, dtype=torch.bfloat16, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    if dtype not in (torch.float32, torch.bfloat16):
        raise ValueError("dequantize: dtype must be float32 or bfloat16")
    o = out if out is not None else torch.empty(q.rows, q.cols, dtype=dtype, device=q.codes.device)
    _need(o, dtype, "out")
    st = q.struct()
    _check(load().qlora_nf4_dequantize(ctypes.byref(st), _ptr(o), QLORA_F32 if dtype == torch.float32 else QLORA_BF16,
                                    _stream(stream)), "qlora_nf4_dequantize")
    return o


def linear_fwd(X: torch.Tensor, q: NF4Weight, A: torch.Tensor, B: torch.Tensor, alpha: float,
               save_u: bool = True, out: torch.Tensor | None = None, U_out: torch.Tensor | None = None,
               workspace: torch.Tensor | None = None, stream=None):
    """Y = X W~^T + (alpha/r) (X A^T) B^T.  Returns (Y, U) with U = (alpha/r) X A^T in bf16 (T x r) or None."""
    T, K = X.shape
    r = A.shape[0]
    for t, n in ((X, "X"), (A, "A"), (B, "B")):
        _need(t, torch.bfloat16, n)
    Y = out if out is not None else torch.empty(T, q.rows, dtype=torch.bfloat16, device=X.device)
    U = U_out if U_out is not None else (torch.empty(T, r, dtype=torch.bfloat16, device=X.device) if save_u else None)
    ws = workspace if workspace is not None else torch.empty(linear_workspace_bytes(T, q.rows, q.cols, r),
                                                             dtype=torch.uint8, device=X.device)
    st = q.struct()
    _check(load().qlora_linear_fwd(_ptr(X), T, ctypes.byref(st), _ptr(A), _ptr(B), r, float(alpha), _ptr(Y), _ptr(U),
                                _ptr(ws), ws.numel(), _stream(stream)), "qlora_linear_fwd")
    return Y, U


def linear_bwd(dY: torch.Tensor, X: torch.Tensor, q: NF4Weight, A: torch.Tensor, B: torch.Tensor, alpha: float,
               U: torch.Tensor | None = None, need_dx: bool = True, dX: torch.Tensor | None = None,
               dA: torch.Tensor | None = None, dB: torch.Tensor | None = None,
               workspace: torch.Tensor | None = None, stream=None):
    """(dX bf16 or None, dA fp32 r x K, dB fp32 N x r); the frozen NF4 weight gets no gradient."""
    T, K = X.shape
    r = A.shape[0]
    for t, n in ((dY, "dY"), (X, "X"), (A, "A"), (B, "B")):
        _need(t, torch.bfloat16, n)
    dev = X.device
    dXo = dX if dX is not None else (torch.empty(T, K, dtype=torch.bfloat16, device=dev) if need_dx else None)
    dAo = dA if dA is not None else torch.empty(r, K, dtype=torch.float32, device=dev)
    dBo = dB if dB is not None else torch.empty(q.rows, r, dtype=torch.float32, device=dev)
    ws = workspace if workspace is not None else torch.empty(linear_workspace_bytes(T, q.rows, q.cols, r),
                                                             dtype=torch.uint8, device=dev)
    st = q.struct()
    _check(load().qlora_linear_bwd(_ptr(dY), _ptr(X), T, ctypes.byref(st), _ptr(A), _ptr(B), r, float(alpha), _ptr(U),
                                _ptr(dXo), _ptr(dAo), _ptr(dBo), _ptr(ws), ws.numel(), _stream(stream)),
           "qlora_linear_bwd")
    return dXo, dAo, dBo


def get_status(stream=None) -> int:
    """Synchronize the stream and return (and clear) the device status bits (STATUS_*)."""
    v = ctypes.c_int()
    rc = load().qlora_get_status(ctypes.byref(v), _stream(stream))
    if rc not in (0, -6, -7):
        _check(rc, "qlora_get_status")
    return v.value


SELFTEST_MBARRIER, SELFTEST_DEVICE_WORD = 0, 1


def set_wait_limit(ns: int) -> None:
    """qlora_set_wait_limit: how long the kernels' bounded waits last on the current device (0: the
    default of 2 s). For tests of the timeout path."""
    _check(load().qlora_set_wait_limit(int(ns)), "qlora_set_wait_limit")


def selftest_wait(kind: int, stream=None) -> None:
    """qlora_selftest_wait: a kernel whose bounded wait must give up (see get_status)."""
    _check(load().qlora_selftest_wait(int(kind), _stream(stream)), "qlora_selftest_wait")


def kernel_launches() -> int:
    """Kernels launched by the library in this process so far."""
    return int(load().qlora_kernel_launches())


def profile_enable(on: bool = True) -> None:
    _check(load().qlora_profile_enable(1 if on else 0), "qlora_profile_enable")


def profile_read() -> dict:
    """{kernel class: (launches, total device ms)} since the last read; clears the record."""
    n = (ctypes.c_int64 * 5)()
    ms = (ctypes.c_double * 5)()
    _check(load().qlora_profile_read(n, ms), "qlora_profile_read")
    return {name: (int(n[i]), float(ms[i])) for i, name in enumerate(PROF_NAMES)}
