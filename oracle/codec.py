"""Blockwise NF4 quantization, double quantization of the block constants, and dequantization.

Test infrastructure (see the package docstring).

Sources:
  PEFT page (zerotofrontier.app/sft/peft)
    "Block-wise quantization in one page": split the tensor into blocks of b consecutive values, keep
      one constant per block, c = max |w_i|, divide by it and store the index of the nearest codebook
      level; to use a weight, look up its level and multiply back by c.
    "Double quantization": the fp32 block constants c1 are themselves data: subtract their mean,
      quantize them to 8-bit floats in blocks of 256, each block with its own fp32 constant c2.
      Overhead: 32/64 = 0.5 bits/param before, about 0.127 after; 4.127 bits (~0.516 B) per weight.
    "The real way": two 4-bit codes per byte.
  QLoRA explainer (prism.theerrors.in), "For the curious": first-level blocks of 64, second-level
    blocks of 256, 0.5 -> ~0.127 bits/param.

Readings where the pages leave a step open:
  R-tie   code(w, a) = number of thresholds T_j with w > T_j * a, in exact arithmetic (a > 0 is the
          block absmax).  This is "nearest level" except in the sub-ulp band between T_j and the true
          midpoint; an exact tie w = T_j * a goes to the lower index.  A block whose absmax is 0
          codes every element as 7 (the exact-zero level).
  R-pack  byte i holds element 2i in its high nibble and element 2i+1 in its low nibble; for odd n
          the last low nibble is 0.  Blocks are 64 consecutive elements of the flattened tensor; the
          last block may be partial and its absmax covers only the elements that exist.
  R-mean  one mean per tensor over all nb block constants: mu = RN32(S / nb), S the fp64 balanced
          pairwise sum of c1 zero-padded to L = max(256, next power of two >= nb) leaves (left subtree
          + right subtree, recursively; padding zeros are exact so S is unique), S / nb rounded to fp64
          and then to fp32.
  R-e4m3  "8-bit float" is E4M3.  Per group g of 256 constants: d_b = RN32(c1_b - mu),
          c2_g = max |d_b|, s2_g = RN32(c2_g / 448) so the group spans the full E4M3 range,
          e_b = E4M3_RNE_satfinite(RN32(d_b / s2_g)); e_b = 0 when s2_g = 0.  Stored: e (uint8 per
          block), s2 (fp32 per group) and mu (fp32).
  R-deq   c1_hat_b = fma(decode(e_b), s2_g, mu) with one rounding; w_hat = RN32(q[code] * c1_hat_b),
          then bf16 round-to-nearest-even for bf16 output.  No clamping of c1_hat.
  R-single the variant without double quantization (PEFT page, "Double quantization": the fp32 block
          constants as stored before the second level; "The real way" lists double quantization as an
          option): the same codes, the fp32 c1 stored per block (0.5 bits/param of overhead), and
          w_hat = RN32(q[code] * c1_b), bf16 round-to-nearest-even for bf16 output.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

from .codebook import nf4_codebook
from .lowp import (rn32_sub, rn32_div, rn32_mul, fma32, bf16_rne_bits, bf16_bits_to_f32,
                   e4m3_decode, e4m3_encode, E4M3_MAX)

BLOCK = 64
DQ_BLOCK = 256
_CHUNK = 1 << 22          # a multiple of BLOCK: chunks start on block boundaries


def num_blocks(n: int, block: int = BLOCK) -> int:
    return -(-n // block)


def num_groups(n: int, block: int = BLOCK, dq_block: int = DQ_BLOCK) -> int:
    return -(-num_blocks(n, block) // dq_block)


def storage_bytes(n: int) -> dict:
    """Bytes of each stored array of an n-element NF4 tensor with double-quantized constants."""
    nb, ng = num_blocks(n), num_groups(n)
    return dict(codes=-(-n // 2), absmax=nb, scale2=4 * ng, offset=4)


def as_f32_values(w) -> np.ndarray:
    """Flattened fp32 values of the input: fp32 as is, bf16 (given as uint16 bit patterns) widened."""
    w = np.asarray(w)
    if w.dtype == np.uint16:
        return bf16_bits_to_f32(w.reshape(-1))
    if w.dtype != np.float32:
        raise TypeError("input must be fp32 values or bf16 bit patterns (uint16)")
    return w.reshape(-1)


def absmax_blocks(w32: np.ndarray, block: int = BLOCK) -> np.ndarray:
    """c1_b = max |w_i| over block b (fp32, exact).  Raises on a non-finite element."""
    w32 = np.asarray(w32, dtype=np.float32).reshape(-1)
    if not np.all(np.isfinite(w32)):
        raise ValueError("non-finite input")
    n = w32.size
    nb = num_blocks(n, block)
    pad = np.zeros(nb * block, dtype=np.float32)
    pad[:n] = np.abs(w32)
    return pad.reshape(nb, block).max(axis=1)


def nf4_codes(w32: np.ndarray, c1: np.ndarray, thresholds: np.ndarray, block: int = BLOCK) -> np.ndarray:
    """Codes per reading R-tie: #{j : w > T_j * a} evaluated exactly (T_j * a is exact in fp64)."""
    w32 = np.asarray(w32, dtype=np.float32).reshape(-1)
    n = w32.size
    T64 = thresholds.astype(np.float64)
    out = np.empty(n, dtype=np.uint8)
    for s in range(0, n, _CHUNK):
        w = w32[s:s + _CHUNK].astype(np.float64)
        a = np.repeat(c1[s // block:(s + w.size + block - 1) // block].astype(np.float64), block)[:w.size]
        cnt = np.zeros(w.size, dtype=np.int64)
        for j in range(T64.size):
            cnt += w > T64[j] * a
        out[s:s + w.size] = np.where(a == 0.0, 7, cnt)
    return out


def pack_codes(codes: np.ndarray) -> np.ndarray:
    """Two codes per byte, even element in the high nibble (R-pack)."""
    c = np.asarray(codes, dtype=np.uint8)
    if c.size % 2:
        c = np.concatenate([c, np.zeros(1, np.uint8)])
    return ((c[0::2] << 4) | c[1::2]).astype(np.uint8)


def unpack_codes(packed: np.ndarray, n: int) -> np.ndarray:
    p = np.asarray(packed, dtype=np.uint8)
    c = np.empty(2 * p.size, dtype=np.uint8)
    c[0::2] = p >> 4
    c[1::2] = p & 0xF
    return c[:n]


def pairwise_tree_sum(x: np.ndarray) -> float:
    """Balanced pairwise sum in fp64 of a power-of-two-length vector: level by level, x[2i] + x[2i+1]."""
    v = np.asarray(x, dtype=np.float64)
    if v.size & (v.size - 1):
        raise ValueError("pairwise_tree_sum: length must be a power of two")
    while v.size > 1:
        v = v[0::2] + v[1::2]
    return float(v[0])


def block_mean(c1: np.ndarray) -> np.float32:
    """mu per reading R-mean."""
    nb = c1.size
    L = max(DQ_BLOCK, 1 << max(0, (nb - 1).bit_length()))
    pad = np.zeros(L, dtype=np.float64)
    pad[:nb] = c1.astype(np.float64)
    S = pairwise_tree_sum(pad)
    return np.float32(S / float(nb))


def double_quantize(c1: np.ndarray, block: int = DQ_BLOCK):
    """(e uint8[nb], s2 fp32[ng], mu fp32) per reading R-e4m3."""
    c1 = np.asarray(c1, dtype=np.float32)
    nb = c1.size
    ng = -(-nb // block)
    mu = block_mean(c1)
    d = rn32_sub(c1, mu)
    pad = np.zeros(ng * block, dtype=np.float32)
    pad[:nb] = np.abs(d)
    c2 = pad.reshape(ng, block).max(axis=1)
    s2 = rn32_div(c2, np.float32(E4M3_MAX))
    s2_b = np.repeat(s2, block)[:nb]
    safe = np.where(s2_b > 0, s2_b, np.float32(1.0))
    t = rn32_div(d, safe)
    e = np.where(s2_b > 0, e4m3_encode(t), np.uint8(0)).astype(np.uint8)
    return e, s2, mu


def double_dequantize(e: np.ndarray, s2: np.ndarray, mu, block: int = DQ_BLOCK) -> np.ndarray:
    """c1_hat_b = fma(decode(e_b), s2_g, mu), one rounding (R-deq)."""
    nb = np.asarray(e).size
    dec = e4m3_decode(e).astype(np.float32)          # every finite E4M3 value is an fp32 value
    s2_b = np.repeat(np.asarray(s2, np.float32), block)[:nb]
    return fma32(dec, s2_b, np.float32(mu))


@dataclass
class NF4Tensor:
    codes: np.ndarray        # uint8[ceil(n/2)]
    absmax_e4m3: np.ndarray  # uint8[nb]
    scale2: np.ndarray       # fp32[ng]
    offset: np.float32       # mu
    n: int
    shape: tuple


def quantize(w, shape=None) -> NF4Tensor:
    """NF4 + double quantization of a tensor given as fp32 values or bf16 bit patterns."""
    w32 = as_f32_values(w)
    q, T = nf4_codebook()
    c1 = absmax_blocks(w32)
    codes = nf4_codes(w32, c1, T)
    e, s2, mu = double_quantize(c1)
    shp = tuple(np.asarray(w).shape) if shape is None else tuple(shape)
    return NF4Tensor(pack_codes(codes), e, s2, np.float32(mu), int(w32.size), shp)


def dequantize(t: NF4Tensor, out: str = "bf16") -> np.ndarray:
    """w_hat per reading R-deq; bf16 output is returned as uint16 bit patterns, fp32 as fp32."""
    q, _ = nf4_codebook()
    c1_hat = double_dequantize(t.absmax_e4m3, t.scale2, t.offset)
    codes = unpack_codes(t.codes, t.n)
    w = np.empty(t.n, dtype=np.float32)
    for s in range(0, t.n, _CHUNK):            # _CHUNK is a multiple of BLOCK
        m = min(_CHUNK, t.n - s)
        c1_e = np.repeat(c1_hat[s // BLOCK:(s + m + BLOCK - 1) // BLOCK], BLOCK)[:m]
        w[s:s + m] = rn32_mul(q[codes[s:s + m]], c1_e)
    if out == "f32":
        return w.reshape(t.shape)
    if out == "bf16":
        return bf16_rne_bits(w).reshape(t.shape)
    raise ValueError(out)


# ---- the variant without double quantization (reading R-single) ------------------------------------

@dataclass
class NF4SingleTensor:
    codes: np.ndarray        # uint8[ceil(n/2)], as in NF4Tensor
    absmax: np.ndarray       # fp32[nb]: the block constants c1 themselves
    n: int
    shape: tuple


def quantize_single(w, shape=None) -> NF4SingleTensor:
    """NF4 codes with the fp32 block constants kept as they are (no second level)."""
    w32 = as_f32_values(w)
    _, T = nf4_codebook()
    c1 = absmax_blocks(w32)
    shp = tuple(np.asarray(w).shape) if shape is None else tuple(shape)
    return NF4SingleTensor(pack_codes(nf4_codes(w32, c1, T)), c1.astype(np.float32), int(w32.size), shp)


def dequantize_single(t: NF4SingleTensor, out: str = "bf16") -> np.ndarray:
    """w_hat = RN32(q[code] * c1_b); bf16 output as uint16 bit patterns, fp32 as fp32."""
    q, _ = nf4_codebook()
    codes = unpack_codes(t.codes, t.n)
    w = np.empty(t.n, dtype=np.float32)
    for s in range(0, t.n, _CHUNK):
        m = min(_CHUNK, t.n - s)
        c1_e = np.repeat(t.absmax[s // BLOCK:(s + m + BLOCK - 1) // BLOCK], BLOCK)[:m]
        w[s:s + m] = rn32_mul(q[codes[s:s + m]], c1_e)
    if out == "f32":
        return w.reshape(t.shape)
    if out == "bf16":
        return bf16_rne_bits(w).reshape(t.shape)
    raise ValueError(out)


def storage_bytes_single(n: int) -> dict:
    """Bytes of each stored array of an n-element NF4 tensor with fp32 block constants."""
    return {"codes": -(-n // 2), "absmax": 4 * num_blocks(n)}

