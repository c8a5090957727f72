"""Oracle: a plain, slow, obviously-correct CPU statement of the QLoRA NF4 hot path.

THIS IS TEST INFRASTRUCTURE, NOT PART OF THE PRODUCT.  Only the tests, the smoke check and the
benchmark's CPU-baseline leg may import it.  The CUDA library never calls it and shares no code,
table or constant generator with it; the only thing both sides see is the seeded input generator
module (`synth`), which holds none of the method's arithmetic.

What it computes, in the pages' order (citations are to the source pages by title and section):

  codebook.py  the 16-level NF4 codebook and its decision thresholds
               [PEFT page, zerotofrontier.app/sft/peft, "NF4, derived from normal quantiles"]
  lowp.py      the number formats the codec rounds through: fp32 single roundings, the fused
               multiply-add, bf16 round-to-nearest-even, and the 8-bit float E4M3 (OCP FP8 spec)
  codec.py     blockwise absmax quantization with two codes per byte, the mean-subtracted double
               quantization of the block constants, and dequantization
               [PEFT page, "Block-wise quantization in one page", "Double quantization",
                "The real way"]
  codebook_study.py  the codebook comparison: any sorted codebook of up to 16 levels with fp32 block
               constants, code entropy and RMS error, and Lloyd's algorithm
               [PEFT page, "NF4, derived from normal quantiles"]
  adamw.py     the AdamW step whose states the paged optimizer keeps in unified memory
               [PEFT page, "Paged optimizers, and QLoRA end to end"]
  linear.py    the QLoRA linear layer, forward and backward, in fp64
               [QLoRA explainer, prism.theerrors.in, "Putting it together";
                PEFT page, "Paged optimizers, and QLoRA end to end"]

Floating point is fp64 except where a step is defined as a rounding to fp32, bf16 or E4M3; those
roundings are written out explicitly so that the CUDA path can be compared bit for bit.
Every choice the pages leave open is named where it is made ("Reading: ...").
"""
from .codebook import (OFFSET, normal_cdf, normal_ppf, nf4_levels_f64, nf4_codebook)
from .lowp import (rn32_add, rn32_sub, rn32_mul, rn32_div, fma32, bf16_rne_bits, bf16_bits_to_f32,
                   e4m3_decode, e4m3_encode, E4M3_MAX)
from .codec import (BLOCK, DQ_BLOCK, num_blocks, num_groups, storage_bytes, absmax_blocks,
                    nf4_codes, pack_codes, unpack_codes, pairwise_tree_sum, block_mean,
                    double_quantize, double_dequantize, quantize, dequantize, NF4Tensor,
                    quantize_single, dequantize_single, storage_bytes_single, NF4SingleTensor)
from .linear import linear_fwd, linear_bwd
from . import codebook_study
from .adamw import adamw_step

__all__ = [n for n in dir() if not n.startswith("_")]
