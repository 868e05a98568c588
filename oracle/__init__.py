"""CPU oracle for the FP8 W8A8 linear path — TEST INFRASTRUCTURE ONLY.

A plain, slow, obviously correct NumPy restatement of what the CUDA path
computes, used to check it.  Only the tests, the smoke check and the CPU
baseline leg of the benchmark may import this package; the product path never
does, and this package imports nothing from the product package.

Sources (two web pages describing the same method):
  [P1] "Quantized Inference for OneRec-V2：生成式推荐开始直接吃 LLM 量化栈",
       section 关键证据 — weights quantized offline per output channel,
       activations quantized per token at run time, FP8 tensor-core matmul
       with FP32 accumulation, output cast back to FP16.
  [P2] "FP8量化在生成式推荐系统OneRec-V2中的优化实践", §1.2 (FP8 range ±448),
       §2.2 (E4M3 format; per-token dynamic scale computed as
       max_code / max|x| with an eps floor), §2.3 (FP8 multiply + FP32
       accumulate + FP16 output).

Where the pages leave a step open the reading taken is stated beside the code
(rounding: round-to-nearest-even, saturating to ±448; eps = 1e-12; scale
stored as amax/448 and codes produced with one fp32 multiply by 448/amax).
Variants from [P2]: E5M2 activations (§2.2; max 57344, same steps),
per-tensor weight scales for the FFN linears (§2.1) and 128x128 block-wise
weight scales for the MoE experts (§2.1, §2.2).

Every function here is pinned by tests against closed forms, hand-worked
rows, a library cast routine and brute force; none is "parity unpinned".
"""
from .e4m3 import E4M3_MAX, e4m3_decode, e4m3_encode
from .e5m2 import E5M2_MAX, e5m2_decode, e5m2_encode
from .quant import EPS, quant_blocks, quant_rows, quant_tensor
from .linear import (linear_blockscaled_ref, linear_f64_unquantized, linear_ref, moe_blockscaled_ref, moe_combine_ref,
                     moe_gather_ref, moe_ref)

__all__ = ["E4M3_MAX", "e4m3_decode", "e4m3_encode", "E5M2_MAX", "e5m2_decode", "e5m2_encode",
           "EPS", "quant_rows", "quant_tensor", "quant_blocks", "linear_ref", "moe_ref",
           "linear_blockscaled_ref", "moe_blockscaled_ref", "moe_gather_ref", "moe_combine_ref",
           "linear_f64_unquantized"]
