"""CPU oracle for the QLoRA NF4 linear layer.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import this
package: only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg
of ``bench.py`` use it.  It shares no code, table, constant generator or
helper with the CUDA library under ``bit_nf4_quantized_17_b200/csrc``.

What it computes, and where the method is stated:

* ``nf4.py``   - the 16-level tables, block-wise absmax quantisation, the
  nearest-level index, 4-bit packing, double quantisation of the block
  scales and dequantisation ("QLoRA技术从入门到精通", section 3(1) and 3(2);
  "LoRA 与 QLoRA：用一块 GPU 微调大模型", section "量化" with its parts
  "分块缩放", "NF4", "存储和计算"; "QLoRA 量化微调", section 7.1).
* ``linear.py`` - the forward pass h = W x + (alpha/r) B A x and its
  backward pass dX, dA, dB with no gradient for W ("LoRA 与 QLoRA：把大模型
  微调拆成可负担的工程", section 2 and section 6; "QLoRA技术从入门到精通",
  section 3(2) and 3(3)).
  ``merge_weight`` is W_hat + (alpha/r) B A, the update merged into a
  restored 16-bit weight ("LoRA 与 QLoRA：把大模型微调拆成可负担的工程",
  section 3).
* ``optim.py`` - the AdamW step for the adapters (the optimiser that updates
  only A and B, "QLoRA技术从入门到精通", section 3(3)).
* ``multi.py`` - several adapters over one base, one per token ("LoRA 与
  QLoRA：把大模型微调拆成可负担的工程", section 3: shared base, one small pair
  per task).
* ``dropout.py`` - LoRA dropout on the adapter input, with the keep mask as an
  input ("LoRA 与 QLoRA：把大模型微调拆成可负担的工程", section 4.3).
* ``bf16.py``  - the bf16 <-> fp32 conversions; the products use the
  dequantised weight rounded to bf16 (``compute_weight``), the compute dtype
  the pages name.

Precision: the encoding steps are carried out in IEEE fp32 exactly as stated
in each function (numpy float32 arithmetic rounds to nearest even); the linear
algebra is carried out in fp64 with numpy matmul as the one library
primitive.

Every function here is pinned by ``tests/test_oracle_*.py`` against values
the pages print, closed forms, invariants, library routines (scipy's normal
quantile) or brute force.  No function is "parity unpinned".
"""

from .bf16 import bf16_bits_to_f32, f32_to_bf16_bits, round_to_bf16
from .nf4 import (
    nf4_levels,
    nf4_raw_quantiles,
    uniform_levels,
    nearest_level,
    block_absmax,
    pack_nibbles,
    unpack_nibbles,
    fixed_point_mean,
    double_quantize,
    dequantize_scales,
    block_scales,
    quantize,
    dequantize,
    compute_weight,
    storage_bits,
)
from .linear import lora_scale, linear_fwd, linear_bwd, lora_down, lora_grads, merge_weight
from .optim import adamw_step
from .multi import linear_fwd_multi, linear_bwd_multi
from .dropout import unpack_keep_mask, linear_fwd_dropout, linear_bwd_dropout

__all__ = [
    "bf16_bits_to_f32", "f32_to_bf16_bits", "round_to_bf16",
    "nf4_levels", "nf4_raw_quantiles", "uniform_levels", "nearest_level",
    "block_absmax", "pack_nibbles", "unpack_nibbles", "fixed_point_mean",
    "double_quantize", "dequantize_scales", "block_scales", "quantize", "dequantize", "compute_weight",
    "storage_bits", "lora_scale", "linear_fwd", "linear_bwd", "lora_down", "lora_grads", "merge_weight", "adamw_step",
    "linear_fwd_multi", "linear_bwd_multi", "unpack_keep_mask", "linear_fwd_dropout",
    "linear_bwd_dropout",
]
