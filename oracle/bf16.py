"""bf16 <-> fp32 conversions for the oracle (test infrastructure only).

bf16 is the upper half of an IEEE fp32 word, so widening is a 16-bit shift
and narrowing is round-to-nearest-even on the dropped 16 bits.  The pages
name bf16 as the compute dtype ("LoRA 与 QLoRA：把大模型微调拆成可负担的
工程", section 8, bnb_4bit_compute_dtype=torch.bfloat16).
"""

import numpy as np


def bf16_bits_to_f32(bits):
    """uint16 bf16 bit patterns -> float32 values (exact)."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32)


def f32_to_bf16_bits(x):
    """float32 values -> uint16 bf16 bit patterns, round to nearest even.

    NaN stays a quiet NaN; infinities and overflow follow IEEE rounding.
    """
    x = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    u = x.view(np.uint32).astype(np.uint64)
    lsb = (u >> np.uint64(16)) & np.uint64(1)
    rounded = ((u + np.uint64(0x7FFF) + lsb) >> np.uint64(16)).astype(np.uint32)
    nan = np.isnan(x)
    rounded = np.where(nan, (u >> np.uint64(16)).astype(np.uint32) | np.uint32(0x40), rounded)
    return rounded.astype(np.uint16)


def round_to_bf16(x):
    """float32 -> nearest bf16 value, returned as float32."""
    return bf16_bits_to_f32(f32_to_bf16_bits(x))
