"""QLoRA linear layer on one B200: block-wise NF4 weights with double-quantised
scales, a bf16 LoRA branch, forward and backward, all in hand-written CUDA
kernels behind the C ABI of ``include/qlora.h`` (``libqlora.so``).

Modules:
- ``qlora``: the Python binding (argument marshalling only). It covers quantise /
  dequantise, the linear forward and backward (also several adapters per batch
  and LoRA dropout), merge and unmerge, AdamW with paged states, and timing.
- ``dp``: data-parallel replicas (token shards, one flat gradient bucket, one
  all-reduce).
- ``optim``: ``AdapterAdamW``, the fp32 master weights and moments of one
  adapter pair, one kernel per step.
- ``workloads``: draws the seeded synthetic inputs.
- ``build``: compiles the library in-tree.
"""

from . import qlora  # noqa: F401  (fails loudly only when a call needs the library)
from .qlora import (  # noqa: F401
    QuantizedWeight, QloraError, qlora_quantize, qlora_dequantize, qlora_linear_fwd,
    qlora_linear_bwd, qlora_linear_fwd_multi, qlora_linear_bwd_multi, qlora_linear_fwd_ex,
    qlora_linear_bwd_ex, dropout_keep_mask, qlora_merge, qlora_merge_dense, qlora_adamw,
    qlora_paged_empty, qlora_paged_prefetch, qlora_check, qlora_levels, qlora_nf4_sizes,
    qlora_linear_workspace, qlora_status_string,
)
