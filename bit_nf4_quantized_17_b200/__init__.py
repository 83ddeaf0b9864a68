"""QLoRA linear layer on one B200: block-wise NF4 weights with double-quantised
scales, a bf16 LoRA branch, forward and backward, all in hand-written CUDA
kernels behind the C ABI of ``include/qlora.h`` (``libqlora.so``).

``qlora`` is the Python binding (argument marshalling only); ``workloads``
draws the seeded synthetic inputs; ``build`` compiles the library in-tree.
"""

from . import qlora  # noqa: F401  (fails loudly only when a call needs the library)
from .qlora import (  # noqa: F401
    QuantizedWeight, QloraError, qlora_quantize, qlora_dequantize, qlora_linear_fwd,
    qlora_linear_bwd, qlora_check, qlora_levels, qlora_nf4_sizes, qlora_linear_workspace,
    qlora_status_string,
)
