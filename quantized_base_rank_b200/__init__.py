"""B200-native (sm_100a) QLoRA-style quantised linear layer.

NF4 blockwise quantisation with double-quantised constants, a blockwise int8
alternative, and the fused forward/backward of Y = X W'^T + (alpha/r) (X A^T) B^T,
behind the C ABI declared in include/qlora.h. ``binding`` loads the built library
(libqlora_b200.so) on first use and fails loudly if it is missing.
"""
from . import binding  # noqa: F401  (the shared library itself loads lazily)

__all__ = ["binding"]
