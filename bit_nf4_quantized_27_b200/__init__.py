"""NF4 frozen linear layer with a LoRA adapter, B200-native.

The compute lives in ``libqlora_nf4.so`` (hand-written sm_100a CUDA behind a C
ABI declared in ``include/qlora_nf4.h``).  ``binding`` marshals arguments to it
with ctypes; it loads the library on first use and raises if it is missing.
Importing this package loads nothing.
"""

__all__ = ["binding", "inputs"]
