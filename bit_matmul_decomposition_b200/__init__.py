"""LLM.int8() mixed-precision decomposed linear layer, native on B200 (sm_100a).

The compute lives in the CUDA library ``libi8linear.so`` built from ``csrc/``; the Python
side only marshals arguments (see ``abi.py``).  Importing the package does not load the
library: the first call does, and fails loudly when it is missing.
"""
__all__ = ["abi", "linear", "synth"]
