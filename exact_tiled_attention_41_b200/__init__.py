"""Exact tiled softmax attention for NVIDIA B200 (sm_100a).

The compute lives in ``lib/libfa.so`` (C ABI in ``include/fa.h``), built with
``python -m exact_tiled_attention_41_b200.build``.  ``abi`` binds it under the
C names; ``attention`` offers torch-tensor entry points.  Importing the package
does not load the library; the first call does, and fails loudly if it is
missing.
"""

__all__ = ["abi", "attention", "workloads"]
