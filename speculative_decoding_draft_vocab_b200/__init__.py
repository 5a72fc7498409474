"""Fused DSpark draft-training loss for NVIDIA B200 (sm_100a).

The product is the C-ABI library ``libdspark.so`` (declared in ``include/dspark.h``)
built from ``csrc/`` by ``build.py``.  ``abi`` is its ctypes binding (same entry-point
names) and ``torch_api`` marshals CUDA tensors into its structs; importing either
raises if the library has not been built.  ``synthetic`` draws the seeded inputs.
"""

__all__ = ["abi", "torch_api", "synthetic", "build"]
