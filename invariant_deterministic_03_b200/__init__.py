"""Batch-invariant inference kernels for NVIDIA B200 (sm_100a).

The product is the C-ABI library ``libbi.so`` (declared in ``include/bi.h``);
``invariant_deterministic_03_b200.bi`` is its ctypes binding and
``invariant_deterministic_03_b200.synth`` the seeded synthetic inputs.
The binding is not imported here, so that the input generators can be used on
a machine where the library is not built.
"""
