"""CPU oracle for the batch-invariant kernels -- TEST INFRASTRUCTURE ONLY.

Nothing on the product path may import, call or link anything in this
package: only the test suite, the smoke check and the CPU-baseline leg of the
benchmark use it. It shares no code, header, table or constant with the CUDA
library; its inputs come from the seeded generators in
``invariant_deterministic_03_b200.synth`` (which hold none of the method's
arithmetic), passed in as arrays.

Two independent views of every operation:

* :mod:`oracle.fp64`  -- the plain mathematical definition in float64
  (numpy; a library matmul serves as the matmul step).
* :mod:`oracle.ordered` -- the same operations in float32 with one fixed,
  written-out summation order (plain C in ``ordered.c``: sequential ``fmaf``
  accumulation), used to show order dependence and to time the CPU baseline.

bf16 tensors cross into the oracle as uint16 bit patterns or as float64
arrays that hold bf16 values exactly (:func:`oracle.fp64.bf16_bits_to_f64`).

:func:`oracle.fp64.forward_rounded` is the fp64 forward with each activation
stored in a narrower format (bf16, fp32, or an fp32 value as a bf16 hi/lo
pair) at named points, for the precision variants of the cross-vendor paper
(arXivDaily 2610.05458, abstract); it gives the expected size of a
mixed-precision forward's logit error from the storage roundings alone.

Parity status: every function of :mod:`oracle.fp64` is pinned by
``tests/test_oracle_pins.py`` against closed forms, exact rational
arithmetic, brute force or the worked examples printed in "Defeating
Nondeterminism in LLM Inference". ``forward`` is pinned structurally there
(causality, identity blocks, one-token closed form) and end to end by
``tests/test_oracle_forward_library.py`` against an independent library
implementation of the same architecture (the ``transformers`` Mistral model
in float64, same weights: agreement ~1e-6). The pages print no logits for
any model, so no pin reproduces a number of theirs for it.
``forward_rounded`` is pinned to ``forward`` (identical with no rounding),
by a liveness check of every storage point, and by the quadrature sum of
independent roundings. The fixed float32 order of :mod:`oracle.ordered`
(``gemm_f32``, ``rmsnorm_f32``, ``attention_f32``) is pinned bit for bit by
scalar emulations with one rounding per operation, each with planted
wrong orders that must not match.
"""
