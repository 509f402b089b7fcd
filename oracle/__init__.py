"""CPU oracle for the routed-expert MoE layer and RAZOR Refill-RMS scoring.

TEST INFRASTRUCTURE ONLY.  This package is a plain, slow, obviously correct
restatement of what the method computes, written from the model cards and the
architecture fact sheet it cites.  Only ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline / reference legs of ``bench.py`` may import it.  It
shares no code with the CUDA library in ``bit_expert_gemm_b200`` and imports
nothing from it; the CUDA library never imports this package.

Floating point is float64 unless a step's precision is fixed by the format
(the NVFP4 quantiser takes its rounding decisions in float32, as the kernel
does, so that codes can be compared bit for bit).

Modules
-------
formats  BF16 / FP16 / FP8 E4M3 / FP4 E2M1 encoders and decoders.
moe      router, softmax + top-k + renormalisation, permutation, SwiGLU expert,
         combine, whole layer.
awq      AWQ W4A16 asymmetric group-32 pack / unpack / dequantise / quantise.
nvfp4    NVFP4 W4A4 group-16 quantise / dequantise.
razor    Refill-RMS score (literal definition and brute-force knock-out),
         additive accumulation, expert selection.

Parity status of each function is stated in its docstring; the pins live in
``tests/test_oracle_*.py``.
"""

from . import formats, moe, awq, nvfp4, razor  # noqa: F401
