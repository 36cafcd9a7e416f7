"""HLWQ Q5 (Hadamard-Lloyd Weight Quantization, 5-bit) for NVIDIA B200 (sm_100a).

The compute lives in libhlwq.so (C ABI, include/hlwq.h); ``dequant_matmul_b200.hlwq``
is its Python binding (importing it loads the library and fails if it is not
built).  ``dequant_matmul_b200.synth`` draws the seeded synthetic inputs.
"""

__version__ = "0.1.0"
