"""Quantised top-k routed MoE FFN forward for B200 (sm_100a).

The compute lives in ``libqmoe.so`` (CUDA kernels behind a C ABI declared in
``include/qmoe.h``).  ``quantized_top_routed_b200.qmoe`` is the thin ctypes
binding with the same call names; ``synth`` makes seeded inputs.  Import the
submodules directly.
"""
