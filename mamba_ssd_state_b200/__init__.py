"""DART layer hot path on B200 (sm_100a): SSD chunked scan with retained chunk
memories, state-memory attention with the gated residual, and the decode step.

The compute lives in ``libdart.so`` (CUDA, C ABI in ``include/dart.h``);
``dart`` is its Python binding and ``synth`` draws seeded synthetic inputs.
Importing the package does not load the library; the first call does.
"""
__all__ = ["dart", "synth", "build"]
