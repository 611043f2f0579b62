"""CSA / HCA hybrid-attention hot path for B200 (sm_100a).

The compute lives in ``csrc/`` (CUDA kernels behind a C ABI declared in
``include/csa.h``, built into ``libcsa.so``).  ``long_context_compressed_b200.csa``
is the thin ctypes binding with the same entry-point names; importing it loads
the library and fails loudly if it has not been built.
``long_context_compressed_b200.synth`` draws seeded synthetic inputs.
"""
