"""B200-native per-token dynamic quantization (DynamicQuant, AdaLayerNormQuant).

The product is the C-ABI library ``libdq.so`` (declared in ``include/dq.h``,
sources in ``csrc/``). ``token_dynamic_quantization_b200.dq`` is its thin
ctypes binding; importing it loads the library and fails loudly if it has not
been built (``python -m token_dynamic_quantization_b200.build``).
``workloads`` holds the seeded synthetic input generators.
"""

__all__ = ["dq", "workloads", "build"]
