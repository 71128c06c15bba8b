"""B200-native per-token dynamic quantization (DynamicQuant, AdaLayerNormQuant),
the PER_TOKEN / PER_GROUP dequantizers and the W8A8 product of the codes.

The product is the C-ABI library ``libdq.so`` (declared in ``include/dq.h``,
sources in ``csrc/``). ``token_dynamic_quantization_b200.dq`` is its thin
ctypes binding; importing it loads the library and fails loudly if it has not
been built (``python -m token_dynamic_quantization_b200.build``).
``workloads`` holds the seeded synthetic input generators and ``sharding``
the row split across ranks.
"""

__all__ = ["dq", "workloads", "build", "sharding"]
