"""libtp: the Megatron-style partitioned Transformer layer on one B200.

The product is the C-ABI library libtp.so (include/libtp.h) built from
csrc/ for sm_100a; `binding` is its Python binding and `inputs` the seeded
synthetic input generators.  Importing this package loads nothing; the
first binding call loads libtp.so and fails loudly if it is not built.
"""
__all__ = ["binding", "inputs"]
