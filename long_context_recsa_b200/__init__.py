"""RecSA (Recursive Sparse Attention) build -> select -> attend on B200 (sm_100a).

The compute path is librecsa.so (C ABI in include/recsa.h); ``long_context_recsa_b200.recsa``
is its Python binding and fails to import when the library has not been built
(``python -m long_context_recsa_b200.build``).  ``long_context_recsa_b200.inputs``
holds the seeded synthetic input generators.
"""
__all__ = ["recsa", "inputs", "build"]
