"""B200 (sm_100a) sparse-MLA decode library.

The compute path is the C-ABI shared library built from ``csrc/`` (see
``include/sparse_mla.h``).  ``sparse_mla_decode_05_b200.api`` is a thin
ctypes binding over it: argument marshalling only, no fallback.  Importing
this package does not load the library; ``api`` does, and fails loudly if
the library is missing.
"""

__all__ = ["inputs"]
