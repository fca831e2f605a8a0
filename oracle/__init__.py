"""CPU oracle for the RNS-CKKS hot path.

TEST INFRASTRUCTURE ONLY.  The test suite, the package smoke check and the
CPU-baseline leg of ``bench.py`` are the only callers allowed.  The product
(the CUDA library and its binding under ``rns_ckks_polynomial_b200``) never
imports this package, and this package never imports the product.

The integer arithmetic lives in ``ckks_oracle.c`` (plain C, ``unsigned
__int128``, each operation written as its definition).  This module adds the
ctypes bindings and the parts of the scheme that need big integers or complex
numbers: the canonical-embedding encoder/decoder and CRT reconstruction.
``oracle.boot`` composes those operations into sin_fold and the whole
bootstrapping refresh.
"""
from .core import *  # noqa: F401,F403
from .encoding import *  # noqa: F401,F403
