"""B200-native RNS-CKKS hot path: a C-ABI CUDA library (libckks_b200.so) plus a
thin Python binding.

    from rns_ckks_polynomial_b200 import Context, primes
    mods = primes(L + K)
    ctx = Context(mods[:L], mods[L:], alpha)
    ctx.ntt_fwd(x)            # x: int64 CUDA tensor [..., limbs, 2048]

The library is loaded on first use; if it is missing the call raises (there is
no CPU fallback).
"""
from .api import Context, primes  # noqa: F401

__all__ = ["Context", "primes"]
