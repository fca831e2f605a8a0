"""Shared test helpers: workload parameters, oracle-side scheme set-up.

Keys and ciphertexts for the parity tests come from the oracle (keygen and
encryption are host-side utilities, never part of the CUDA path); all random
draws come from the seeded generators in ``rns_ckks_polynomial_b200.synth``.
"""
from dataclasses import dataclass
from fractions import Fraction

import numpy as np

from rns_ckks_polynomial_b200 import synth

N = 2048
SLOTS = N // 2
SCALE = 2**60


@dataclass
class Params:
    L: int
    K: int
    alpha: int
    n: int = N

    @property
    def dnum(self):
        return (self.L + self.alpha - 1) // self.alpha


def u64(t):
    """torch int64 tensor / array -> numpy uint64 (same bits)."""
    a = t.numpy() if hasattr(t, "numpy") else np.asarray(t)
    return np.ascontiguousarray(a.astype(np.uint64))


def primes(orc, p: Params):
    allp = orc.gen_primes(p.n, p.L + p.K)
    return allp


class Scheme:
    """Oracle-side keys and encryptions for one parameter set."""

    def __init__(self, orc, p: Params, seed: int):
        self.orc, self.p, self.seed = orc, p, seed
        self.mods = primes(orc, p)
        self.q = self.mods[: p.L]
        self.s = synth.ternary(p.n, seed, 1).numpy()
        self._stream = 100

    def _next(self):
        self._stream += 1
        return self._stream

    def keygen_galois(self, g):
        p = self.p
        a = u64(synth.uniform_residues((p.dnum, p.L + p.K, p.n), self.mods, self.seed,
                                       self._next()))
        e = synth.gaussian((p.dnum, p.n), self.seed, self._next()).numpy()
        return self.orc.keygen_galois(self.s, g, a, e, self.mods, p.L, p.K, p.alpha)

    def keygen_relin(self):
        p = self.p
        a = u64(synth.uniform_residues((p.dnum, p.L + p.K, p.n), self.mods, self.seed,
                                       self._next()))
        e = synth.gaussian((p.dnum, p.n), self.seed, self._next()).numpy()
        return self.orc.keygen_relin(self.s, a, e, self.mods, p.L, p.K, p.alpha)

    def encrypt_slots(self, z, scale=SCALE):
        p = self.p
        m = self.orc.encode(np.asarray(z), p.n, scale)
        a = u64(synth.uniform_residues((p.L, p.n), self.q, self.seed, self._next()))
        e = synth.gaussian((p.n,), self.seed, self._next()).numpy()
        return self.orc.encrypt(m, self.s, a, e, self.q)

    def decrypt_slots(self, ct, scale=SCALE):
        L = ct.shape[-2]
        res = self.orc.decrypt(ct, self.s, self.mods[:L])
        return self.orc.decode(res, self.mods[:L], scale)

    def rescaled_scale(self, scale_in, level):
        """Scale after dividing by q_{level-1}."""
        return Fraction(scale_in) / int(self.mods[level - 1])


def galois_for_rotation(r, n=N):
    return pow(5, r, 2 * n)


def rot_left(z, r):
    return np.roll(np.asarray(z), -r)
