"""Helpers for the GPU parity tests: contexts, host<->device conversion."""
import functools

import numpy as np
import pytest
import torch

from rns_ckks_polynomial_b200 import Context, synth

from .helpers import N, Params

gpu = pytest.mark.gpu


def need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def dev(a):
    """numpy uint64 -> CUDA int64 tensor (same bits)."""
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int64)).cuda()


def host(t):
    """CUDA int64 tensor -> numpy uint64."""
    return t.cpu().numpy().view(np.uint64)


@functools.lru_cache(maxsize=8)
def context(L, K, alpha):
    import oracle
    mods = [int(x) for x in oracle.gen_primes(N, L + K)]
    return Context(mods[:L], mods[L:], alpha)


def ctx_for(p: Params):
    return context(p.L, p.K, p.alpha)


def residues(shape, mods, seed, stream, device="cpu"):
    t = synth.uniform_residues(shape, mods, seed, stream, device=device)
    return t


def assert_bits_equal(got, want, what=""):
    got = np.asarray(got)
    want = np.asarray(want)
    assert got.shape == want.shape, (what, got.shape, want.shape)
    bad = np.nonzero(got != want)
    if bad[0].size:
        first = tuple(int(i[0]) for i in bad)
        raise AssertionError("%s: %d of %d words differ; first at %s: got %d want %d" % (
            what, bad[0].size, got.size, first, int(got[first]), int(want[first])))
