"""The seeded input generators: reproducible per (seed, stream), in range, with
the stated distributions.  Every parity test and the bench draw from these,
so a silent change here would change every workload."""
import math

import pytest
import torch

from rns_ckks_polynomial_b200 import primes, synth


def test_config_seeds_are_distinct():
    assert [synth.config_seed(c) for c in range(1, 6)] == [0xC0FFEE00 + c for c in range(1, 6)]


def test_uniform_residues_reproducible_and_in_range():
    q = primes(5)
    a = synth.uniform_residues((3, 5, 2048), q, 7, 1)
    b = synth.uniform_residues((3, 5, 2048), q, 7, 1)
    c = synth.uniform_residues((3, 5, 2048), q, 7, 2)
    assert a.dtype == torch.int64 and a.shape == (3, 5, 2048)
    assert torch.equal(a, b)
    assert not torch.equal(a, c)
    for l, m in enumerate(q):
        limb = a[:, l, :]
        assert int(limb.min()) >= 0 and int(limb.max()) < m
        # uniform over [0, q): the mean of 6144 draws lies within 5 standard errors of q / 2
        assert abs(float(limb.double().mean()) / m - 0.5) < 5 * math.sqrt(1 / 12 / limb.numel())
    with pytest.raises(ValueError):
        synth.uniform_residues((2, 4, 8), q, 7, 1)


def test_ternary_gaussian_and_real_distributions():
    s = synth.ternary(300000, 3, 1)
    counts = [int((s == v).sum()) for v in (-1, 0, 1)]
    assert sum(counts) == 300000
    assert all(abs(cnt / 300000 - 1 / 3) < 0.01 for cnt in counts)
    e = synth.gaussian((300000,), 3, 2)
    assert int(e.abs().max()) <= math.ceil(6 * synth.SIGMA)
    assert abs(float(e.double().std()) - synth.SIGMA) < 0.05
    assert abs(float(e.double().mean())) < 0.05
    z = synth.uniform_real((100000,), -1, 1, 3, 3)
    assert float(z.min()) >= -1 and float(z.max()) < 1
    assert abs(float(z.mean())) < 0.02
    assert torch.equal(synth.ternary(1000, 3, 1), synth.ternary(1000, 3, 1))
