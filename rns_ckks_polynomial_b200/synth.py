"""Seeded synthetic inputs, shared by the tests, the oracle calls and the bench.

This module only draws random numbers: it holds none of the scheme's
arithmetic (no transforms, no modular products, no prime search).  Every
draw is keyed by (seed, stream) so that each tensor of a workload has its own
reproducible stream, independent of how many threads or ranks consume it.

Distributions (the pages fix only the parameters; the distributions follow
the standard RNS-CKKS choices): uniform residues in [0, q) per limb, ternary
secret uniform over {-1, 0, 1}, rounded Gaussian error with sigma = 3.2
truncated at 6 sigma, uniform real slot values.
"""
import torch

SIGMA = 3.2


def config_seed(config_no: int) -> int:
    """Base seed of workload `config_no` (1-based)."""
    return 0xC0FFEE00 + int(config_no)


def _gen(seed: int, stream: int, device="cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed((int(seed) * 1_000_003 + int(stream) * 7_919 + 17) % (2**63 - 1))
    return g


def uniform_residues(shape, mods, seed, stream, device="cpu"):
    """int64 tensor of `shape` (..., limbs, n) with entry [..., l, k] uniform in
    [0, mods[l]).  `mods` is a sequence or tensor of `limbs` moduli < 2^62.
    The values are non-negative and < 2^62, so the int64 storage holds the
    same bits as the uint64 residues the library expects."""
    shape = tuple(int(s) for s in shape)
    g = _gen(seed, stream, device)
    q = torch.as_tensor([int(m) for m in mods], dtype=torch.int64, device=device)
    if q.numel() != shape[-2]:
        raise ValueError("mods must have one entry per limb")
    raw = torch.randint(0, 2**62, shape, generator=g, dtype=torch.int64, device=device)
    return torch.remainder(raw, q.view(*([1] * (len(shape) - 2)), -1, 1))


def uniform_below(shape, bound, seed, stream, device="cpu"):
    """int64 tensor uniform in [0, bound) (used where every limb's modulus
    exceeds `bound`)."""
    g = _gen(seed, stream, device)
    return torch.randint(0, int(bound), tuple(shape), generator=g, dtype=torch.int64,
                         device=device)


def ternary(n, seed, stream):
    """Secret coefficients uniform over {-1, 0, 1}; int64 [n]."""
    g = _gen(seed, stream)
    return torch.randint(-1, 2, (int(n),), generator=g, dtype=torch.int64)


def gaussian(shape, seed, stream, sigma=SIGMA):
    """Rounded Gaussian error, truncated at 6 sigma; int64."""
    g = _gen(seed, stream)
    v = torch.randn(tuple(shape), generator=g, dtype=torch.float64) * sigma
    v = torch.clamp(v, -6 * sigma, 6 * sigma)
    return torch.round(v).to(torch.int64)


def uniform_real(shape, lo, hi, seed, stream):
    """float64 uniform in [lo, hi)."""
    g = _gen(seed, stream)
    return torch.rand(tuple(shape), generator=g, dtype=torch.float64) * (hi - lo) + lo
