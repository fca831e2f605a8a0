"""The folded tensor-core basis conversion (ckks_ctx_set_conversion engine
"folded") against the CPU oracle, stage by stage, and against the other
engines on the full boot-level rotation.

The folded form computes the same exact sum as the integer pipes and the
byte-plane tensor-core form (the data's byte weights folded into the
conversion matrix modulo each target prime, then eight int8 plane products),
so every word must match the oracle's.
"""
import numpy as np
import pytest
import torch

from rns_ckks_polynomial_b200 import synth

from .gpu_common import assert_bits_equal, context, ctx_for, dev, host, need_gpu
from .helpers import N, Params, galois_for_rotation, u64

pytestmark = pytest.mark.gpu

SEED = synth.config_seed(1) + 7000


@pytest.fixture(autouse=True)
def _gpu():
    need_gpu()
    yield
    torch.cuda.synchronize()
    torch.cuda.empty_cache()


def _res(shape, mods, stream):
    return u64(synth.uniform_residues(shape, mods, SEED, stream))


def _top(mods, shape):
    """Every residue at q - 1 (the largest products and sums)."""
    return np.ascontiguousarray(np.broadcast_to((np.asarray(mods, dtype=np.uint64) - 1)[None, None, :, None],
                                                shape), dtype=np.uint64)


@pytest.mark.parametrize("L,K,alpha", [(4, 1, 1), (6, 2, 2), (5, 2, 2), (112, 8, 8), (20, 3, 7),
                                       (40, 20, 20), (70, 33, 33), (130, 64, 64), (120, 60, 60)])
def test_folded_stages_match_oracle(orc, L, K, alpha):
    """ModUp and ModDown with the folded conversion, bit-exact against the
    oracle on seeded residues (ragged last digits, 1 to 64 sources per
    conversion) and on all-(q - 1) inputs."""
    p = Params(L, K, alpha)
    ctx = ctx_for(p)
    mods = np.array(ctx.mods, dtype=np.uint64)
    c = _res((2, L, N), mods[:L], 50)
    c[1] = mods[:L, None] - 1
    key = _res((p.dnum, 2, L + K, N), mods, 51)
    acc_top = _top(mods, (1, 2, L + K, N))
    want_d = orc.modup(c, mods, L, K, alpha)
    want_a = orc.key_inner(want_d, key, 5, mods, L, K, alpha)
    want_m = orc.moddown(want_a, mods, L, K)
    want_top = orc.moddown(acc_top, mods, L, K)
    try:
        ctx.set_conversion("folded")
        dig = ctx.modup(dev(c))
        ctx.device_status()
        assert_bits_equal(host(dig), want_d, "modup (folded)")
        acc = ctx.key_inner(dig, dev(key), 5)
        assert_bits_equal(host(ctx.moddown(acc)), want_m, "moddown (folded)")
        assert_bits_equal(host(ctx.moddown(dev(acc_top))), want_top, "moddown all q-1 (folded)")
        ctx.device_status()
    finally:
        ctx.set_conversion("auto")


def test_folded_general_primes(orc):
    """Primes just above 2^59 (not of the 2^60 - delta form): the generic
    128-bit reduction in the folded epilogue."""
    from rns_ckks_polynomial_b200 import Context
    L, K, alpha = 12, 9, 9
    out, c = [], (1 << 59) + 1
    while len(out) < L + K:
        if orc.is_prime(c):
            out.append(c)
        c += 2 * N
    ctx = Context(out[:L], out[L:], alpha)
    try:
        mods = np.array(out, dtype=np.uint64)
        x = _res((2, L, N), mods[:L], 60)
        key = _res((2, 2, L + K, N), mods, 61)
        ctx.set_conversion("folded")
        assert_bits_equal(host(ctx.keyswitch(dev(x), dev(key))), orc.keyswitch(x, key, mods, L, K, alpha),
                          "keyswitch, general primes (folded)")
        ctx.device_status()
    finally:
        ctx.close()


def test_folded_boot_rotation_matches_other_engines(orc):
    """The boot-level rotation (2100 + 60 primes, alpha = 60, 4 keys, 8
    ciphertexts) with the folded conversion gives the same words as the
    byte-plane tensor-core engine, whose own parity with the oracle the
    config-5 test covers; ciphertext 2 under key 3 is also recomputed by the
    oracle."""
    p = Params(2100, 60, 60)
    ctx = ctx_for(p)
    seed = synth.config_seed(5)
    mods = np.array(ctx.mods, dtype=np.uint64)
    gal = [galois_for_rotation(k) for k in (1, 2, 4, 8)]
    ct = synth.uniform_residues((8, 2, 2100, N), mods[:2100], seed, 1, device="cuda")
    keys = [synth.uniform_residues((35, 2, 2160, N), mods, seed, 10 + r, device="cuda") for r in range(4)]
    try:
        ctx.set_conversion("tensor")
        ref = ctx.rotate(ct, keys, gal)
        ctx.set_conversion("folded")
        got = ctx.rotate(ct, keys, gal)
        ctx.device_status()
    finally:
        ctx.set_conversion("auto")
    assert torch.equal(got, ref)
    want = orc.rotate(host(ct[2:3]), [host(keys[3])], np.array([gal[3]], dtype=np.uint64), mods, 2100, 60, 60)
    assert_bits_equal(host(got[3, 2:3]), want[0], "folded boot rotation, ciphertext 2, key 3")


def test_folded_layer_and_bsgs_shapes(orc):
    """ct x ct with relinearisation and a BSGS transform at 112 + 8 primes,
    alpha = 8, through the folded conversion, bit-exact against the oracle."""
    p = Params(112, 8, 8)
    ctx = context(112, 8, 8)
    mods = np.array(ctx.mods, dtype=np.uint64)
    a, b = _res((2, 2, 112, N), mods[:112], 70), _res((2, 2, 112, N), mods[:112], 71)
    rlk = _res((p.dnum, 2, 120, N), mods, 72)
    x = _res((2, 2, 112, N), mods[:112], 73)
    diags = _res((3, 4, 112, N), mods[:112], 74)
    baby = [_res((p.dnum, 2, 120, N), mods, 75 + i) for i in range(3)]
    giant = [_res((p.dnum, 2, 120, N), mods, 80 + i) for i in range(2)]
    try:
        ctx.set_conversion("folded")
        got_m = host(ctx.mul_relin_rescale(dev(a), dev(b), dev(rlk)))
        got_b = host(ctx.bsgs_lintrans(dev(x), dev(diags), [dev(k) for k in baby], [dev(k) for k in giant], 4, 3))
        ctx.device_status()
    finally:
        ctx.set_conversion("auto")
    assert_bits_equal(got_m, orc.mul_relin_rescale(a, b, rlk, mods, 112, 8, 8), "mul_relin_rescale (folded)")
    assert_bits_equal(got_b, orc.bsgs(x, diags, baby, giant, 4, 3, mods, 112, 8, 8), "bsgs (folded)")
