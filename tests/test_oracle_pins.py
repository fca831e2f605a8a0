"""Pins of the CPU oracle against facts fixed outside it.

No page prints a test vector (no prime list, NTT output, key or ciphertext),
so each oracle function is pinned by closed forms, invariants, brute force on
small inputs and by decryption against float64 plaintext arithmetic.  Each
check is chosen so that a plausible slip (a wrong twiddle or index, a dropped
term, a sign, a transposed operand) fails at least one of them.
"""
import random

import numpy as np
import pytest

from rns_ckks_polynomial_b200 import synth

from .helpers import N, SCALE, SLOTS, Params, Scheme, galois_for_rotation, rot_left, u64

SEED = synth.config_seed(0)


# ------------------------------------------------------------------ helpers
def _sprp(m, a):
    """Strong probable-prime test to base a (independent of the oracle)."""
    d, s = m - 1, 0
    while d % 2 == 0:
        d //= 2
        s += 1
    x = pow(a, d, m)
    if x in (1, m - 1):
        return True
    for _ in range(s - 1):
        x = x * x % m
        if x == m - 1:
            return True
    return False


def _probably_prime(m):
    if m < 2:
        return False
    for p in (2, 3, 5, 7, 11, 13, 17, 19, 23, 29, 31, 37, 41, 43, 47):
        if m % p == 0:
            return m == p
    rng = random.Random(m)
    bases = [2, 3, 5, 7, 11, 13] + [rng.randrange(2, m - 1) for _ in range(16)]
    return all(_sprp(m, a) for a in bases)


def _brv(x, bits):
    return int(format(x, "0%db" % bits)[::-1], 2)


def _rand_res(shape, mods, stream):
    return u64(synth.uniform_residues(shape, mods, SEED, stream))


# ------------------------------------------------------------------ primes, psi
def test_primes_follow_the_scan_rule(orc):
    P = [int(x) for x in orc.gen_primes(N, 16)]
    # independent downward scan from 2^60 over candidates 1 mod 2n
    c = (2**60 - 1) // (2 * N) * (2 * N) + 1
    expect = []
    while len(expect) < 16:
        if _probably_prime(c):
            expect.append(c)
        c -= 2 * N
    assert P == expect
    for q in P:
        assert q % (2 * N) == 1 and 2**59 < q < 2**60
    assert P == sorted(P, reverse=True)


def test_first_prime_value(orc):
    # the largest prime below 2^60 that is 1 mod 4096
    q0 = int(orc.gen_primes(N, 1)[0])
    assert q0 == 1152921504606830593
    for c in range(q0 + 2 * N, 2**60, 2 * N):
        assert not _probably_prime(c)


def test_psi_is_smallest_primitive_root(orc):
    for q in [int(x) for x in orc.gen_primes(N, 3)]:
        psi = orc.find_psi(q, N)
        assert pow(psi, N, q) == q - 1
        assert pow(psi, 2 * N, q) == 1
        # independent root: first base g (from 3 upward) whose power has order 2n
        g = 3
        while True:
            x = pow(g, (q - 1) // (2 * N), q)
            if pow(x, N, q) == q - 1:
                break
            g += 1
        roots = [pow(x, k, q) for k in range(1, 2 * N, 2)]
        assert psi == min(roots)
    assert orc.find_psi(1152921504606830593, N) == 459811883340678


# ------------------------------------------------------------------ NTT
def test_ntt_of_monomials_is_the_evaluation_vector(orc):
    """NTT(1) = all ones and NTT(X) = (psi^(2 brv(k) + 1))_k: fixes the
    output ordering without using any code under test."""
    q = int(orc.gen_primes(N, 1)[0])
    psi = orc.find_psi(q, N)
    one = np.zeros(N, dtype=np.uint64)
    one[0] = 1
    x = np.zeros(N, dtype=np.uint64)
    x[1] = 1
    out = orc.ntt_fwd(np.stack([one, x])[:, None, :], [q])
    assert np.all(out[0, 0] == 1)
    bits = N.bit_length() - 1
    expect = [pow(psi, 2 * _brv(k, bits) + 1, q) for k in range(N)]
    assert [int(v) for v in out[1, 0]] == expect


def test_fast_ntt_equals_definition(orc):
    mods = orc.gen_primes(N, 3)
    a = _rand_res((3, N), mods, 1)
    fast = orc.ntt_fwd(a, mods)
    bits = N.bit_length() - 1
    for l, q in enumerate(mods):
        slow = orc.ntt_naive(a[l], q, N)
        assert np.array_equal(fast[l], slow)
        # a few outputs straight from the definition with Python integers
        psi, qq = orc.find_psi(q, N), int(q)
        coeffs = [int(v) for v in a[l]]
        for k in (0, 1, 7, 1000, N - 1):
            w = pow(psi, 2 * _brv(k, bits) + 1, qq)
            acc = 0
            for c in reversed(coeffs):
                acc = (acc * w + c) % qq
            assert int(fast[l, k]) == acc


def test_ntt_roundtrip_identity(orc):
    mods = orc.gen_primes(N, 3)
    x = _rand_res((2, 3, N), mods, 2)
    y = orc.ntt_fwd(x, mods)
    assert not np.array_equal(x, y)
    assert np.array_equal(orc.ntt_inv(y, mods), x)


def test_negacyclic_schoolbook_tiny(orc):
    """oracle schoolbook vs numpy full convolution folded by X^n = -1."""
    n = 16
    q = int(orc.gen_primes(n, 1)[0])
    rng = np.random.default_rng(3)
    a = rng.integers(0, 1000, n)
    b = rng.integers(0, 1000, n)
    full = np.convolve(a, b)
    fold = full[:n].copy()
    fold[: len(full) - n] -= full[n:]
    expect = [int(v) % q for v in fold]
    got = orc.negacyclic_mul(a.astype(np.uint64), b.astype(np.uint64), q)
    assert [int(v) for v in got] == expect


@pytest.mark.parametrize("n", [16, N])
def test_convolution_theorem(orc, n):
    q = orc.gen_primes(n, 1)
    a = _rand_res((1, n), q, 4)
    b = _rand_res((1, n), q, 5)
    prod = orc.ntt_inv(orc.pointwise("mul", orc.ntt_fwd(a, q), orc.ntt_fwd(b, q), q), q)
    assert np.array_equal(prod[0], orc.negacyclic_mul(a[0], b[0], q[0]))


def test_pointwise_sum_and_difference_by_linearity(orc):
    """The NTT is linear, so evaluation-domain sums and differences come back
    as coefficient sums and differences mod q, taken here with Python integers.
    Operands include 0 and q - 1 so both wrap directions are hit; a swapped
    operand in 'sub' flips every nonzero difference."""
    mods = orc.gen_primes(N, 3)
    a = _rand_res((2, 3, N), mods, 6)
    b = _rand_res((2, 3, N), mods, 7)
    for l, m in enumerate(mods):
        a[0, l, :4] = [0, int(m) - 1, 0, int(m) - 1]
        b[0, l, :4] = [0, int(m) - 1, int(m) - 1, 0]
    fa, fb = orc.ntt_fwd(a, mods), orc.ntt_fwd(b, mods)
    s = orc.ntt_inv(orc.pointwise("add", fa, fb, mods), mods)
    d = orc.ntt_inv(orc.pointwise("sub", fa, fb, mods), mods)
    for l, m in enumerate(int(v) for v in mods):
        for bi in range(2):
            av = [int(v) for v in a[bi, l]]
            bv = [int(v) for v in b[bi, l]]
            assert [int(v) for v in s[bi, l]] == [(x + y) % m for x, y in zip(av, bv)]
            assert [int(v) for v in d[bi, l]] == [(x - y) % m for x, y in zip(av, bv)]
    # directly in the evaluation domain: every output is a reduced residue
    for op in ("add", "sub", "mul"):
        r = orc.pointwise(op, fa, fb, mods)
        assert all(int(r[:, l].max()) < int(m) for l, m in enumerate(mods))


# ------------------------------------------------------------------ automorphism
def test_automorph_coeff_monomials(orc):
    q = int(orc.gen_primes(N, 1)[0])
    for j, g in [(1, 5), (500, 5), (3, 4095), (2047, 25)]:
        x = np.zeros(N, dtype=np.uint64)
        x[j] = 1
        out = orc.automorph_coeff(x, q, g)
        e = j * g % (2 * N)
        expect = np.zeros(N, dtype=np.uint64)
        if e < N:
            expect[e] = 1
        else:
            expect[e - N] = q - 1
        assert np.array_equal(out, expect)


@pytest.mark.parametrize("g", [5, 25, 625, 1505, 4095])
def test_automorph_ntt_permutation_matches_coefficients(orc, g):
    mods = orc.gen_primes(N, 2)
    x = _rand_res((2, N), mods, 6)
    via_ntt = orc.automorph_ntt(orc.ntt_fwd(x, mods), g)
    coef = np.stack([orc.automorph_coeff(x[l], mods[l], g) for l in range(2)])
    assert np.array_equal(via_ntt, orc.ntt_fwd(coef, mods))
    ginv = pow(g, -1, 2 * N)
    assert np.array_equal(orc.automorph_ntt(via_ntt, ginv), orc.ntt_fwd(x, mods))


# ------------------------------------------------------------------ encoding
def test_encode_constant_closed_form(orc):
    m = orc.encode(np.full(SLOTS, 0.25), N, SCALE)
    assert int(m[0]) == SCALE // 4
    assert np.all(m[1:] == 0)


def test_encode_decode_roundtrip_and_rotation(orc):
    mods = orc.gen_primes(N, 2)
    z = synth.uniform_real((SLOTS,), -1, 1, SEED, 7).numpy()
    m = orc.encode(z, N, SCALE)
    res = np.stack([np.array([int(v) % int(q) for v in m], dtype=np.uint64) for q in mods])
    back = orc.decode(res, mods, SCALE)
    assert np.max(np.abs(back - z)) < 1e-12
    # X -> X^5 rotates slots left by one; X -> X^(5^3) by three
    for r in (1, 3):
        g = galois_for_rotation(r)
        rot = np.stack([orc.automorph_coeff(res[l], mods[l], g) for l in range(2)])
        assert np.max(np.abs(orc.decode(rot, mods, SCALE) - rot_left(z, r))) < 1e-12
    # conjugation (g = -1): complex conjugate of every slot
    zc = z + 1j * synth.uniform_real((SLOTS,), -1, 1, SEED, 8).numpy()
    mc = orc.encode(zc, N, SCALE)
    rc = np.stack([np.array([int(v) % int(q) for v in mc], dtype=np.uint64) for q in mods])
    conj = np.stack([orc.automorph_coeff(rc[l], mods[l], 2 * N - 1) for l in range(2)])
    assert np.max(np.abs(orc.decode(conj, mods, SCALE) - np.conj(zc))) < 1e-12


def test_encoding_is_multiplicative(orc):
    mods = orc.gen_primes(N, 3)
    z1 = synth.uniform_real((SLOTS,), -1, 1, SEED, 9).numpy()
    z2 = synth.uniform_real((SLOTS,), -1, 1, SEED, 10).numpy()
    m1, m2 = orc.encode(z1, N, SCALE), orc.encode(z2, N, SCALE)
    r1 = np.stack([np.array([int(v) % int(q) for v in m1], dtype=np.uint64) for q in mods])
    r2 = np.stack([np.array([int(v) % int(q) for v in m2], dtype=np.uint64) for q in mods])
    prod = np.stack([orc.negacyclic_mul(r1[l], r2[l], mods[l]) for l in range(3)])
    assert np.max(np.abs(orc.decode(prod, mods, SCALE * SCALE) - z1 * z2)) < 1e-12


def test_batch_encoder_matches_encode_and_decodes(orc):
    """encode_many (one long-double matrix product) against encode() row by
    row, within one unit per coefficient, on real and complex slots; the
    residues of encode_ntt_many decode back to the slots; a constant row
    gives the closed form (c scale, 0, ..., 0)."""
    mods = orc.gen_primes(N, 2)
    Z = np.stack([synth.uniform_real((SLOTS,), -1, 1, SEED, 60 + i).numpy() / 32 for i in range(3)])
    Zc = Z + 1j * np.stack([synth.uniform_real((SLOTS,), -1, 1, SEED, 70 + i).numpy() for i in range(3)])
    for rows, scale in ((Z, SCALE), (Zc, 2**40)):
        many = orc.encode_many(rows, N, scale)
        for i in range(rows.shape[0]):
            assert np.max(np.abs(many[i] - orc.encode(rows[i], N, scale))) <= 1
    nt = orc.encode_ntt_many(Zc, mods, 2**40, N)
    for i in range(Zc.shape[0]):
        back = orc.decode(orc.ntt_inv(nt[i], mods), mods, 2**40)
        assert np.max(np.abs(back - Zc[i])) < 1e-9
    const = orc.encode_many(np.full((1, SLOTS), 0.25), N, SCALE)[0]
    assert int(const[0]) == SCALE // 4 and np.all(const[1:] == 0)


# ------------------------------------------------------------------ basis conversion
def test_basis_conversion_crt_identity(orc):
    mods = [int(x) for x in orc.gen_primes(N, 8)]
    src, dst = mods[:3], mods[3:]
    S = 1
    for q in src:
        S *= q
    rng = random.Random(11)
    n = 64
    X = [rng.randrange(S) for _ in range(n)] + [0, S - 1]
    n = len(X)
    x = np.array([[v % q for v in X] for q in src], dtype=np.uint64)
    out = orc.basis_convert(x, np.array(src, dtype=np.uint64), np.array(dst, dtype=np.uint64))
    for k in range(n):
        t0 = dst[0]
        u = (int(out[0, k]) - X[k]) * pow(S, -1, t0) % t0
        assert 0 <= u < len(src)
        for t_i, t in enumerate(dst):
            assert int(out[t_i, k]) == (X[k] + u * S) % t


def _crt(res_cols, mods):
    Q = 1
    for q in mods:
        Q *= q
    x = 0
    for r, q in zip(res_cols, mods):
        qh = Q // q
        x += int(r) * qh * pow(qh % q, -1, q)
    return x % Q, Q


@pytest.mark.parametrize("L,K,alpha", [(6, 2, 2), (5, 2, 2), (4, 1, 1), (7, 2, 3), (1, 1, 1),
                                       (1, 3, 1)])
def test_modup_crt_identity(orc, L, K, alpha):
    """Including the single-prime chain L = 1 (the level a refresh starts
    from) and a ragged last digit (7 = 3 + 3 + 1)."""
    p = Params(L, K, alpha)
    mods = [int(x) for x in orc.gen_primes(N, L + K)]
    m64 = np.array(mods, dtype=np.uint64)
    c = _rand_res((1, L, N), m64[:L], 12)
    dig = orc.modup(c, m64, L, K, alpha)
    assert dig.shape == (1, p.dnum, L + K, N)
    coef_in = orc.ntt_inv(c[0], m64[:L])
    for j in range(p.dnum):
        lo, hi = j * alpha, min(L, (j + 1) * alpha)
        assert np.array_equal(dig[0, j, lo:hi], c[0, lo:hi])
        coef = orc.ntt_inv(dig[0, j], m64)
        for k in (0, 5, N - 1):
            X, Qj = _crt([coef_in[i, k] for i in range(lo, hi)], mods[lo:hi])
            tgt = [t for t in range(L + K) if not lo <= t < hi]
            t0 = mods[tgt[0]]
            u = (int(coef[tgt[0], k]) - X) * pow(Qj, -1, t0) % t0
            assert 0 <= u < hi - lo
            for t in tgt:
                assert int(coef[t, k]) == (X + u * Qj) % mods[t]


@pytest.mark.parametrize("L,K", [(4, 2), (1, 1), (1, 3), (3, 1)])
def test_moddown_floor_identity(orc, L, K):
    mods = [int(x) for x in orc.gen_primes(N, L + K)]
    m64 = np.array(mods, dtype=np.uint64)
    acc_coef = _rand_res((1, 2, L + K, N), m64, 13)
    acc = orc.ntt_fwd(acc_coef, m64)
    out = orc.moddown(acc, m64, L, K)
    out_coef = orc.ntt_inv(out, m64[:L])
    P = 1
    for q in mods[L:]:
        P *= q
    for c in range(2):
        for k in (0, 9, N - 1):
            X, _ = _crt([acc_coef[0, c, t, k] for t in range(L + K)], mods)
            F = X // P
            v = (F - int(out_coef[0, c, 0, k])) % mods[0]
            assert 0 <= v < K
            for i in range(L):
                assert int(out_coef[0, c, i, k]) == (F - v) % mods[i]


def test_rescale_is_exact_floor(orc):
    lp1 = 5
    mods = [int(x) for x in orc.gen_primes(N, lp1)]
    m64 = np.array(mods, dtype=np.uint64)
    coef = _rand_res((1, 2, lp1, N), m64, 14)
    out = orc.rescale(orc.ntt_fwd(coef, m64), m64)
    out_coef = orc.ntt_inv(out, m64[: lp1 - 1])
    for c in range(2):
        for k in (0, 3, N - 1):
            C, _ = _crt([coef[0, c, i, k] for i in range(lp1)], mods)
            F = C // mods[-1]
            for i in range(lp1 - 1):
                assert int(out_coef[0, c, i, k]) == F % mods[i]


# ------------------------------------------------------------------ scheme level
def test_rotation_decrypts_to_slot_rotation_config1(orc):
    """Tiny RNS-CKKS parameters: 4 ciphertext primes, 1 special, alpha = 1."""
    sch = Scheme(orc, Params(4, 1, 1), SEED + 1)
    z = synth.uniform_real((SLOTS,), -1, 1, SEED, 20).numpy()
    ct = sch.encrypt_slots(z)
    assert np.max(np.abs(sch.decrypt_slots(ct) - z)) < 1e-8
    key = sch.keygen_galois(5)
    out = orc.rotate(ct[None], [key], np.array([5], dtype=np.uint64), sch.mods, 4, 1, 1)
    err = np.max(np.abs(sch.decrypt_slots(out[0, 0]) - rot_left(z, 1)))
    assert err < 1e-8


@pytest.mark.parametrize("K", [1, 2])
def test_rotation_on_a_single_prime_chain(orc, K):
    """L = 1, the level a refresh starts from: one digit, K special primes,
    the message at scale 2^40 below q_0.  Rotation by 3 and conjugation
    decrypt to the rotated and conjugated slots."""
    scale = 2**40
    sch = Scheme(orc, Params(1, K, 1), SEED + 12 + K)
    z = synth.uniform_real((SLOTS,), -1, 1, SEED, 25).numpy() + \
        1j * synth.uniform_real((SLOTS,), -1, 1, SEED, 26).numpy()
    ct = sch.encrypt_slots(z, scale)
    gal = [galois_for_rotation(3), 2 * N - 1]
    keys = [sch.keygen_galois(g) for g in gal]
    out = orc.rotate(ct[None], keys, np.array(gal, dtype=np.uint64), sch.mods, 1, K, 1)
    assert np.max(np.abs(sch.decrypt_slots(out[0, 0], scale) - rot_left(z, 3))) < 1e-6
    assert np.max(np.abs(sch.decrypt_slots(out[1, 0], scale) - np.conj(z))) < 1e-6


def test_rotation_at_the_boot_chain_size(orc):
    """The boot chain itself: 2100 ciphertext primes, 60 special, 35 digits of
    60 (about 20 s).  Rotation by 8 with config 5's Galois element 1505 = 5^8
    decrypts to the rotated slots; the decryption reads q_0..q_2 only, where
    m + e is far below Q/2."""
    assert galois_for_rotation(8) == 1505
    p = Params(2100, 60, 60)
    sch = Scheme(orc, p, SEED + 15)
    z = synth.uniform_real((SLOTS,), -1, 1, SEED, 27).numpy()
    ct = sch.encrypt_slots(z)
    key = sch.keygen_galois(1505)
    out = orc.rotate(ct[None], [key], np.array([1505], dtype=np.uint64), sch.mods, 2100, 60, 60)
    assert out.shape == (1, 1, 2, 2100, N)
    low = np.ascontiguousarray(out[0, 0][:, :3])
    assert np.max(np.abs(sch.decrypt_slots(low) - rot_left(z, 8))) < 1e-8


def test_hoisted_rotations_small_digits(orc):
    """Ragged digits (L = 5, alpha = 2) and several keys on one ModUp."""
    p = Params(5, 2, 2)
    sch = Scheme(orc, p, SEED + 2)
    z = synth.uniform_real((SLOTS,), -1, 1, SEED, 21).numpy()
    ct = sch.encrypt_slots(z)
    rs = [1, 2, 7]
    keys = [sch.keygen_galois(galois_for_rotation(r)) for r in rs]
    gal = np.array([galois_for_rotation(r) for r in rs], dtype=np.uint64)
    out = orc.rotate(ct[None], keys, gal, sch.mods, p.L, p.K, p.alpha)
    for i, r in enumerate(rs):
        assert np.max(np.abs(sch.decrypt_slots(out[i, 0]) - rot_left(z, r))) < 1e-8


def test_unhoisted_rotation_order_decrypts_and_differs_in_low_bits(orc):
    """The automorphism-first order (no hoisting) decrypts to the same slot rotation as the hoisted
    order, with different low bits (the approximate ModUp does not commute with phi_g)."""
    p = Params(5, 2, 2)
    sch = Scheme(orc, p, SEED + 5)
    z = synth.uniform_real((SLOTS,), -1, 1, SEED, 23).numpy()
    ct = sch.encrypt_slots(z)
    rs = [1, 3]
    keys = [sch.keygen_galois(galois_for_rotation(r)) for r in rs]
    gal = np.array([galois_for_rotation(r) for r in rs], dtype=np.uint64)
    a = orc.rotate_unhoisted(ct[None], keys, gal, sch.mods, p.L, p.K, p.alpha)
    h = orc.rotate(ct[None], keys, gal, sch.mods, p.L, p.K, p.alpha)
    for i, r in enumerate(rs):
        assert np.max(np.abs(sch.decrypt_slots(a[i, 0]) - rot_left(z, r))) < 1e-8
    assert not np.array_equal(a, h)
    # with g = 1 there is no automorphism, so the two orders coincide
    k1 = sch.keygen_galois(1)
    one = np.array([1], dtype=np.uint64)
    assert np.array_equal(orc.rotate_unhoisted(ct[None], [k1], one, sch.mods, p.L, p.K, p.alpha),
                          orc.rotate(ct[None], [k1], one, sch.mods, p.L, p.K, p.alpha))


@pytest.mark.slow
def test_rotation_and_relin_config3_params(orc):
    """Layer-shaped parameters: 112 primes, alpha = 8, 8 special primes."""
    p = Params(112, 8, 8)
    sch = Scheme(orc, p, SEED + 3)
    za = synth.uniform_real((SLOTS,), -1, 1, SEED, 30).numpy()
    zb = synth.uniform_real((SLOTS,), -1, 1, SEED, 31).numpy()
    ca, cb = sch.encrypt_slots(za), sch.encrypt_slots(zb)
    g = galois_for_rotation(2)
    key = sch.keygen_galois(g)
    out = orc.rotate(ca[None], [key], np.array([g], dtype=np.uint64), sch.mods, 112, 8, 8)
    assert np.max(np.abs(sch.decrypt_slots(out[0, 0]) - rot_left(za, 2))) < 1e-8
    rlk = sch.keygen_relin()
    prod = orc.mul_relin_rescale(ca[None], cb[None], rlk, sch.mods, 112, 8, 8)
    assert prod.shape == (1, 2, 111, N)
    sc = sch.rescaled_scale(SCALE * SCALE, 112)
    assert np.max(np.abs(sch.decrypt_slots(prod[0], sc) - za * zb)) < 1e-8


def test_relin_small(orc):
    p = Params(6, 2, 2)
    sch = Scheme(orc, p, SEED + 4)
    za = synth.uniform_real((SLOTS,), -1, 1, SEED, 40).numpy()
    zb = synth.uniform_real((SLOTS,), -1, 1, SEED, 41).numpy()
    ca, cb = sch.encrypt_slots(za), sch.encrypt_slots(zb)
    rlk = sch.keygen_relin()
    prod = orc.mul_relin_rescale(ca[None], cb[None], rlk, sch.mods, p.L, p.K, p.alpha)
    sc = sch.rescaled_scale(SCALE * SCALE, p.L)
    assert np.max(np.abs(sch.decrypt_slots(prod[0], sc) - za * zb)) < 1e-8


def bsgs_plaintexts(orc, M, bb, gg, mods, scale=SCALE):
    """pt_{g,b} = Encode(rot_{-bb g}(diag_{bb g + b})), diag_k[i] = M[i][(i+k) mod S]."""
    S = M.shape[0]
    idx = np.arange(S)
    out = []
    for g in range(gg):
        row = []
        for b in range(bb):
            k = bb * g + b
            diag = M[idx, (idx + k) % S]
            row.append(orc.encode_ntt(np.roll(diag, bb * g), mods, scale, N))
        out.append(np.stack(row))
    return np.stack(out)


def test_bsgs_banded_matvec(orc):
    """bb = gg = 4 over a matrix with 16 nonzero diagonals: decrypts to M x."""
    p = Params(6, 2, 2)
    bb = gg = 4
    sch = Scheme(orc, p, SEED + 5)
    rng_m = synth.uniform_real((SLOTS, SLOTS), -1 / 32, 1 / 32, SEED, 50).numpy()
    idx = np.arange(SLOTS)
    M = np.zeros((SLOTS, SLOTS))
    for k in range(bb * gg):
        M[idx, (idx + k) % SLOTS] = rng_m[idx, (idx + k) % SLOTS]
    x = synth.uniform_real((SLOTS,), -1, 1, SEED, 51).numpy()
    ct = sch.encrypt_slots(x)
    diags = bsgs_plaintexts(orc, M, bb, gg, sch.q)
    baby = [sch.keygen_galois(galois_for_rotation(b)) for b in range(1, bb)]
    giant = [sch.keygen_galois(galois_for_rotation(bb * g)) for g in range(1, gg)]
    y = orc.bsgs(ct[None], diags, baby, giant, bb, gg, sch.mods, p.L, p.K, p.alpha)
    sc = sch.rescaled_scale(SCALE * SCALE, p.L)
    assert np.max(np.abs(sch.decrypt_slots(y[0], sc) - M @ x)) < 1e-8


def test_bsgs_at_the_layer_chain_size(orc):
    """Config 4's shape: 112 + 8 primes, bb = gg = 32, 31 baby and 31 giant
    keys.  M has nonzero diagonals at offsets spread over the
    32 x 32 (giant, baby) grid, including both ends and both sides of a giant
    boundary; absent diagonals are zero plaintexts.  Decrypts (through
    q_0..q_2) to M x."""
    p = Params(112, 8, 8)
    bb = gg = 32
    sch = Scheme(orc, p, SEED + 16)
    offs = [0, 1, 31, 32, 33, 100, 511, 1000, 1023]
    vals = synth.uniform_real((len(offs), SLOTS), -1 / 8, 1 / 8, SEED, 60).numpy()
    idx = np.arange(SLOTS)
    M = np.zeros((SLOTS, SLOTS))
    diags = np.zeros((gg, bb, p.L, N), dtype=np.uint64)
    for v, k in zip(vals, offs):
        M[idx, (idx + k) % SLOTS] = v
        g, b = divmod(k, bb)
        diags[g, b] = orc.encode_ntt(np.roll(v, bb * g), sch.q, SCALE, N)
    baby = [sch.keygen_galois(galois_for_rotation(b)) for b in range(1, bb)]
    giant = [sch.keygen_galois(galois_for_rotation(bb * g)) for g in range(1, gg)]
    x = synth.uniform_real((SLOTS,), -1, 1, SEED, 61).numpy()
    y = orc.bsgs(sch.encrypt_slots(x)[None], diags, baby, giant, bb, gg, sch.mods, p.L, p.K, p.alpha)
    sc = sch.rescaled_scale(SCALE * SCALE, p.L)
    low = np.ascontiguousarray(y[0][:, :3])
    assert np.max(np.abs(sch.decrypt_slots(low, sc) - M @ x)) < 1e-8


def test_every_input_is_read(orc):
    """Flipping one residue of any input changes the output, for every
    oracle operation and every one of its inputs (an operation that ignored
    an input, or part of it, would pass tests whose inputs happen not to
    matter)."""
    p = Params(6, 2, 2)
    L, K, alpha = p.L, p.K, p.alpha
    mods = orc.gen_primes(N, L + K)
    q = mods[:L]

    def flip(a, at, m):
        b = a.copy()
        b[at] = (int(b[at]) + 1) % int(m)
        return b

    def check(fn, args, idx, at, m):
        base = fn(*args)
        args2 = list(args)
        args2[idx] = flip(args[idx], at, m)
        got = fn(*args2)
        base = base if isinstance(base, tuple) else (base,)
        got = got if isinstance(got, tuple) else (got,)
        assert any(not np.array_equal(x, y) for x, y in zip(base, got)), (fn.__name__, idx, at)

    a, b = _rand_res((2, L, N), q, 70), _rand_res((2, L, N), q, 71)
    key, key2 = _rand_res((p.dnum, 2, L + K, N), mods, 72), _rand_res((p.dnum, 2, L + K, N), mods, 73)
    ct = _rand_res((1, 2, L, N), q, 74)
    gal = np.array([5], dtype=np.uint64)
    check(lambda x: orc.ntt_fwd(x, q), [a], 0, (1, 5, 7), q[5])
    check(lambda x: orc.ntt_inv(x, q), [a], 0, (0, 0, N - 1), q[0])
    for i in range(2):
        check(lambda x, y: orc.pointwise("mul", x, y, q), [a, b], i, (1, 3, 9), q[3])
    check(lambda x: orc.automorph_ntt(x, 5), [a], 0, (0, 2, 100), q[2])
    check(lambda x: orc.modup(x, mods, L, K, alpha), [a], 0, (1, 5, 11), q[5])
    dig = orc.modup(a, mods, L, K, alpha)
    check(lambda d, k: orc.key_inner(d, k, 5, mods, L, K, alpha), [dig, key], 0, (0, 2, L + 1, 3),
          mods[L + 1])
    check(lambda d, k: orc.key_inner(d, k, 5, mods, L, K, alpha), [dig, key], 1, (1, 1, 4, 8), mods[4])
    acc = orc.key_inner(dig, key, 1, mods, L, K, alpha)
    check(lambda x: orc.moddown(x, mods, L, K), [acc], 0, (0, 1, L, 17), mods[L])
    check(lambda x: orc.moddown(x, mods, L, K), [acc], 0, (1, 0, 2, 17), mods[2])
    for idx, at, m in ((0, (0, 4, 5), q[4]), (1, (2, 0, L + 1, 6), mods[L + 1])):
        check(lambda d, k: orc.keyswitch(d, k, mods, L, K, alpha), [a, key], idx, at, m)
    for fn in (orc.rotate, orc.rotate_unhoisted):
        for at in ((0, 0, 1, 4), (0, 1, 3, 4)):
            check(lambda c: fn(c, [key], gal, mods, L, K, alpha), [ct], 0, at, q[at[2]])
        check(lambda k: fn(ct, [k], gal, mods, L, K, alpha), [key], 0, (1, 0, L, 5), mods[L])
    check(lambda c: orc.rescale(c, q), [ct], 0, (0, 1, L - 1, 2), q[L - 1])
    check(lambda c: orc.rescale(c, q), [ct], 0, (0, 0, 0, 2), q[0])
    ct2 = _rand_res((1, 2, L, N), q, 75)
    for idx, at, m in ((0, (0, 1, 1, 1), q[1]), (1, (0, 0, 5, 1), q[5]),
                       (2, (0, 1, L, 9), mods[L])):
        check(lambda x, y, k: orc.mul_relin_rescale(x, y, k, mods, L, K, alpha), [ct, ct2, key], idx,
              at, m)
    diags = _rand_res((2, 2, L, N), q, 76)
    bs = lambda x, d, kb, kg: orc.bsgs(x, d, [kb], [kg], 2, 2, mods, L, K, alpha)
    for idx, at, m in ((0, (0, 1, 2, 3), q[2]), (1, (1, 1, 0, 3), q[0]), (2, (0, 0, 1, 3), q[1]),
                       (3, (1, 1, L, 3), mods[L])):
        check(bs, [ct, diags, key, key2], idx, at, m)
    check(lambda x: orc.modraise(x, q), [a[:, :3].copy()], 0, (1, 2, 7), q[2])
    check(lambda c, k: orc.conj_extract(c, k, mods, L, K, alpha), [ct, key], 0, (0, 1, 0, 0), q[0])
    check(lambda c, k: orc.conj_extract(c, k, mods, L, K, alpha), [ct, key], 1, (2, 1, 3, 0), mods[3])
    for idx in range(2):
        check(lambda r, i: orc.restore_merge(r, i, q), [ct, ct2], idx, (0, idx, 4, 4), q[4])
