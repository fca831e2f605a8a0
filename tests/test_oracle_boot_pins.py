"""Pins of the oracle's bootstrapping steps: modraise, the monomial product,
conj_extract, restore_merge and the coeff_to_slot / slot_to_coeff transforms.

The pages name these steps (Kestrel engine write-up, the boot profile in
section 5.3) but give no formulas; the oracle follows the textbook forms.
Each pin checks a fact fixed outside the oracle: the centred CRT lift written
with Python integers, the closed form of X^e on monomials, X^{n/2} acting as i
on the slots, and decryption of each step against float64 arithmetic on the
plaintext (its real and imaginary parts, or its coefficients)."""
from fractions import Fraction

import numpy as np
import pytest

from rns_ckks_polynomial_b200 import synth

from .helpers import N, SCALE, Params, Scheme, galois_for_rotation, u64

SEED = synth.config_seed(0) + 0x100


def _complex_slots(n, stream):
    re = synth.uniform_real((n // 2,), -1, 1, SEED, stream).numpy()
    im = synth.uniform_real((n // 2,), -1, 1, SEED, stream + 1).numpy()
    return re + 1j * im


def _centred_coeffs(sch, ct):
    """Decryption of ct as centred Python integers (CRT over the ct's primes)."""
    L = ct.shape[-2]
    res = sch.orc.decrypt(ct, sch.s, sch.mods[:L])
    return sch.orc.crt_centered(res, sch.mods[:L])


# ------------------------------------------------------------------ X^e
@pytest.mark.parametrize("n", [16, N])
def test_mul_monomial_on_monomials(orc, n):
    """X^j X^e = (-1)^floor((j+e)/n) X^((j+e) mod n), for e in [0, 2n)."""
    mods = orc.gen_primes(n, 2)
    for j, e in [(0, 0), (1, n // 2), (n - 1, 1), (3, n - 3), (5, n + 2), (n - 1, 2 * n - 1)]:
        x = np.zeros((2, n), dtype=np.uint64)
        x[:, j] = 1
        y = orc.ntt_inv(orc.mul_monomial(orc.ntt_fwd(x, mods), e, mods), mods)
        t, sign = (j + e) % n, (-1) ** ((j + e) // n)
        for l, q in enumerate(int(v) for v in mods):
            want = np.zeros(n, dtype=object)
            want[t] = sign % q
            assert [int(v) for v in y[l]] == list(want)


def test_mul_monomial_half_is_i_on_slots(orc):
    """zeta^(n/2 * 5^j) = i for every slot j, so X^{n/2} multiplies each slot
    by i; applied twice it negates the polynomial."""
    mods = orc.gen_primes(N, 3)
    z = _complex_slots(N, 10)
    pt = orc.encode_ntt(z, mods, SCALE, N)
    out = orc.mul_monomial(pt, N // 2, mods)
    got = orc.decode(orc.ntt_inv(out, mods), mods, SCALE)
    assert np.max(np.abs(got - 1j * z)) < 1e-12
    twice = orc.mul_monomial(out, N // 2, mods)
    neg = np.array([[(int(q) - int(v)) % int(q) for v in pt[l]] for l, q in enumerate(mods)],
                   dtype=np.uint64)
    assert np.array_equal(twice, neg)


def test_mul_monomial_half_in_the_ntt_domain(orc):
    """NTT(X^{n/2})[k] = psi^{(n/2)(2 brv(k) + 1)} = i_q (-1)^{brv(k)} with
    i_q = psi^{n/2}: +i_q on the first n/2 evaluation slots, -i_q on the rest.
    So X^{n/2} x is a pointwise product by those constants."""
    mods = orc.gen_primes(N, 3)
    x = u64(synth.uniform_residues((2, 3, N), mods, SEED, 15))
    iq = [pow(int(orc.find_psi(int(q), N)), N // 2, int(q)) for q in mods]
    assert all(v * v % int(q) == int(q) - 1 for v, q in zip(iq, mods))
    c = np.array([[v] * (N // 2) + [int(q) - v] * (N // 2) for v, q in zip(iq, mods)],
                 dtype=np.uint64)
    want = orc.pointwise("mul", x, np.broadcast_to(c, x.shape).copy(), mods)
    assert np.array_equal(orc.mul_monomial(x, N // 2, mods), want)


# ------------------------------------------------------------------ modraise
def test_modraise_is_the_centred_crt_lift(orc):
    """Coefficients over q_0..q_2 -> their centred integer X in (-Q/2, Q/2],
    reduced modulo all six primes; the residues below q_3 are unchanged.
    The boundary values 0, 1, (Q-1)/2, (Q+1)/2, Q-1 are included."""
    mods = orc.gen_primes(N, 6)
    l = 3
    q = [int(v) for v in mods]
    Q = q[0] * q[1] * q[2]
    x = u64(synth.uniform_residues((2, l, N), mods[:l], SEED, 20))
    specials = [0, 1, (Q - 1) // 2, (Q + 1) // 2, Q - 1, Q // 3]
    for k, X in enumerate(specials):
        for i in range(l):
            x[0, i, k] = X % q[i]
    y = orc.ntt_inv(orc.modraise(orc.ntt_fwd(x, mods[:l]), mods), mods)
    assert y.shape == (2, 6, N)
    for p in range(2):
        X = orc.crt_centered(x[p], mods[:l])
        for t in range(6):
            assert [int(v) for v in y[p, t]] == [v % q[t] for v in X]
    # the centring decision at the boundary
    assert orc.crt_centered(y[0, :, :5], mods)[:5] == [0, 1, (Q - 1) // 2, -(Q - 1) // 2, -1]


def test_modraise_decrypts_to_message_plus_small_multiple_of_q(orc):
    """A ciphertext kept on q_0, q_1 and raised to six primes decrypts to
    m + e + Q_2 I with an integer polynomial I, |I_k| <= (h + 1) / 2 + 1 for a
    secret of Hamming weight h."""
    p = Params(6, 2, 2)
    sch = Scheme(orc, p, SEED + 1)
    z = _complex_slots(N, 30)
    ct = sch.encrypt_slots(z)
    low = np.ascontiguousarray(ct[:, :2])
    Q2 = int(sch.mods[0]) * int(sch.mods[1])
    raised = orc.modraise(low, sch.q)
    assert np.array_equal(raised[:, :2], low)
    v_low = _centred_coeffs(sch, low)
    v_full = _centred_coeffs(sch, raised)
    h = int(np.count_nonzero(sch.s))
    I = []
    for a, b in zip(v_full, v_low):
        assert (a - b) % Q2 == 0
        I.append((a - b) // Q2)
    assert max(abs(v) for v in I) <= (h + 1) // 2 + 1
    assert any(I)
    # the low decryption is the message: it decodes to z
    got = sch.decrypt_slots(low)
    assert np.max(np.abs(got - z)) < 1e-8


# ------------------------------------------------------------------ conj_extract, restore_merge
def _conj_scheme(orc):
    p = Params(6, 2, 2)
    sch = Scheme(orc, p, SEED + 2)
    return sch, sch.keygen_galois(2 * N - 1)


def test_conj_extract_gives_real_and_imaginary_parts(orc):
    sch, ck = _conj_scheme(orc)
    p = sch.p
    w = _complex_slots(N, 40)
    ct = sch.encrypt_slots(w)
    re, im = orc.conj_extract(ct[None], ck, sch.mods, p.L, p.K, p.alpha)
    got_re = sch.decrypt_slots(re[0], 2 * SCALE)
    got_im = sch.decrypt_slots(im[0], 2 * SCALE)
    assert np.max(np.abs(got_re - w.real)) < 1e-8
    assert np.max(np.abs(got_im - w.imag)) < 1e-8


def test_restore_merge_and_round_trip(orc):
    sch, ck = _conj_scheme(orc)
    p = sch.p
    a = synth.uniform_real((N // 2,), -1, 1, SEED, 50).numpy()
    b = synth.uniform_real((N // 2,), -1, 1, SEED, 51).numpy()
    ca, cb = sch.encrypt_slots(a), sch.encrypt_slots(b)
    merged = orc.restore_merge(ca[None], cb[None], sch.q)
    assert np.max(np.abs(sch.decrypt_slots(merged[0]) - (a + 1j * b))) < 1e-8
    # merge(extract(ct)) has slots 2w
    w = _complex_slots(N, 52)
    ct = sch.encrypt_slots(w)
    re, im = orc.conj_extract(ct[None], ck, sch.mods, p.L, p.K, p.alpha)
    back = orc.restore_merge(re, im, sch.q)
    assert np.max(np.abs(sch.decrypt_slots(back[0], 2 * SCALE) - w)) < 1e-8


# ------------------------------------------------------------------ coeff_to_slot / slot_to_coeff
def _transform_scheme(orc, n, bb, gg):
    p = Params(6, 2, 2, n=n)
    sch = Scheme(orc, p, SEED + 3 + n)
    baby = [sch.keygen_galois(galois_for_rotation(b, n)) for b in range(1, bb)]
    giant = [sch.keygen_galois(galois_for_rotation(bb * g, n)) for g in range(1, gg)]
    return sch, baby, giant


def _at_level(sch, L, keys):
    """Moduli and keys for a ciphertext on q_0..q_{L-1}: the special primes
    follow the ciphertext primes, and each key keeps the limbs of those primes
    and the first ceil(L / alpha) digits (a key reduced modulo a divisor of
    its modulus is a key for that modulus)."""
    p = sch.p
    keep = list(range(L)) + list(range(p.L, p.L + p.K))
    mods = np.ascontiguousarray(sch.mods[keep])
    dn = (L + p.alpha - 1) // p.alpha
    return mods, [np.ascontiguousarray(k[:dn][:, :, keep]) for k in keys]


def _lintrans(orc, sch, ct, M, bb, gg, baby, giant):
    p = sch.p
    L = ct.shape[-2]
    mods, keys = _at_level(sch, L, baby + giant)
    diags = orc.lintrans_plaintexts(M, bb, gg, mods[:L], SCALE, p.n)
    y = orc.bsgs(ct[None], diags, keys[: bb - 1], keys[bb - 1:], bb, gg, mods, L, p.K, p.alpha)
    return y[0]


def test_embedding_matrix_rows_are_orthogonal(orc):
    """U U^H = (n/2) I, and U applied to (m_lo + i m_hi) / scale equals the
    decoder's slots of m."""
    n = 64
    U = orc.embedding_matrix(n)
    assert np.max(np.abs(U @ U.conj().T - (n // 2) * np.eye(n // 2))) < 1e-12
    assert np.max(np.abs(orc.coeff_to_slot_matrix(n) @ orc.slot_to_coeff_matrix(n)
                         - np.eye(n // 2))) < 1e-12
    m = synth.uniform_real((n,), -1, 1, SEED, 60).numpy()
    v = m[: n // 2] + 1j * m[n // 2:]
    assert np.max(np.abs(U @ v - orc.decode_coeffs_float(m, n))) < 1e-12


@pytest.mark.parametrize("n,bb,gg", [(64, 8, 4), (256, 16, 8)])
def test_coeff_to_slot_gives_the_coefficients_as_slots(orc, n, bb, gg):
    """coeff_to_slot of an encryption of polynomial m decrypts to slots
    (m_k + i m_{k+n/2}) / scale, read off the decrypted input's coefficients."""
    sch, baby, giant = _transform_scheme(orc, n, bb, gg)
    z = _complex_slots(n, 70)
    ct = sch.encrypt_slots(z)
    m = _centred_coeffs(sch, ct)
    want = np.array([(Fraction(m[k]) / SCALE) for k in range(n // 2)], dtype=float) + \
        1j * np.array([(Fraction(m[k + n // 2]) / SCALE) for k in range(n // 2)], dtype=float)
    y = _lintrans(orc, sch, ct, orc.coeff_to_slot_matrix(n), bb, gg, baby, giant)
    sc = sch.rescaled_scale(SCALE * SCALE, sch.p.L)
    assert np.max(np.abs(sch.decrypt_slots(y, sc) - want)) < 1e-8


@pytest.mark.parametrize("n,bb,gg", [(64, 8, 4), (256, 16, 8)])
def test_slot_to_coeff_puts_the_slots_into_the_coefficients(orc, n, bb, gg):
    """slot_to_coeff of an encryption of slots v decrypts to a polynomial with
    coefficients scale * Re v_k (k < n/2) and scale * Im v_{k-n/2} (k >= n/2)."""
    sch, baby, giant = _transform_scheme(orc, n, bb, gg)
    v = _complex_slots(n, 80)
    ct = sch.encrypt_slots(v)
    y = _lintrans(orc, sch, ct, orc.slot_to_coeff_matrix(n), bb, gg, baby, giant)
    sc = sch.rescaled_scale(SCALE * SCALE, sch.p.L)
    got = np.array([float(Fraction(c) / sc) for c in _centred_coeffs(sch, y)])
    assert np.max(np.abs(got - np.concatenate([v.real, v.imag]))) < 1e-8


def test_linear_part_of_bootstrapping(orc):
    """modraise -> coeff_to_slot -> conj_extract -> restore_merge ->
    slot_to_coeff on a ciphertext kept on two primes: the result decrypts to
    2 t, where t = m + e + Q_2 I is the raised plaintext (no evaluation of the
    modular reduction in between, so nothing removes Q_2 I)."""
    n, bb, gg = 64, 8, 4
    sch, baby, giant = _transform_scheme(orc, n, bb, gg)
    p = sch.p
    ck = sch.keygen_galois(2 * n - 1)
    z = _complex_slots(n, 90)
    low = np.ascontiguousarray(sch.encrypt_slots(z)[:, :2])
    ct = orc.modraise(low, sch.q)
    t = _centred_coeffs(sch, ct)
    a = _lintrans(orc, sch, ct, orc.coeff_to_slot_matrix(n), bb, gg, baby, giant)
    mods5, (ck5,) = _at_level(sch, p.L - 1, [ck])
    re, im = orc.conj_extract(a[None], ck5, mods5, p.L - 1, p.K, p.alpha)
    merged = orc.restore_merge(re, im, sch.mods[: p.L - 1])[0]
    out = _lintrans(orc, sch, merged, orc.slot_to_coeff_matrix(n), bb, gg, baby, giant)
    assert out.shape == (2, p.L - 2, n)
    sc = (Fraction(SCALE * SCALE, int(sch.mods[p.L - 1])) * SCALE) / int(sch.mods[p.L - 2])
    got = [Fraction(c) / sc for c in _centred_coeffs(sch, out)]
    want = [Fraction(2 * v, SCALE) for v in t]
    big = max(abs(w) for w in want)
    assert big > 2**50  # the lift really added multiples of Q_2
    assert max(abs(float(g - w)) for g, w in zip(got, want)) < 1e-9 * float(big)


# ------------------------------------------------------------------ sin_fold and the whole refresh
def _boot_scheme(orc, n, bb, gg, seed):
    p = Params(20, 4, 4, n=n)
    sch = Scheme(orc, p, seed)
    keys = {"relin": sch.keygen_relin(), "conj": sch.keygen_galois(2 * n - 1),
            "baby": [sch.keygen_galois(galois_for_rotation(b, n)) for b in range(1, bb)],
            "giant": [sch.keygen_galois(galois_for_rotation(bb * g, n)) for g in range(1, gg)]}
    return sch, keys


def test_sin_fold_is_sine_of_two_pi_x(orc):
    """Slots x = I + f, integers |I| <= 20 and |f| <= 0.01: sin_fold with r = 8
    consumes 6 + 8 levels and decrypts to sin(2 pi x), to 1e-9."""
    from oracle import boot
    n, r = 64, 8
    sch = Scheme(orc, Params(20, 4, 4, n=n), SEED + 7)
    chain = boot.Chain(sch.mods, 20, 4, 4)
    rlk = sch.keygen_relin()
    x = (synth.uniform_below((n // 2,), 41, SEED, 100).numpy() - 20
         + synth.uniform_real((n // 2,), -0.01, 0.01, SEED, 101).numpy())
    ct = sch.encrypt_slots(x)
    out, s = boot.sin_fold(ct, Fraction(SCALE), r, rlk, chain)
    assert out.shape == (2, 20 - 6 - r, n)
    got = sch.decrypt_slots(out, s)
    assert np.max(np.abs(got - np.sin(2 * np.pi * x))) < 1e-9


def test_bootstrap_removes_the_multiple_of_q0(orc):
    """A ciphertext on q_0 holding slots z at scale 2^50, refreshed onto the
    20-prime chain: modraise adds q_0 I, and the refresh returns a ciphertext
    2 + 6 + 8 levels down whose coefficients are
    (q_0 / 2 pi) sin(2 pi m_k / q_0) / Delta (to 1e-7), i.e. m_k / Delta up to
    the sine's own cubic term, and whose slots are z to within that term."""
    import math

    from oracle import boot
    n, bb, gg, r = 64, 8, 4, 8
    delta = 2**50
    sch, keys = _boot_scheme(orc, n, bb, gg, SEED + 8)
    chain = boot.Chain(sch.mods, 20, 4, 4)
    z = _complex_slots(n, 110)
    low = np.ascontiguousarray(sch.encrypt_slots(z, delta)[:, :1])
    q0 = int(sch.mods[0])
    m = _centred_coeffs(sch, low)
    t = _centred_coeffs(sch, orc.modraise(low, sch.q))
    assert any((a - b) // q0 for a, b in zip(t, m))
    out, s = boot.bootstrap(low, delta, r, keys, chain, bb, gg)
    assert out.shape == (2, 20 - 2 - 6 - r, n)
    got = np.array([float(Fraction(c) / s) for c in _centred_coeffs(sch, out)])
    sine = np.array([q0 / (2 * math.pi) * math.sin(2 * math.pi * v / q0) / delta for v in m])
    assert np.max(np.abs(got - sine)) < 1e-7
    mm = np.array(m, dtype=float) / delta
    cubic = np.max(np.abs(mm) * (2 * np.pi * np.abs(mm) * delta / q0) ** 2 / 6)
    assert np.max(np.abs(got - mm)) < cubic + 1e-7
    slots = sch.decrypt_slots(out, s)
    assert np.max(np.abs(slots - z)) < n * (cubic + 1e-7)


# ------------------------------------------------------------------ factored transforms
@pytest.mark.parametrize("n", [16, 64, 256])
@pytest.mark.parametrize("depth", [1, 2, 3])
def test_special_fft_factorization(orc, n, depth):
    """F_depth ... F_1 R = U and H_depth ... H_1 = R U^-1 against the dense
    embedding matrix; a group of k butterfly stages has at most 2^(k+1) - 1
    diagonals, all multiples of its stride, and its BSGS plan covers them."""
    S = n // 2
    U = orc.embedding_matrix(n)
    R = np.eye(S)[orc.bit_reverse_indices(S)]
    assert sorted(orc.bit_reverse_indices(S)) == list(range(S))
    P, Q = np.eye(S, dtype=complex), np.eye(S, dtype=complex)
    for F in orc.factored_slot_to_coeff(n, depth):
        P = orc.diag_to_dense(F, S) @ P
    for H in orc.factored_coeff_to_slot(n, depth):
        Q = orc.diag_to_dense(H, S) @ Q
    assert np.max(np.abs(P @ R - U)) < 1e-12
    assert np.max(np.abs(Q @ U - R)) < 1e-12
    for grp, F in zip(orc.stage_groups(n, depth), orc.factored_slot_to_coeff(n, depth)):
        assert len(F) <= 2 ** (len(grp) + 1) - 1
        stride, t0, bb, gg = orc.bsgs_plan(F, S)
        assert all(k % stride == 0 for k in F)
        covered = {(stride * (t0 + bb * g + b)) % S for g in range(gg) for b in range(bb)}
        assert set(F) <= covered


def _factored_scheme(orc, n, depth, seed):
    from oracle import boot
    sch = Scheme(orc, Params(20, 4, 4, n=n), seed)
    keys = {"rot": {a: sch.keygen_galois(galois_for_rotation(a, n))
                    for a in boot.factored_rotation_amounts(n, depth)},
            "conj": sch.keygen_galois(2 * n - 1), "relin": sch.keygen_relin()}
    return sch, boot.Chain(sch.mods, 20, 4, 4), keys


def test_factored_transforms_decrypt(orc):
    """Two-level coeff_to_slot puts (m_k + i m_{k+n/2}) / scale into slot
    brv(k); two-level slot_to_coeff of those bit-reversed slots gives U v."""
    from oracle import boot
    n, depth = 64, 2
    S = n // 2
    sch, chain, keys = _factored_scheme(orc, n, depth, SEED + 9)
    ct = sch.encrypt_slots(_complex_slots(n, 120))
    m = _centred_coeffs(sch, ct)
    v = np.array([float(Fraction(m[k], SCALE)) + 1j * float(Fraction(m[k + S], SCALE))
                  for k in range(S)])
    w = v[orc.bit_reverse_indices(S)]
    y, sc = boot.lintrans_factored(ct, Fraction(SCALE), orc.factored_coeff_to_slot(n, depth), SCALE,
                                   keys["rot"], chain)
    assert y.shape == (2, 20 - depth, n)
    assert np.max(np.abs(sch.decrypt_slots(y, sc) - w)) < 1e-8
    y2, sc2 = boot.lintrans_factored(sch.encrypt_slots(w), Fraction(SCALE),
                                     orc.factored_slot_to_coeff(n, depth), SCALE, keys["rot"], chain)
    assert np.max(np.abs(sch.decrypt_slots(y2, sc2) - orc.embedding_matrix(n) @ v)) < 1e-8


def test_bootstrap_with_factored_transforms(orc):
    """The refresh with two-level transforms: 2 * 2 + 6 + 8 levels, and the
    same sine form of the coefficients as the dense refresh."""
    import math

    from oracle import boot
    n, depth, r = 64, 2, 8
    delta = 2**50
    sch, chain, keys = _factored_scheme(orc, n, depth, SEED + 10)
    z = _complex_slots(n, 130)
    low = np.ascontiguousarray(sch.encrypt_slots(z, delta)[:, :1])
    q0 = int(sch.mods[0])
    m = _centred_coeffs(sch, low)
    out, s = boot.bootstrap_factored(low, delta, r, depth, keys, chain)
    assert out.shape == (2, 20 - 2 * depth - 6 - r, n)
    got = np.array([float(Fraction(c) / s) for c in _centred_coeffs(sch, out)])
    sine = np.array([q0 / (2 * math.pi) * math.sin(2 * math.pi * v / q0) / delta for v in m])
    assert np.max(np.abs(got - sine)) < 1e-7


@pytest.mark.slow
@pytest.mark.skipif(not __import__("os").environ.get("CKKS_SLOW_PINS"),
                    reason="about 90 s of CPU; set CKKS_SLOW_PINS=1")
def test_bootstrap_at_ring_degree_2048(orc):
    """The refresh at n = 2048 with a dense ternary secret, three-level
    factored transforms and r = 9: 2 * 3 + 6 + 9 = 21 levels (23 primes down
    to 2), and the sine form of the coefficients within 1e-5."""
    import math

    from oracle import boot
    n, depth, r, L = N, 3, 9, 23
    delta = 2**50
    sch = Scheme(orc, Params(L, 4, 4), SEED + 11)
    chain = boot.Chain(sch.mods, L, 4, 4)
    keys = {"rot": {a: sch.keygen_galois(galois_for_rotation(a, n))
                    for a in boot.factored_rotation_amounts(n, depth)},
            "conj": sch.keygen_galois(2 * n - 1), "relin": sch.keygen_relin()}
    low = np.ascontiguousarray(sch.encrypt_slots(_complex_slots(n, 140), delta)[:, :1])
    q0 = int(sch.mods[0])
    m = _centred_coeffs(sch, low)
    out, s = boot.bootstrap_factored(low, delta, r, depth, keys, chain)
    assert out.shape == (2, L - 2 * depth - 6 - r, n)
    got = np.array([float(Fraction(c) / s) for c in _centred_coeffs(sch, out)])
    sine = np.array([q0 / (2 * math.pi) * math.sin(2 * math.pi * v / q0) / delta for v in m])
    assert np.max(np.abs(got - sine)) < 1e-5


def test_refresh_with_levels_is_the_factored_refresh(orc):
    """Fed the encoded levels, the plaintext-taking refresh is the factored
    refresh bit for bit (zeros stand for absent diagonals)."""
    import math

    from oracle import boot
    n, depth, r = 64, 2, 8
    delta = 2**50
    sch, chain, keys = _factored_scheme(orc, n, depth, SEED + 12)
    low = np.ascontiguousarray(sch.encrypt_slots(_complex_slots(n, 150), delta)[:, :1])
    want, s_want = boot.bootstrap_factored(low, delta, r, depth, keys, chain)

    def levels(factors, scalar, top, pt_scale):
        out = []
        for i, F in enumerate(factors):
            if i == 0:
                F = {k: scalar * d for k, d in F.items()}
            plan = orc.bsgs_plan(F, n // 2)
            pts, _ = orc.plan_plaintexts(F, plan, n // 2, sch.mods[:top - i], pt_scale, n)
            out.append((plan, [[np.zeros((top - i, n), np.uint64) if v is None else v for v in row]
                               for row in pts]))
        return out

    q0 = int(sch.mods[0])
    cts = levels(orc.factored_coeff_to_slot(n, depth), 0.5, 20, 2**60)
    stc = levels(orc.factored_slot_to_coeff(n, depth), q0 / (2 * math.pi * delta),
                 20 - depth - 6 - r, 2**50)
    got, s_got = boot.refresh_with_levels(low, r, cts, stc, keys, chain)
    assert s_got == s_want
    assert np.array_equal(got, want)
