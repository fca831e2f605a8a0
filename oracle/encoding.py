"""Canonical-embedding encoder/decoder and CRT (test infrastructure only).

The pages fix n = 2048, 1024 slots and scale 2^60 (Kestrel FHE relay README,
section 1; Kestrel engine write-up, section 4.1) but not the slot order.  The
reading used here is the standard one: slot j holds m(zeta^(5^j mod 2n)) / scale
with zeta = exp(i pi / n), so the Galois element 5^r rotates the slots left
by r.

encode: m_k = round_half_away( scale * (2/n) Re sum_j z_j zeta^(-k e_j) ),
        e_j = 5^j mod 2n, evaluated as an O(n^2) sum in long double.
decode: CRT-reconstruct each coefficient over all primes with Python integers,
        centre it into (-Q/2, Q/2], divide by the scale and evaluate
        z_j = sum_k m_k zeta^(k e_j) in long double.
"""
import numpy as np

# pi to long-double precision (numpy.pi is a float64 constant)
_PI = np.arctan(np.longdouble(1)) * 4


def slot_exponents(n):
    """e_j = 5^j mod 2n for the n/2 slots."""
    return np.array([pow(5, j, 2 * n) for j in range(n // 2)], dtype=np.int64)


def _angle_matrix(n, sign):
    """Integer exponent table (sign * k * e_j) mod 2n, shape [n][n/2]."""
    e = slot_exponents(n)
    k = np.arange(n, dtype=np.int64)
    return (sign * np.outer(k, e)) % (2 * n)


def encode(z, n, scale):
    """Slots z (complex or real, length n/2) -> integer coefficients (int64)."""
    z = np.asarray(z, dtype=np.clongdouble)
    if z.shape != (n // 2,):
        raise ValueError("expected %d slots" % (n // 2))
    idx = _angle_matrix(n, -1)
    ang = _PI * idx.astype(np.longdouble) / np.longdouble(n)
    re = np.cos(ang) * z.real[None, :] - np.sin(ang) * z.imag[None, :]
    m = (np.longdouble(2) / np.longdouble(n)) * re.sum(axis=1)
    v = m * np.longdouble(scale)
    r = np.sign(v) * np.floor(np.abs(v) + np.longdouble(0.5))
    return np.array([int(x) for x in r], dtype=np.int64)


def crt_centered(res, mods):
    """res[L][n] residues -> list of n Python ints in (-Q/2, Q/2]."""
    mods = [int(q) for q in mods]
    Q = 1
    for q in mods:
        Q *= q
    coeffs = []
    for i, q in enumerate(mods):
        qhat = Q // q
        coeffs.append(qhat * pow(qhat % q, -1, q))
    res = np.asarray(res)
    n = res.shape[-1]
    out = []
    for k in range(n):
        x = 0
        for i in range(len(mods)):
            x += int(res[i, k]) * coeffs[i]
        x %= Q
        if x > Q // 2:
            x -= Q
        out.append(x)
    return out


def decode(res, mods, scale):
    """Coefficient residues [L][n] (a decryption) -> complex slots.  `scale`
    may be an int or a fractions.Fraction (the tracked scale after rescale)."""
    from fractions import Fraction
    m = crt_centered(res, mods)
    n = np.asarray(res).shape[-1]
    sc = Fraction(scale)
    mf = [float(Fraction(x) / sc) for x in m]
    return decode_coeffs_float(np.array(mf, dtype=np.float64), n)


def decode_coeffs_float(mf, n):
    """Real coefficients already divided by the scale -> complex slots."""
    mf = np.asarray(mf, dtype=np.longdouble)
    idx = _angle_matrix(n, 1)
    ang = _PI * idx.astype(np.longdouble) / np.longdouble(n)
    re = (np.cos(ang) * mf[:, None]).sum(axis=0)
    im = (np.sin(ang) * mf[:, None]).sum(axis=0)
    return (re + 1j * im).astype(np.complex128)


def encode_ntt(z, mods, scale, n):
    """Encode slots and return NTT residues [L][n] over mods."""
    from .core import ntt_fwd
    m = encode(z, n, scale)
    res = np.stack([np.array([x % int(q) for x in m.tolist()], dtype=np.uint64)
                    for q in mods])
    return ntt_fwd(res, mods)


def embedding_matrix(n):
    """U[j][k] = zeta^(k e_j), j, k < n/2, zeta = exp(i pi / n), e_j = 5^j mod 2n.

    Slot j of a polynomial with real coefficients m is sum_k m_k zeta^(k e_j);
    since zeta^(n/2 e_j) = i (e_j = 1 mod 4), the slots are U (m_lo + i m_hi)
    with m_lo = m[:n/2] and m_hi = m[n/2:].  slot_to_coeff applies U to the
    slots, coeff_to_slot applies U^-1 = (2/n) U^H (the rows of U are orthogonal:
    the e_j are distinct mod 2n, so every off-diagonal row product is a full
    sum over the powers of a non-trivial root of unity)."""
    e = slot_exponents(n)
    k = np.arange(n // 2, dtype=np.int64)
    idx = np.outer(e, k) % (2 * n)
    ang = _PI * idx.astype(np.longdouble) / np.longdouble(n)
    return (np.cos(ang) + 1j * np.sin(ang)).astype(np.complex128)


def coeff_to_slot_matrix(n):
    """(2/n) U^H: slots U v -> slots v."""
    return (2.0 / n) * embedding_matrix(n).conj().T


def slot_to_coeff_matrix(n):
    """U: slots v -> slots U v, i.e. the encoding of the coefficients (Re v, Im v)."""
    return embedding_matrix(n)


def lintrans_plaintexts(M, bb, gg, mods, scale, n):
    """BSGS plaintexts of a slot matrix M (S x S, S = n/2, S = bb gg):
    pt_{g,b} = Encode(rot_{-bb g}(diag_{bb g + b})), diag_k[i] = M[i][(i + k) mod S],
    NTT residues [gg][bb][L][n]."""
    S = M.shape[0]
    if S != n // 2 or bb * gg != S:
        raise ValueError("need an (n/2) x (n/2) matrix and bb * gg = n/2")
    idx = np.arange(S)
    out = np.zeros((gg, bb, len(mods), n), dtype=np.uint64)
    for g in range(gg):
        for b in range(bb):
            k = bb * g + b
            diag = M[idx, (idx + k) % S]
            out[g, b] = encode_ntt(np.roll(diag, bb * g), mods, scale, n)
    return out


__all__ = ["slot_exponents", "encode", "crt_centered", "decode", "decode_coeffs_float",
           "encode_ntt", "embedding_matrix", "coeff_to_slot_matrix", "slot_to_coeff_matrix",
           "lintrans_plaintexts"]
