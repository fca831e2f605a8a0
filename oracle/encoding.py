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


def encode_many(Z, n, scale):
    """Encode every row of Z ([count][n/2] slots) as encode() does, with the
    sum over slots written as one long-double matrix product against the
    table zeta^(-k e_j).  The sums run in another order than encode()'s, so
    a coefficient can differ from encode()'s by one where scale times the sum
    falls within long-double rounding of a half-integer; both are
    round(scale * tau^-1(z)) to within that rounding."""
    Z = np.atleast_2d(np.asarray(Z, dtype=np.clongdouble))
    if Z.shape[1] != n // 2:
        raise ValueError("expected rows of %d slots" % (n // 2))
    ang = _PI * _angle_matrix(n, -1).astype(np.longdouble) / np.longdouble(n)
    re = np.cos(ang) @ Z.real.T
    if np.any(Z.imag != 0):
        re = re - np.sin(ang) @ Z.imag.T
    v = (np.longdouble(2) / np.longdouble(n)) * re * np.longdouble(scale)
    r = np.sign(v) * np.floor(np.abs(v) + np.longdouble(0.5))
    return np.ascontiguousarray(r.T.astype(np.int64))


def encode_ntt_many(Z, mods, scale, n):
    """encode_many, then the residues of every coefficient modulo each prime
    and the forward NTT: [count][L][n]."""
    from .core import ntt_fwd
    m = encode_many(Z, n, scale)
    q = np.array([int(v) for v in mods], dtype=np.int64)
    out = np.empty((m.shape[0], len(q), n), dtype=np.uint64)
    for c in range(0, m.shape[0], 64):  # bounded temporaries
        res = np.mod(m[c:c + 64, None, :], q[None, :, None]).astype(np.uint64)
        out[c:c + 64] = ntt_fwd(res, mods)
    return out


def embedding_matrix(n):
    """U[j][k] = zeta^(k e_j), j, k < n/2, zeta = exp(i pi / n), e_j = 5^j mod 2n
    (reading R14 of the design notes).

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


# ---------------------------------------------------------------- factored transforms
#
# Reading R16 of the design notes: the pages time coeff_to_slot and
# slot_to_coeff (Kestrel engine write-up, boot profile in section 5.3) but give
# no factorization; this is the textbook special-FFT one.
#
# U evaluates V(X) = sum_k v_k X^k at the S = n/2 points w_j = zeta^(5^j).  Split
# V(X) = E(X^2) + X O(X^2).  The squares w_j^2 are the points of the same problem
# for S/2 (zeta^2, 5^j mod n), and w_{j+S/2} = -w_j because 5^(S/2) = 1 + n
# (mod 2n).  Hence z_j = E_j + w_j O_j and z_{j+S/2} = E_j - w_j O_j: a
# butterfly stage over a half-size transform of the even and of the odd
# coefficients.  Unrolled, U = G_m ... G_1 R with m = log2 S, R the bit-reversal
# permutation and G_s (block length len = 2^s) acting on each block of len
# slots as [[I, D], [I, -D]], D = diag(zeta_len^(5^j)), j < len/2, zeta_len a
# primitive (4 len)-th root of unity.  Every G_s has three slot diagonals
# (offsets 0, len/2, -len/2), so a group of consecutive stages a..b has at
# most 2^(b-a+2) - 1 diagonals, all multiples of 2^(a-1).
#
# A matrix is held in diagonal form {k: d_k}, d_k[i] = M[i][(i + k) mod S], so
# (M x)_i = sum_k d_k[i] x[(i + k) mod S].


def bit_reverse_indices(S):
    bits = S.bit_length() - 1
    return np.array([int(format(i, "0%db" % bits)[::-1], 2) if bits else 0 for i in range(S)])


def _stage_diagonals(n, s, inverse=False):
    """G_s (or its inverse) in diagonal form."""
    S = n // 2
    ln = 1 << s
    h = ln // 2
    e = np.array([pow(5, j, 4 * ln) for j in range(h)], dtype=np.int64)
    ang = 2 * _PI * e.astype(np.longdouble) / np.longdouble(4 * ln)
    D = (np.cos(ang) + 1j * np.sin(ang)).astype(np.complex128)
    pos = np.arange(S) % ln
    top = pos < h
    j = np.where(top, pos, pos - h)
    d0, dp, dm = np.zeros(S, complex), np.zeros(S, complex), np.zeros(S, complex)
    if not inverse:
        # top rows: u + D v;  bottom rows: u - D v
        d0[top], dp[top] = 1, D[j[top]]
        dm[~top], d0[~top] = 1, -D[j[~top]]
    else:
        # [[I, D], [I, -D]]^-1 = 1/2 [[I, I], [D^-1, -D^-1]]
        d0[top], dp[top] = 0.5, 0.5
        dm[~top], d0[~top] = 0.5 / D[j[~top]], -0.5 / D[j[~top]]
    out = {0: d0}
    if h == S // 2 and S > 1:
        out[h] = dp + dm               # +h and -h are the same offset mod S
    else:
        out[h] = dp
        out[(S - h) % S] = dm
    return out


def diag_product(A, B, S):
    """Diagonal form of A B: d_{a+b}[i] += A_a[i] B_b[i + a]."""
    out = {}
    for a, da in A.items():
        for b, db in B.items():
            k = (a + b) % S
            out[k] = out.get(k, 0) + da * np.roll(db, -a)
    return out


def diag_to_dense(Dg, S):
    M = np.zeros((S, S), dtype=complex)
    i = np.arange(S)
    for k, d in Dg.items():
        M[i, (i + k) % S] += d
    return M


def stage_groups(n, depth):
    """Split the log2(n/2) butterfly stages into `depth` consecutive groups,
    the later groups at least as long as the earlier ones."""
    m = (n // 2).bit_length() - 1
    base, extra = divmod(m, depth)
    sizes = [base + (1 if g >= depth - extra else 0) for g in range(depth)]
    out, s = [], 1
    for sz in sizes:
        out.append(list(range(s, s + sz)))
        s += sz
    return out


def factored_slot_to_coeff(n, depth):
    """Diagonal forms F_1..F_depth with U = F_depth ... F_1 R (F_1 applied first)."""
    S = n // 2
    mats = []
    for grp in stage_groups(n, depth):
        F = {0: np.ones(S, complex)}
        for s in grp:
            F = diag_product(_stage_diagonals(n, s), F, S)
        mats.append(F)
    return mats


def factored_coeff_to_slot(n, depth):
    """Diagonal forms H_1..H_depth with R U^-1 = H_depth ... H_1 (H_1 applied
    first): the inverse stages in reverse order; the output slots come out in
    bit-reversed order, which factored_slot_to_coeff takes back."""
    S = n // 2
    mats = []
    for grp in reversed(stage_groups(n, depth)):
        F = {0: np.ones(S, complex)}
        for s in reversed(grp):
            F = diag_product(_stage_diagonals(n, s, inverse=True), F, S)
        mats.append(F)
    return mats


def bsgs_plan(Dg, S, tol=0.0):
    """Baby-step giant-step plan for a diagonal form whose nonzero offsets are
    stride * t, t in a window [t0, t0 + T): offsets stride (t0 + bb g + b),
    g < gg, b < bb, with bb the power of two nearest sqrt(T).  Returns
    (stride, t0, bb, gg)."""
    ks = sorted(k for k, d in Dg.items() if np.max(np.abs(d)) > tol)
    if ks == [0]:
        return 1, 0, 1, 1
    stride = int(np.gcd.reduce([k for k in ks if k] + [S]))
    ts = sorted(((k // stride) + S // stride // 2) % (S // stride) - S // stride // 2 for k in ks)
    t0, T = ts[0], ts[-1] - ts[0] + 1
    bb = 1 << max(0, round(np.log2(np.sqrt(T))))
    gg = -(-T // bb)
    return stride, t0, bb, gg


def plan_plaintexts(Dg, plan, S, mods, scale, n):
    """pt_{g,b} = Encode(rot_{-G_g}(d_{G_g + stride b})) with G_g = stride (t0 + bb g);
    None where that diagonal is absent.  Also returns the giant offsets G_g."""
    stride, t0, bb, gg = plan
    pts, giants = [], []
    for g in range(gg):
        G = (stride * (t0 + bb * g)) % S
        giants.append(G)
        row = []
        for b in range(bb):
            k = (G + stride * b) % S
            d = Dg.get(k)
            row.append(None if d is None else encode_ntt(np.roll(d, G), mods, scale, n))
        pts.append(row)
    return pts, giants


__all__ = ["slot_exponents", "encode", "crt_centered", "decode", "decode_coeffs_float",
           "encode_ntt", "embedding_matrix", "coeff_to_slot_matrix", "slot_to_coeff_matrix",
           "lintrans_plaintexts", "bit_reverse_indices", "diag_product", "diag_to_dense",
           "stage_groups", "factored_slot_to_coeff", "factored_coeff_to_slot", "bsgs_plan",
           "plan_plaintexts", "encode_many", "encode_ntt_many"]
