"""ctypes bindings to the oracle's C arithmetic (test infrastructure only).

Every array is a C-contiguous numpy ``uint64`` (residues) or ``int64``
(small signed coefficients).  Shapes follow the library's limb-major layout
``[batch][component][limb][n]``.
"""
import ctypes as C

import numpy as np

from . import build as _build

_LIB = None
_u64p = C.POINTER(C.c_uint64)
_i64p = C.POINTER(C.c_int64)


def _lib():
    global _LIB
    if _LIB is None:
        _LIB = C.CDLL(_build.build())
        L = _LIB
        L.oracle_is_prime.argtypes = [C.c_uint64]
        L.oracle_is_prime.restype = C.c_int
        L.oracle_gen_primes.argtypes = [C.c_int, C.c_int, _u64p]
        L.oracle_gen_primes.restype = C.c_int
        L.oracle_find_psi.argtypes = [C.c_uint64, C.c_int]
        L.oracle_find_psi.restype = C.c_uint64
        for name in ("oracle_ntt_fwd", "oracle_ntt_inv"):
            getattr(L, name).argtypes = [_u64p, _u64p, C.c_int, C.c_int, C.c_int]
            getattr(L, name).restype = None
        L.oracle_ntt_naive.argtypes = [_u64p, _u64p, C.c_uint64, C.c_int]
        L.oracle_pointwise.argtypes = [C.c_int, _u64p, _u64p, _u64p, _u64p,
                                       C.c_int, C.c_int, C.c_int]
        L.oracle_automorph_coeff.argtypes = [_u64p, _u64p, C.c_uint64, C.c_int, C.c_uint64]
        L.oracle_automorph_ntt.argtypes = [_u64p, _u64p, C.c_int, C.c_int, C.c_int,
                                           C.c_uint64]
        L.oracle_basis_convert.argtypes = [_u64p, _u64p, C.c_int, _u64p, _u64p,
                                           C.c_int, C.c_int]
        L.oracle_modup.argtypes = [_u64p, _u64p, _u64p, C.c_int, C.c_int, C.c_int,
                                   C.c_int, C.c_int]
        L.oracle_key_inner.argtypes = [_u64p, _u64p, C.c_uint64, _u64p, _u64p,
                                       C.c_int, C.c_int, C.c_int, C.c_int, C.c_int]
        L.oracle_moddown.argtypes = [_u64p, _u64p, _u64p, C.c_int, C.c_int,
                                     C.c_int, C.c_int]
        L.oracle_keyswitch.argtypes = [_u64p, _u64p, _u64p, _u64p, C.c_int, C.c_int,
                                       C.c_int, C.c_int, C.c_int]
        L.oracle_rotate.argtypes = [_u64p, C.POINTER(_u64p), _u64p, C.c_int, _u64p,
                                    _u64p, C.c_int, C.c_int, C.c_int, C.c_int, C.c_int]
        L.oracle_rotate_unhoisted.argtypes = L.oracle_rotate.argtypes
        L.oracle_rescale.argtypes = [_u64p, _u64p, _u64p, C.c_int, C.c_int, C.c_int]
        L.oracle_mul_relin_rescale.argtypes = [_u64p, _u64p, _u64p, _u64p, _u64p,
                                               C.c_int, C.c_int, C.c_int, C.c_int,
                                               C.c_int]
        L.oracle_bsgs.argtypes = [_u64p, _u64p, C.POINTER(_u64p), C.POINTER(_u64p),
                                  C.c_int, C.c_int, _u64p, _u64p, C.c_int, C.c_int,
                                  C.c_int, C.c_int, C.c_int]
        L.oracle_keygen.argtypes = [_i64p, _u64p, _u64p, _i64p, _u64p, _u64p,
                                    C.c_int, C.c_int, C.c_int, C.c_int]
        L.oracle_secret_galois.argtypes = [_i64p, C.c_uint64, _u64p, _u64p, C.c_int,
                                           C.c_int]
        L.oracle_secret_square.argtypes = [_i64p, _u64p, _u64p, C.c_int, C.c_int]
        L.oracle_encrypt.argtypes = [_i64p, _i64p, _u64p, _i64p, _u64p, _u64p,
                                     C.c_int, C.c_int]
        L.oracle_decrypt.argtypes = [_u64p, _i64p, _u64p, _u64p, C.c_int, C.c_int]
        L.oracle_negacyclic_mul.argtypes = [_u64p, _u64p, _u64p, C.c_uint64, C.c_int]
        L.oracle_mul_monomial.argtypes = [_u64p, _u64p, _u64p, C.c_int, C.c_int, C.c_int,
                                          C.c_int]
        L.oracle_modraise.argtypes = [_u64p, _u64p, _u64p, C.c_int, C.c_int, C.c_int, C.c_int]
        L.oracle_conj_extract.argtypes = [_u64p, _u64p, _u64p, _u64p, _u64p, C.c_int,
                                          C.c_int, C.c_int, C.c_int, C.c_int]
        L.oracle_restore_merge.argtypes = [_u64p, _u64p, _u64p, _u64p, C.c_int, C.c_int,
                                           C.c_int]
        L.oracle_num_threads.restype = C.c_int
        L.oracle_set_num_threads.argtypes = [C.c_int]
        L.oracle_set_num_threads.restype = None
    return _LIB


# _u / _i / _ptr_array return the (possibly copied) arrays with their
# pointers; callers keep those arrays bound to a local (named with a leading
# underscore where nothing else reads it) so the memory outlives the C call.
def _u(a):
    a = np.ascontiguousarray(a, dtype=np.uint64)
    return a, a.ctypes.data_as(_u64p)


def _i(a):
    a = np.ascontiguousarray(a, dtype=np.int64)
    return a, a.ctypes.data_as(_i64p)


def _ptr_array(arrs):
    kept = [_u(a) for a in arrs]
    arr = (_u64p * max(1, len(kept)))(*[p for _, p in kept])
    return kept, arr


def num_threads():
    """Threads the oracle's OpenMP loops use."""
    return int(_lib().oracle_num_threads())


def set_num_threads(t):
    """Threads for the oracle's following OpenMP loops (timing only)."""
    _lib().oracle_set_num_threads(int(t))


def digit_count(L, alpha):
    return (L + alpha - 1) // alpha


# ---------------------------------------------------------------- parameters

def is_prime(m):
    return bool(_lib().oracle_is_prime(int(m)))


def gen_primes(n, count):
    """First `count` primes q = 1 mod 2n below 2^60, largest first."""
    out = np.zeros(count, dtype=np.uint64)
    rc = _lib().oracle_gen_primes(n, count, out.ctypes.data_as(_u64p))
    if rc != 0:
        raise ValueError("not enough primes in (2^59, 2^60)")
    return out


def find_psi(q, n):
    return int(_lib().oracle_find_psi(int(q), n))


# ---------------------------------------------------------------- transforms

def ntt_naive(a, q, n):
    a, pa = _u(a)
    out = np.zeros(n, dtype=np.uint64)
    _lib().oracle_ntt_naive(pa, out.ctypes.data_as(_u64p), int(q), n)
    return out


def ntt_fwd(x, mods):
    """Forward NTT of x[..., limbs, n] (copy returned); limb l uses mods[l]."""
    x = np.array(x, dtype=np.uint64, copy=True, order="C")
    limbs, n = x.shape[-2], x.shape[-1]
    batch = x.size // (limbs * n) if x.size else 0
    _m, pm = _u(mods)
    _lib().oracle_ntt_fwd(x.ctypes.data_as(_u64p), pm, limbs, batch, n)
    return x


def ntt_inv(x, mods):
    x = np.array(x, dtype=np.uint64, copy=True, order="C")
    limbs, n = x.shape[-2], x.shape[-1]
    batch = x.size // (limbs * n) if x.size else 0
    _m, pm = _u(mods)
    _lib().oracle_ntt_inv(x.ctypes.data_as(_u64p), pm, limbs, batch, n)
    return x


def pointwise(op, a, b, mods):
    """op in {'mul', 'add', 'sub'}; arrays [..., limbs, n]."""
    code = {"mul": 0, "add": 1, "sub": 2}[op]
    a, pa = _u(a)
    b, pb = _u(b)
    out = np.zeros_like(a)
    limbs, n = a.shape[-2], a.shape[-1]
    _m, pm = _u(mods)
    _lib().oracle_pointwise(code, pa, pb, out.ctypes.data_as(_u64p), pm, limbs,
                            a.size // (limbs * n), n)
    return out


def automorph_coeff(a, q, g):
    a, pa = _u(a)
    out = np.zeros_like(a)
    _lib().oracle_automorph_coeff(pa, out.ctypes.data_as(_u64p), int(q), a.shape[-1], int(g))
    return out


def automorph_ntt(x, g):
    x, px = _u(x)
    out = np.zeros_like(x)
    limbs, n = x.shape[-2], x.shape[-1]
    _lib().oracle_automorph_ntt(px, out.ctypes.data_as(_u64p), limbs,
                                x.size // (limbs * n), n, int(g))
    return out


def negacyclic_mul(a, b, q):
    a, pa = _u(a)
    b, pb = _u(b)
    out = np.zeros_like(a)
    _lib().oracle_negacyclic_mul(pa, pb, out.ctypes.data_as(_u64p), int(q), a.shape[-1])
    return out


# ---------------------------------------------------------------- key switching

def basis_convert(x, src, dst):
    """x[S][n] residues of one integer per coefficient over primes src ->
    approximate residues over primes dst, [T][n] (coefficient domain)."""
    x, px = _u(x)
    s, ps = _u(src)
    d, pd = _u(dst)
    n = x.shape[-1]
    out = np.zeros((len(d), n), dtype=np.uint64)
    _lib().oracle_basis_convert(px, ps, len(s), out.ctypes.data_as(_u64p), pd, len(d), n)
    return out


def modup(c_ntt, mods, L, K, alpha):
    """c_ntt[B][L][n] -> digits[B][dnum][L+K][n] (NTT domain)."""
    c, pc = _u(c_ntt)
    B, n = c.shape[0], c.shape[-1]
    dn = digit_count(L, alpha)
    out = np.zeros((B, dn, L + K, n), dtype=np.uint64)
    _m, pm = _u(mods)
    _lib().oracle_modup(pc, out.ctypes.data_as(_u64p), pm, L, K, alpha, B, n)
    return out


def key_inner(digits, key, galois, mods, L, K, alpha):
    """digits[B][dnum][L+K][n], key[dnum][2][L+K][n] -> acc[B][2][L+K][n]."""
    d, pd = _u(digits)
    _k, pk = _u(key)
    B, n = d.shape[0], d.shape[-1]
    out = np.zeros((B, 2, L + K, n), dtype=np.uint64)
    _m, pm = _u(mods)
    _lib().oracle_key_inner(pd, pk, int(galois), out.ctypes.data_as(_u64p), pm, L, K,
                            alpha, B, n)
    return out


def moddown(acc, mods, L, K):
    """acc[B][2][L+K][n] -> out[B][2][L][n]."""
    a, pa = _u(acc)
    B, n = a.shape[0], a.shape[-1]
    out = np.zeros((B, 2, L, n), dtype=np.uint64)
    _m, pm = _u(mods)
    _lib().oracle_moddown(pa, out.ctypes.data_as(_u64p), pm, L, K, B, n)
    return out


def keyswitch(d, key, mods, L, K, alpha):
    """d[B][L][n] (NTT) -> out[B][2][L][n]."""
    d, pd = _u(d)
    _k, pk = _u(key)
    B, n = d.shape[0], d.shape[-1]
    out = np.zeros((B, 2, L, n), dtype=np.uint64)
    _m, pm = _u(mods)
    _lib().oracle_keyswitch(pd, pk, out.ctypes.data_as(_u64p), pm, L, K, alpha, B, n)
    return out


def rotate(ct, keys, galois, mods, L, K, alpha):
    """ct[B][2][L][n] -> out[nkeys][B][2][L][n] with hoisted ModUp."""
    c, pc = _u(ct)
    B, n = c.shape[0], c.shape[-1]
    _kept, karr = _ptr_array(keys)
    _g, pg = _u(galois)
    out = np.zeros((len(keys), B, 2, L, n), dtype=np.uint64)
    _m, pm = _u(mods)
    _lib().oracle_rotate(pc, karr, pg, len(keys), out.ctypes.data_as(_u64p), pm, L, K,
                         alpha, B, n)
    return out


def rotate_unhoisted(ct, keys, galois, mods, L, K, alpha):
    """ct[B][2][L][n] -> out[nkeys][B][2][L][n], automorphism before the key switch."""
    c, pc = _u(ct)
    B, n = c.shape[0], c.shape[-1]
    _kept, karr = _ptr_array(keys)
    _g, pg = _u(galois)
    out = np.zeros((len(keys), B, 2, L, n), dtype=np.uint64)
    _m, pm = _u(mods)
    _lib().oracle_rotate_unhoisted(pc, karr, pg, len(keys), out.ctypes.data_as(_u64p), pm, L, K,
                                   alpha, B, n)
    return out


def rescale(ct, mods):
    """ct[B][2][l+1][n] -> [B][2][l][n], dividing by mods[l]."""
    c, pc = _u(ct)
    B, lp1, n = c.shape[0], c.shape[2], c.shape[-1]
    out = np.zeros((B, 2, lp1 - 1, n), dtype=np.uint64)
    _m, pm = _u(mods)
    _lib().oracle_rescale(pc, out.ctypes.data_as(_u64p), pm, lp1, B, n)
    return out


def mul_relin_rescale(a, b, rlk, mods, L, K, alpha):
    a, pa = _u(a)
    b, pb = _u(b)
    _r, pr = _u(rlk)
    B, n = a.shape[0], a.shape[-1]
    out = np.zeros((B, 2, L - 1, n), dtype=np.uint64)
    _m, pm = _u(mods)
    _lib().oracle_mul_relin_rescale(pa, pb, pr, out.ctypes.data_as(_u64p), pm, L, K,
                                    alpha, B, n)
    return out


def bsgs(x, diags, baby_keys, giant_keys, bb, gg, mods, L, K, alpha):
    """x[B][2][L][n], diags[gg][bb][L][n] -> y[B][2][L-1][n]."""
    xx, px = _u(x)
    _dg, pd = _u(diags)
    _kb, ab = _ptr_array(baby_keys)
    _kg, ag = _ptr_array(giant_keys)
    B, n = xx.shape[0], xx.shape[-1]
    out = np.zeros((B, 2, L - 1, n), dtype=np.uint64)
    _m, pm = _u(mods)
    _lib().oracle_bsgs(px, pd, ab, ag, bb, gg, out.ctypes.data_as(_u64p), pm, L, K,
                       alpha, B, n)
    return out


# ---------------------------------------------------------------- bootstrapping steps

def mul_monomial(x, e, mods):
    """x[..., limbs, n] (NTT domain) times X^e in Z_q[X]/(X^n + 1), NTT domain."""
    x, px = _u(x)
    out = np.zeros_like(x)
    limbs, n = x.shape[-2], x.shape[-1]
    _m, pm = _u(mods)
    _lib().oracle_mul_monomial(px, out.ctypes.data_as(_u64p), pm, limbs,
                               x.size // (limbs * n), n, int(e))
    return out


def modraise(x, mods_full):
    """x[..., l, n] over mods_full[:l] (NTT domain) -> [..., Lf, n] over all of
    mods_full: each coefficient lifted to its centred value and reduced."""
    x, px = _u(x)
    l, n = x.shape[-2], x.shape[-1]
    Lf = len(mods_full)
    P = x.size // (l * n)
    out = np.zeros(x.shape[:-2] + (Lf, n), dtype=np.uint64)
    _m, pm = _u(mods_full)
    _lib().oracle_modraise(px, out.ctypes.data_as(_u64p), pm, l, Lf, P, n)
    return out


def conj_extract(ct, conj_key, mods, L, K, alpha):
    """ct[B][2][L][n] -> (re, im), each [B][2][L][n], slots 2 Re w and 2 Im w."""
    c, pc = _u(ct)
    _k, pk = _u(conj_key)
    B, n = c.shape[0], c.shape[-1]
    re = np.zeros((B, 2, L, n), dtype=np.uint64)
    im = np.zeros((B, 2, L, n), dtype=np.uint64)
    _m, pm = _u(mods)
    _lib().oracle_conj_extract(pc, pk, re.ctypes.data_as(_u64p), im.ctypes.data_as(_u64p),
                               pm, L, K, alpha, B, n)
    return re, im


def restore_merge(re, im, mods):
    """re, im [B][2][L][n] with slots a, b -> [B][2][L][n] with slots a + i b."""
    r, pr = _u(re)
    _im, pi = _u(im)
    B, L, n = r.shape[0], r.shape[2], r.shape[-1]
    out = np.zeros_like(r)
    _m, pm = _u(mods)
    _lib().oracle_restore_merge(pr, pi, out.ctypes.data_as(_u64p), pm, L, B, n)
    return out


# ---------------------------------------------------------------- keys, enc/dec

def secret_galois(s, g, mods):
    s, ps = _i(s)
    n = s.shape[-1]
    out = np.zeros((len(mods), n), dtype=np.uint64)
    _m, pm = _u(mods)
    _lib().oracle_secret_galois(ps, int(g), out.ctypes.data_as(_u64p), pm, len(_m), n)
    return out


def secret_square(s, mods):
    s, ps = _i(s)
    n = s.shape[-1]
    out = np.zeros((len(mods), n), dtype=np.uint64)
    _m, pm = _u(mods)
    _lib().oracle_secret_square(ps, out.ctypes.data_as(_u64p), pm, len(_m), n)
    return out


def keygen(s, sprime_ntt, a, e, mods, L, K, alpha):
    """Switching key s' -> s: [dnum][2][L+K][n]. a[dnum][L+K][n] uniform NTT
    residues, e[dnum][n] small error coefficients."""
    s, ps = _i(s)
    _sp, psp = _u(sprime_ntt)
    a, pa = _u(a)
    e, pe = _i(e)
    n = s.shape[-1]
    dn = digit_count(L, alpha)
    out = np.zeros((dn, 2, L + K, n), dtype=np.uint64)
    _m, pm = _u(mods)
    _lib().oracle_keygen(ps, psp, pa, pe, out.ctypes.data_as(_u64p), pm, L, K, alpha, n)
    return out


def keygen_galois(s, g, a, e, mods, L, K, alpha):
    return keygen(s, secret_galois(s, g, mods), a, e, mods, L, K, alpha)


def keygen_relin(s, a, e, mods, L, K, alpha):
    return keygen(s, secret_square(s, mods), a, e, mods, L, K, alpha)


def encrypt(m_coeffs, s, a, e, mods):
    """Secret-key encryption of integer coefficients m -> ct[2][L][n]."""
    mm, pm_ = _i(m_coeffs)
    s, ps = _i(s)
    a, pa = _u(a)
    e, pe = _i(e)
    L, n = len(mods), mm.shape[-1]
    out = np.zeros((2, L, n), dtype=np.uint64)
    _m, pm = _u(mods)
    _lib().oracle_encrypt(pm_, ps, pa, pe, out.ctypes.data_as(_u64p), pm, L, n)
    return out


def decrypt(ct, s, mods):
    """ct[2][L][n] -> coefficient residues [L][n] of c0 + c1 s."""
    c, pc = _u(ct)
    s, ps = _i(s)
    L, n = len(mods), c.shape[-1]
    out = np.zeros((L, n), dtype=np.uint64)
    _m, pm = _u(mods)
    _lib().oracle_decrypt(pc, ps, out.ctypes.data_as(_u64p), pm, L, n)
    return out


__all__ = [k for k in dir() if not k.startswith("_")]
