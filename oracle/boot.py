"""Bootstrapping on the oracle: sin_fold and the whole refresh, composed from
the oracle's integer operations (test infrastructure only).

The pages name the steps of a refresh and their times (Kestrel engine
write-up, the boot profile in section 5.3: modraise, coeff_to_slot,
rotate_k, conj_extract, sin_fold_re, sin_fold_im, restore_merge,
slot_to_coeff) and show a refresh taking a ciphertext to 2083 of 2100 primes,
i.e. 17 levels.  They give no formulas.  The readings used here are the
textbook ones:

* modraise: the ciphertext on q_0 alone is lifted coefficient by coefficient
  to the whole chain (oracle_modraise); its plaintext becomes t = m + q_0 I.
  Its slots are read at scale q_0, so they hold t / q_0 = m / q_0 + I.
* coeff_to_slot: one dense BSGS transform with (1/n) U^H (the factor 1/2 is
  the one conj_extract doubles back), 1 level.
* conj_extract: real and imaginary parts, each slot now t_k / q_0.
* sin_fold: sin(2 pi x) on every slot by the cosine form
  cos(2 pi (x - 1/4)): the angle is divided by 2^r, cos is evaluated by its
  Taylor polynomial up to theta^14 (6 levels), then folded back by r
  double-angle steps cos 2a = 2 cos^2 a - 1 (r levels).  With r = 9 this is
  15 levels, which with the two transforms makes the 17 of the pages' log.
* restore_merge: re + i im.
* slot_to_coeff: one dense BSGS transform with U q_0 / (2 pi Delta), 1 level;
  sin(2 pi t / q_0) = sin(2 pi m / q_0) ~ 2 pi m / q_0 gives back m / Delta.

Scales are tracked exactly as Fractions.  A product by a real constant c is
an integer product by k = round(c S q / s) followed by a rescale by q, which
sets the scale to S exactly (relative error at most 1 / (2k)); constants are
added as round(a s) to every NTT value of c0 (a constant polynomial's NTT is
the constant).  Ciphertexts are only added at equal level and scale.
"""
import math
from fractions import Fraction

import numpy as np

from . import core
from .encoding import lintrans_plaintexts

TAYLOR_TERMS = 8          # cos theta = sum_{k<8} (-1)^k theta^{2k} / (2k)!


class Chain:
    """Primes and keys of one parameter set: q_0..q_{L-1}, p_0..p_{K-1}."""

    def __init__(self, mods, L, K, alpha):
        self.mods = np.ascontiguousarray(np.asarray(mods, dtype=np.uint64))
        self.L, self.K, self.alpha = L, K, alpha

    def q(self, l):
        return int(self.mods[l])

    def mods_at(self, l):
        """q_0..q_{l-1} followed by the special primes."""
        keep = list(range(l)) + list(range(self.L, self.L + self.K))
        return np.ascontiguousarray(self.mods[keep])

    def key_at(self, key, l):
        """A key for level L reduced to level l: the limbs of q_0..q_{l-1} and
        of the special primes, and the first ceil(l / alpha) digits."""
        keep = list(range(l)) + list(range(self.L, self.L + self.K))
        dn = (l + self.alpha - 1) // self.alpha
        return np.ascontiguousarray(key[:dn][:, :, keep])


def level(ct):
    return ct.shape[-2]


def drop(ct, l):
    """Keep q_0..q_{l-1} (exact: a ciphertext mod Q is one mod every divisor)."""
    return np.ascontiguousarray(ct[..., :l, :])


def _const(c, mods, n):
    return np.stack([np.full(n, int(c) % int(q), dtype=np.uint64) for q in mods])


def mul_int(ct, k, chain):
    l, n = level(ct), ct.shape[-1]
    return core.pointwise("mul", ct, np.broadcast_to(_const(k, chain.mods[:l], n), ct.shape).copy(),
                          chain.mods[:l])


def add_const(ct, a, scale, chain):
    """Slots + a (a real): round(a * scale) added to c0."""
    l, n = level(ct), ct.shape[-1]
    out = ct.copy()
    c = _const(round(Fraction(a) * scale), chain.mods[:l], n)
    out[0] = core.pointwise("add", ct[0], c, chain.mods[:l])
    return out


def mul_const(ct, scale, c, target, chain):
    """Slots * c, then rescale: returns (ct one level down, scale = target)."""
    l = level(ct)
    k = round(Fraction(c) * target * chain.q(l - 1) / scale)
    prod = mul_int(ct, k, chain)
    return core.rescale(prod[None], chain.mods[:l])[0], Fraction(target)


def mul(a, sa, b, sb, rlk, chain):
    """ct x ct with relinearisation and rescale, at the lower of the two levels."""
    l = min(level(a), level(b))
    a, b = drop(a, l), drop(b, l)
    out = core.mul_relin_rescale(a[None], b[None], chain.key_at(rlk, l), chain.mods_at(l), l,
                                 chain.K, chain.alpha)[0]
    return out, Fraction(sa) * Fraction(sb) / chain.q(l - 1)


def add(a, sa, b, sb, chain):
    if level(a) != level(b) or sa != sb:
        raise ValueError("added ciphertexts must share level and scale")
    l = level(a)
    return core.pointwise("add", a, b, chain.mods[:l]), sa


def sin_fold(ct, scale, r, rlk, chain):
    """Slots x -> sin(2 pi x) for |x| + 1/4 <= 2^r / (8 pi) * 1.6 (the angle
    after division stays within 0.8).  Consumes 6 + r levels.
    Returns (ct, scale)."""
    S = Fraction(2**60)
    w = 2 * math.pi / 2**r
    th, s_th = mul_const(ct, scale, w, S, chain)
    th = add_const(th, -w / 4, s_th, chain)
    # powers of u = theta^2: u, u^2 at depth 1, 2; u^3, u^4 at 3; u^5..u^7 at 4
    pw = {}
    pw[1] = mul(th, s_th, th, s_th, rlk, chain)
    pw[2] = mul(*pw[1], *pw[1], rlk, chain)
    pw[3] = mul(*pw[2], *pw[1], rlk, chain)
    pw[4] = mul(*pw[2], *pw[2], rlk, chain)
    pw[5] = mul(*pw[4], *pw[1], rlk, chain)
    pw[6] = mul(*pw[4], *pw[2], rlk, chain)
    pw[7] = mul(*pw[4], *pw[3], rlk, chain)
    top = level(pw[7][0])                 # every term is brought here, then one rescale
    acc, s_acc = None, S
    for k in range(1, TAYLOR_TERMS):
        a_k = (-1) ** k / math.factorial(2 * k)
        c, s = pw[k]
        term, s_t = mul_const(drop(c, top), s, a_k, S, chain)
        acc = term if acc is None else add(acc, s_acc, term, s_t, chain)[0]
    acc = add_const(acc, 1.0, s_acc, chain)       # the k = 0 term
    c, s_c = acc, s_acc
    for _ in range(r):                              # cos 2a = 2 cos^2 a - 1
        c, s_c = mul(c, s_c, c, s_c, rlk, chain)
        c = mul_int(c, 2, chain)
        c = add_const(c, -1.0, s_c, chain)
    return c, s_c


def coeff_to_slot_plaintexts(n, bb, gg, mods, pt_scale):
    from .encoding import coeff_to_slot_matrix
    return lintrans_plaintexts(0.5 * coeff_to_slot_matrix(n), bb, gg, mods, pt_scale, n)


def slot_to_coeff_plaintexts(n, bb, gg, mods, pt_scale, q0, delta):
    from .encoding import slot_to_coeff_matrix
    f = q0 / (2 * math.pi * delta)
    return lintrans_plaintexts(f * slot_to_coeff_matrix(n), bb, gg, mods, pt_scale, n)


def lintrans(ct, scale, diags, pt_scale, bb, gg, baby, giant, chain):
    l = level(ct)
    keys = [chain.key_at(k, l) for k in baby + giant]
    y = core.bsgs(ct[None], diags, keys[: bb - 1], keys[bb - 1:], bb, gg, chain.mods_at(l), l,
                  chain.K, chain.alpha)[0]
    return y, Fraction(scale) * Fraction(pt_scale) / chain.q(l - 1)


def rotation_amounts(plan, S):
    """Left-rotation amounts a BSGS plan needs keys for (Galois 5^r each)."""
    stride, t0, bb, gg = plan
    amounts = {(stride * b) % S for b in range(1, bb)}
    amounts |= {(stride * (t0 + bb * g)) % S for g in range(gg)}
    return sorted(a for a in amounts if a)


def bsgs_plan_apply(ct, scale, pts, plan, pt_scale, keys, chain):
    """The integer part of lintrans_planned: pts[g][b] NTT residues over the
    ciphertext's primes (zeros where a diagonal is absent),
    y = Rescale( sum_g Rot_{G_g}( sum_b pts[g][b] * Rot_{stride b}(x) ) ),
    G_g = stride (t0 + bb g) mod n/2.  keys: {r: Galois key of 5^r} over the
    full chain.  The baby rotations share one ModUp (hoisted); a giant step
    with G_g = 0 is not rotated."""
    n = ct.shape[-1]
    S = n // 2
    l = level(ct)
    stride, t0, bb, gg = plan
    mods_l = chain.mods_at(l)
    qs = chain.mods[:l]
    babies = [ct]
    if bb > 1:
        amounts = [(stride * b) % S for b in range(1, bb)]
        gal = np.array([pow(5, a, 2 * n) for a in amounts], dtype=np.uint64)
        rot = core.rotate(ct[None], [chain.key_at(keys[a], l) for a in amounts], gal, mods_l, l,
                          chain.K, chain.alpha)
        babies += [rot[i, 0] for i in range(len(amounts))]
    acc = None
    for g in range(gg):
        inner = None
        for b in range(bb):
            pt = pts[g][b]
            if pt is None:
                continue
            prod = core.pointwise("mul", babies[b], np.broadcast_to(pt, babies[b].shape).copy(), qs)
            inner = prod if inner is None else core.pointwise("add", inner, prod, qs)
        if inner is None:
            continue
        G = (stride * (t0 + bb * g)) % S
        if G:
            gal = np.array([pow(5, G, 2 * n)], dtype=np.uint64)
            inner = core.rotate(inner[None], [chain.key_at(keys[G], l)], gal, mods_l, l, chain.K,
                                chain.alpha)[0, 0]
        acc = inner if acc is None else core.pointwise("add", acc, inner, qs)
    out = core.rescale(acc[None], qs)[0]
    return out, Fraction(scale) * Fraction(pt_scale) / chain.q(l - 1)


def lintrans_planned(ct, scale, Dg, plan, pt_scale, keys, chain):
    """y = sum_g Rot_{G_g}( sum_b pt_{g,b} * Rot_{stride b}(x) ), then one
    rescale, for a matrix in diagonal form with plan (stride, t0, bb, gg)
    (encoding.bsgs_plan); the plaintexts come from encoding.plan_plaintexts
    and absent diagonals are skipped."""
    from .encoding import plan_plaintexts
    n = ct.shape[-1]
    l = level(ct)
    pts, _ = plan_plaintexts(Dg, plan, n // 2, chain.mods[:l], pt_scale, n)
    return bsgs_plan_apply(ct, scale, pts, plan, pt_scale, keys, chain)


def lintrans_factored(ct, scale, factors, pt_scale, keys, chain, first_factor_scalar=1.0):
    """Apply diagonal forms F_1, F_2, ... in turn (one level each); the scalar
    multiplies F_1's diagonals."""
    from .encoding import bsgs_plan
    S = ct.shape[-1] // 2
    for i, F in enumerate(factors):
        if i == 0 and first_factor_scalar != 1.0:
            F = {k: first_factor_scalar * d for k, d in F.items()}
        ct, scale = lintrans_planned(ct, scale, F, bsgs_plan(F, S), pt_scale, keys, chain)
    return ct, scale


def factored_rotation_amounts(n, depth):
    """Every rotation the factored coeff_to_slot and slot_to_coeff of this
    depth use (the two share their diagonal offsets)."""
    from .encoding import bsgs_plan, factored_coeff_to_slot, factored_slot_to_coeff
    S = n // 2
    out = set()
    for F in factored_coeff_to_slot(n, depth) + factored_slot_to_coeff(n, depth):
        out |= set(rotation_amounts(bsgs_plan(F, S), S))
    return sorted(out)


def bootstrap_factored(ct_q0, delta, r, depth, keys, chain):
    """bootstrap() with coeff_to_slot and slot_to_coeff as `depth` factored
    levels each (slots in bit-reversed order in between, which the slot-wise
    steps do not mind).  keys: 'rot' {r: key of 5^r} for
    factored_rotation_amounts(n, depth), 'conj', 'relin'.  Uses
    2 depth + 6 + r levels."""
    from .encoding import factored_coeff_to_slot, factored_slot_to_coeff
    n = ct_q0.shape[-1]
    q0 = chain.q(0)
    ct = core.modraise(ct_q0, chain.mods[: chain.L])
    ct, scale = lintrans_factored(ct, Fraction(q0), factored_coeff_to_slot(n, depth), 2**60,
                                  keys["rot"], chain, first_factor_scalar=0.5)
    l = level(ct)
    re, im = core.conj_extract(ct[None], chain.key_at(keys["conj"], l), chain.mods_at(l), l,
                               chain.K, chain.alpha)
    sre, s_out = sin_fold(re[0], scale, r, keys["relin"], chain)
    sim, _ = sin_fold(im[0], scale, r, keys["relin"], chain)
    merged = core.restore_merge(sre[None], sim[None], chain.mods[: level(sre)])[0]
    f = q0 / (2 * math.pi * delta)
    return lintrans_factored(merged, s_out, factored_slot_to_coeff(n, depth), 2**50, keys["rot"],
                             chain, first_factor_scalar=f)


def refresh_with_levels(ct_q0, r, cts_levels, stc_levels, keys, chain):
    """The refresh of bootstrap_factored with every transform level given as
    (plan, pts), pts[g][b] the level's plaintexts as NTT residues over its
    primes (zeros where a diagonal is absent): coeff_to_slot's at scale 2^60,
    slot_to_coeff's at 2^50.  The integer function of the refresh for any
    plaintexts, so a parity test can feed seeded residues.  Returns
    (ct, scale)."""
    ct = core.modraise(ct_q0, chain.mods[: chain.L])
    scale = Fraction(chain.q(0))
    for plan, pts in cts_levels:
        ct, scale = bsgs_plan_apply(ct, scale, pts, plan, 2**60, keys["rot"], chain)
    l = level(ct)
    re, im = core.conj_extract(ct[None], chain.key_at(keys["conj"], l), chain.mods_at(l), l,
                               chain.K, chain.alpha)
    sre, s_out = sin_fold(re[0], scale, r, keys["relin"], chain)
    sim, _ = sin_fold(im[0], scale, r, keys["relin"], chain)
    ct = core.restore_merge(sre[None], sim[None], chain.mods[: level(sre)])[0]
    scale = s_out
    for plan, pts in stc_levels:
        ct, scale = bsgs_plan_apply(ct, scale, pts, plan, 2**50, keys["rot"], chain)
    return ct, scale


def bootstrap(ct_q0, delta, r, keys, chain, bb, gg):
    """Refresh a ciphertext on q_0 holding slots z at scale `delta`
    (delta well below q_0).  `keys` holds 'baby', 'giant' (Galois keys for
    5^b and 5^{bb g}), 'conj' (2n - 1) and 'relin', all for the full chain.
    Returns (ct, scale) with slots ~ z, 2 + 6 + r levels below the top."""
    n = ct_q0.shape[-1]
    q0 = chain.q(0)
    ct = core.modraise(ct_q0, chain.mods[: chain.L])
    scale = Fraction(q0)
    cts_scale = Fraction(2**60)
    l = level(ct)
    ct, scale = lintrans(ct, scale, coeff_to_slot_plaintexts(n, bb, gg, chain.mods[:l], 2**60),
                         cts_scale, bb, gg, keys["baby"], keys["giant"], chain)
    l = level(ct)
    re, im = core.conj_extract(ct[None], chain.key_at(keys["conj"], l), chain.mods_at(l), l,
                               chain.K, chain.alpha)
    sre, s_out = sin_fold(re[0], scale, r, keys["relin"], chain)
    sim, _ = sin_fold(im[0], scale, r, keys["relin"], chain)
    merged = core.restore_merge(sre[None], sim[None], chain.mods[: level(sre)])[0]
    stc_scale = 2**50
    l = level(merged)
    diags = slot_to_coeff_plaintexts(n, bb, gg, chain.mods[:l], stc_scale, q0, delta)
    return lintrans(merged, s_out, diags, stc_scale, bb, gg, keys["baby"], keys["giant"], chain)


__all__ = ["Chain", "drop", "mul_int", "add_const", "mul_const", "mul", "add", "sin_fold",
           "coeff_to_slot_plaintexts", "slot_to_coeff_plaintexts", "lintrans", "bootstrap",
           "rotation_amounts", "bsgs_plan_apply", "lintrans_planned", "lintrans_factored",
           "factored_rotation_amounts", "bootstrap_factored", "refresh_with_levels",
           "TAYLOR_TERMS"]
