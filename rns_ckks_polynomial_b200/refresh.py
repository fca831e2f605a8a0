"""The bootstrapping refresh as a schedule of C-ABI calls (every arithmetic
step runs in the library's kernels; this module only orders the calls and
tracks scales).

The pages name the steps and their times (Kestrel engine write-up, the boot
profile in section 5.3: modraise, coeff_to_slot, conj_extract, sin_fold_re,
sin_fold_im, restore_merge, slot_to_coeff) but give no formulas; the forms
are the textbook ones:

* modraise lifts a ciphertext on q_0 to the whole chain; its slots, read at
  scale q_0, hold m / q_0 + I.
* coeff_to_slot and slot_to_coeff are factored special FFTs, `depth` BSGS
  levels each (ckks_bsgs_lintrans_plan); the caller supplies every level's
  plaintext diagonals, encoded over that level's primes, and its plan
  (stride, t0, bb, gg).  coeff_to_slot's first level carries the factor 1/2
  that conj_extract doubles back; slot_to_coeff's first level carries
  q_0 / (2 pi Delta).
* sin_fold computes sin(2 pi x) = cos(2 pi (x - 1/4)): the angle divided by
  2^r, cos by its Taylor polynomial up to theta^14, then r double-angle steps.
  6 + r levels.
* A real constant c is an integer product by k = round(c S q / s) followed
  by a rescale by q, which sets the scale to S exactly; constants are added
  as round(a s) to component 0.  Ciphertexts are only added at equal level
  and scale.

Each level l runs on its own context (primes q_0..q_{l-1} and the chain's
special primes), all sharing one key set made for the whole chain
(ckks_ctx_set_key_chain) and one workspace, grown to the largest call's need
(the calls run in order on one stream, so reuse is safe; per-context
workspaces would cost tens of GB per level at 2100 primes)."""
import math
from fractions import Fraction

import torch

from .api import OP_BSGS, OP_CONJ_EXTRACT, OP_MODRAISE, OP_MRR, OP_RESCALE, Context

TAYLOR_TERMS = 8


def stage_groups(n, depth):
    """The log2(n/2) butterfly stages of the special FFT in `depth`
    consecutive groups, the later groups at least as long as the earlier."""
    m = (n // 2).bit_length() - 1
    base, extra = divmod(m, depth)
    out, s = [], 1
    for g in range(depth):
        size = base + (1 if g >= depth - extra else 0)
        out.append(list(range(s, s + size)))
        s += size
    return out


def group_plan(n, grp):
    """BSGS plan (stride, t0, bb, gg) of a group of butterfly stages a..b:
    its diagonals sit at stride t, stride = 2^(a-1), |t| <= 2^(b-a+1) - 1,
    taken modulo M = (n/2) / stride (every residue once the window wraps)."""
    S = n // 2
    stride = 1 << (grp[0] - 1)
    M = S // stride
    k = len(grp)
    if 2 ** (k + 1) - 1 >= M:
        t0, T = -(M // 2), M
    else:
        t0, T = -(2 ** k - 1), 2 ** (k + 1) - 1
    bb = 1 << max(0, round(math.log2(math.sqrt(T))))
    return stride, t0, bb, -(-T // bb)


def factored_plans(n, depth):
    """Plans of the coeff_to_slot levels (inverse stages, last group first)
    and of the slot_to_coeff levels (first group first)."""
    groups = stage_groups(n, depth)
    stc = [group_plan(n, g) for g in groups]
    return stc[::-1], stc


def plan_rotations(plans, n):
    """The left-rotation amounts whose Galois keys the plans use."""
    S = n // 2
    out = set()
    for stride, t0, bb, gg in plans:
        out |= {(stride * b) % S for b in range(1, bb)}
        out |= {(stride * (t0 + bb * g)) % S for g in range(gg)}
    return sorted(a for a in out if a)


class Refresh:
    def __init__(self, q, p, alpha, keys, device=0):
        """q: the chain's ciphertext primes q_0..q_{L-1}; p: its special primes;
        keys: 'relin' and 'conj' device tensors and 'rot' {r: tensor}, all in
        the whole chain's key layout."""
        self.q, self.p, self.alpha = [int(v) for v in q], [int(v) for v in p], alpha
        self.L = len(self.q)
        self.keys = keys
        self.device = device
        self._ctx = {}
        self._buf = None
        self._consts = {}

    def _ws(self, ctx, op, batch, aux=0):
        need = max(ctx.workspace_bytes(op, batch, aux), 16)
        if self._buf is None or self._buf.numel() < need:
            self._buf = None
            self._buf = torch.empty(need, dtype=torch.uint8, device=torch.device("cuda", self.device))
        return self._buf

    def ctx(self, l):
        c = self._ctx.get(l)
        if c is None:
            # below alpha primes the one digit is the start of the keys' first digit
            c = Context(self.q[:l], self.p, min(self.alpha, l), device=self.device)
            c.set_key_chain(self.L, (self.L + self.alpha - 1) // self.alpha)
            self._ctx[l] = c
        return c

    def close(self):
        for c in self._ctx.values():
            c.close()
        self._ctx.clear()
        self._buf = None
        self._consts.clear()

    # ------------------------------------------------------------ constants
    def _kvec(self, value, l):
        """The residues of an integer constant modulo q_0..q_{l-1} as a device
        vector, kept for later calls (a refresh issues the same constants every
        time, so repeated refreshes upload nothing)."""
        v = int(value)
        key = (v, l)
        t = self._consts.get(key)
        if t is None:
            t = torch.tensor([v % qi for qi in self.q[:l]], dtype=torch.int64,
                             device=torch.device("cuda", self.device))
            self._consts[key] = t
        return t

    @staticmethod
    def level(ct):
        return ct.shape[-2]

    def drop(self, ct, l):
        return ct[..., :l, :].contiguous()

    def mul_int(self, ct, k):
        l = self.level(ct)
        return self.ctx(l).pointwise_scalar("mul", ct, self._kvec(k, l))

    def add_const(self, ct, a, scale):
        l = self.level(ct)
        out = ct.clone()
        self.ctx(l).add_const_c0(out, self._kvec(round(Fraction(a) * scale), l))
        return out

    def mul_const(self, ct, scale, c, target):
        l = self.level(ct)
        k = round(Fraction(c) * target * self.q[l - 1] / scale)
        cx = self.ctx(l)
        prod = self.mul_int(ct, k)
        return cx.rescale(prod, ws=self._ws(cx, OP_RESCALE, ct.shape[0], l)), Fraction(target)

    def mul(self, a, sa, b, sb):
        l = min(self.level(a), self.level(b))
        a, b = self.drop(a, l), self.drop(b, l)
        cx = self.ctx(l)
        out = cx.mul_relin_rescale(a, b, self.keys["relin"], ws=self._ws(cx, OP_MRR, a.shape[0]))
        return out, Fraction(sa) * Fraction(sb) / self.q[l - 1]

    def add(self, a, sa, b, sb):
        if self.level(a) != self.level(b) or sa != sb:
            raise ValueError("added ciphertexts must share level and scale")
        out = torch.empty_like(a)
        self.ctx(self.level(a)).pointwise("add", a, b, out=out)
        return out, sa

    # ------------------------------------------------------------ steps
    def sin_fold(self, ct, scale, r):
        """Slots x -> sin(2 pi x); 6 + r levels.  Returns (ct, scale)."""
        S = Fraction(2**60)
        w = 2 * math.pi / 2**r
        th, s_th = self.mul_const(ct, scale, w, S)
        th = self.add_const(th, -w / 4, s_th)
        pw = {1: self.mul(th, s_th, th, s_th)}
        pw[2] = self.mul(*pw[1], *pw[1])
        pw[3] = self.mul(*pw[2], *pw[1])
        pw[4] = self.mul(*pw[2], *pw[2])
        pw[5] = self.mul(*pw[4], *pw[1])
        pw[6] = self.mul(*pw[4], *pw[2])
        pw[7] = self.mul(*pw[4], *pw[3])
        top = self.level(pw[7][0])
        acc = None
        for k in range(1, TAYLOR_TERMS):
            a_k = (-1) ** k / math.factorial(2 * k)
            c, s = pw[k]
            term, s_t = self.mul_const(self.drop(c, top), s, a_k, S)
            acc = term if acc is None else self.add(acc, S, term, s_t)[0]
        acc = self.add_const(acc, 1.0, S)
        c, s_c = acc, S
        for _ in range(r):
            c, s_c = self.mul(c, s_c, c, s_c)
            c = self.mul_int(c, 2)
            c = self.add_const(c, -1.0, s_c)
        return c, s_c

    def lintrans(self, ct, scale, levels, pt_scale):
        """levels: [(plan, pts)] applied in turn, one level each; pts a device
        tensor [gg][bb][l][n] over the level's primes."""
        for plan, pts in levels:
            stride, t0, bb, gg = plan
            S = ct.shape[-1] // 2
            l = self.level(ct)
            rot = self.keys["rot"]
            baby = [rot[(stride * b) % S] for b in range(1, bb)]
            giant = [None if G == 0 else rot[G] for G in
                     ((stride * (t0 + bb * g)) % S for g in range(gg))]
            cx = self.ctx(l)
            ct = cx.bsgs_lintrans_plan(ct, pts, baby, giant, plan,
                                       ws=self._ws(cx, OP_BSGS, ct.shape[0], bb * 1000 + gg))
            scale = Fraction(scale) * Fraction(pt_scale) / self.q[l - 1]
        return ct, scale

    def refresh(self, ct_q0, r, cts_levels, stc_levels, mark=None):
        """A ciphertext [B][2][1][n] on q_0 -> (ciphertext, scale), the slots
        back at the message scale.  cts_levels / stc_levels as for lintrans,
        encoded at 2^60 and 2^50.  mark, if given, is called with each step's
        name after its calls are issued (a timing hook: it may record an
        event on the current stream)."""
        mark = mark or (lambda name: None)
        top = self.ctx(self.L)
        ct = top.modraise(ct_q0, ws=self._ws(top, OP_MODRAISE, ct_q0.shape[0], ct_q0.shape[2]))
        mark("modraise")
        ct, scale = self.lintrans(ct, Fraction(self.q[0]), cts_levels, 2**60)
        mark("coeff_to_slot")
        l = self.level(ct)
        cx = self.ctx(l)
        re, im = cx.conj_extract(ct, self.keys["conj"], ws=self._ws(cx, OP_CONJ_EXTRACT, ct.shape[0]))
        mark("conj_extract")
        sre, s_out = self.sin_fold(re, scale, r)
        mark("sin_fold_re")
        sim, _ = self.sin_fold(im, scale, r)
        mark("sin_fold_im")
        merged = self.ctx(self.level(sre)).restore_merge(sre, sim)
        mark("restore_merge")
        out = self.lintrans(merged, s_out, stc_levels, 2**50)
        mark("slot_to_coeff")
        return out
