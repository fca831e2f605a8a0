"""Python binding of the C ABI: argument marshalling only.

Tensors are torch int64 (or uint64) CUDA tensors holding uint64 residues in
the limb-major layout of include/ckks.h; every call runs on the current torch
CUDA stream of the tensor's device.  Outputs and workspaces are allocated with
torch when the caller does not pass them.  All arithmetic happens in the CUDA
library; nothing here computes on the data.
"""
import ctypes as C

import torch

from .native import check, lib

N = 2048

PW = {"mul": 0, "add": 1, "sub": 2}
OP_MODUP, OP_MODDOWN, OP_KEYSWITCH, OP_ROTATE, OP_RESCALE, OP_MRR, OP_BSGS = 1, 2, 3, 4, 5, 6, 7
OP_ROTATE_UNHOISTED = 8
OP_MODRAISE, OP_CONJ_EXTRACT = 9, 10
OP_ROTATE_STREAMED = 11


def primes(count, n=N):
    """First `count` primes q = 1 mod 2n in (2^59, 2^60), largest first (host)."""
    out = (C.c_uint64 * max(1, count))()
    check("ckks_primes", lib().ckks_primes(n, count, out))
    return [int(out[i]) for i in range(count)]


def _ptr(t, name, shape=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError("%s must be a torch tensor" % name)
    if t.dtype not in (torch.int64, torch.uint64):
        raise TypeError("%s must be int64/uint64 residues" % name)
    if not t.is_cuda:
        raise ValueError("%s must be a CUDA tensor" % name)
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError("%s has shape %s, expected %s" % (name, tuple(t.shape), tuple(shape)))
    return C.c_void_p(t.data_ptr())


def _stream(t):
    return C.c_void_p(torch.cuda.current_stream(t.device).cuda_stream)


class Context:
    """Owns a ckks_ctx: primes q (L) and p (K), digit size alpha."""

    def __init__(self, q, p, alpha, device=0, n=N):
        self.q, self.p = [int(x) for x in q], [int(x) for x in p]
        self.L, self.K, self.alpha, self.n = len(self.q), len(self.p), int(alpha), n
        self.dnum = (self.L + self.alpha - 1) // self.alpha
        self.device = torch.device("cuda", device)
        qa = (C.c_uint64 * self.L)(*self.q)
        pa = (C.c_uint64 * max(1, self.K))(*self.p)
        h = C.c_void_p()
        check("ckks_ctx_create",
              lib().ckks_ctx_create(qa, self.L, pa, self.K, self.alpha, n, device, C.byref(h)))
        self._h = h

    @property
    def mods(self):
        return self.q + self.p

    def close(self):
        if getattr(self, "_h", None):
            lib().ckks_ctx_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def device_status(self):
        """Synchronise the device and raise if a bounded device wait expired."""
        check("ckks_device_status", lib().ckks_device_status(self._h))

    def selftest_wait_expiry(self):
        """Launch the bounded-wait expiry self-test; device_status() then raises."""
        check("ckks_selftest_wait_expiry", lib().ckks_selftest_wait_expiry(self._h))

    CONVERSION = {"auto": 0, "integer": 1, "tensor": 2, "folded": 3}

    @property
    def _kshape(self):
        """Shape of a switching key for this context: [dnum][2][L+K][n], or the
        longer chain's layout after set_key_chain."""
        kl = getattr(self, "key_L", self.L)
        dn = getattr(self, "key_dnum", None) or (kl + self.alpha - 1) // self.alpha
        return (dn, 2, kl + self.K, self.n)

    def set_key_chain(self, key_L, key_dnum=None):
        """Keys passed from now on were made for a chain of key_L >= L
        ciphertext primes with the same special primes, in key_dnum digits
        (default ceil(key_L / alpha)) whose first blocks cover this context's
        digits: one key set made at the top level serves the context of every
        lower level."""
        check("ckks_ctx_set_key_chain", lib().ckks_ctx_set_key_chain(self._h, int(key_L)))
        self.key_L = int(key_L)
        self.key_dnum = None if key_dnum is None else int(key_dnum)

    def set_conversion(self, engine):
        """Where ModUp/ModDown basis conversions run: "auto" (the folded tensor-core
        form from 8 source primes on, else the integer pipes), "integer" (integer
        pipes), "tensor" (int8 tensor cores, byte planes of both operands) or
        "folded" (int8 tensor cores, the data's byte weights folded into the
        matrix).  Results are bit-identical."""
        check("ckks_ctx_set_conversion",
              lib().ckks_ctx_set_conversion(self._h, self.CONVERSION.get(engine, -1)
                                            if isinstance(engine, str) else int(engine)))

    # ------------------------------------------------------------ helpers
    def _empty(self, *shape):
        return torch.empty(shape, dtype=torch.int64, device=self.device)

    def workspace_bytes(self, op, batch, aux=0):
        return int(lib().ckks_workspace_bytes(self._h, op, batch, aux))

    def _ws(self, ws, op, batch, aux=0):
        need = self.workspace_bytes(op, batch, aux)
        if ws is None:
            ws = torch.empty(max(need, 16), dtype=torch.uint8, device=self.device)
        elif ws.numel() * ws.element_size() < need:
            raise ValueError("workspace too small: %d < %d bytes" % (ws.numel() * ws.element_size(), need))
        return ws, C.c_void_p(ws.data_ptr())

    # ------------------------------------------------------------ a1/a2
    def ntt_fwd(self, x, limb_begin=0):
        """In place over x[..., limbs, n]."""
        limbs = x.shape[-2]
        batch = x.numel() // (limbs * self.n) if x.numel() else 0
        check("ckks_ntt_fwd", lib().ckks_ntt_fwd(self._h, _ptr(x, "x"), batch, limb_begin, limbs,
                                                 _stream(x)))
        return x

    def ntt_inv(self, x, limb_begin=0):
        limbs = x.shape[-2]
        batch = x.numel() // (limbs * self.n) if x.numel() else 0
        check("ckks_ntt_inv", lib().ckks_ntt_inv(self._h, _ptr(x, "x"), batch, limb_begin, limbs,
                                                 _stream(x)))
        return x

    def _group(self, name, xs, limb_begins):
        xs = list(xs)
        begins = list(limb_begins) if limb_begins is not None else [0] * len(xs)
        if len(begins) != len(xs):
            raise ValueError("one limb_begin per tensor")
        g = len(xs)
        ptrs = (C.c_void_p * max(1, g))(*[_ptr(x, "x").value for x in xs])
        limbs = [x.shape[-2] for x in xs]
        batch = [x.numel() // (l * self.n) if x.numel() else 0 for x, l in zip(xs, limbs)]
        arr = lambda v: (C.c_int * max(1, g))(*v)  # noqa: E731
        stream = _stream(xs[0]) if xs else None
        check(name, getattr(lib(), name)(self._h, ptrs, arr(batch), arr(begins), arr(limbs), g, stream))
        return xs

    def ntt_fwd_group(self, xs, limb_begins=None):
        """Forward NTT of every tensor x[..., limbs, n] of `xs` in place, in one launch."""
        return self._group("ckks_ntt_fwd_group", xs, limb_begins)

    def ntt_inv_group(self, xs, limb_begins=None):
        """Inverse NTT of every tensor of `xs` in place, in one launch."""
        return self._group("ckks_ntt_inv_group", xs, limb_begins)

    # ------------------------------------------------------------ a3/a4
    def pointwise(self, op, a, b, out=None, limb_begin=0):
        out = torch.empty_like(a) if out is None else out
        limbs = a.shape[-2]
        batch = a.numel() // (limbs * self.n) if a.numel() else 0
        for t, nm in ((b, "b"), (out, "out")):
            if t.shape != a.shape:
                raise ValueError("%s shape mismatch" % nm)
        check("ckks_pointwise", lib().ckks_pointwise(self._h, PW[op], _ptr(a, "a"), _ptr(b, "b"),
                                                     _ptr(out, "out"), batch, limb_begin, limbs,
                                                     _stream(a)))
        return out

    def automorph(self, x, galois, out=None):
        out = torch.empty_like(x) if out is None else out
        limbs = x.shape[-2]
        batch = x.numel() // (limbs * self.n) if x.numel() else 0
        check("ckks_automorph", lib().ckks_automorph(self._h, _ptr(x, "in"), _ptr(out, "out"), batch,
                                                     limbs, int(galois), _stream(x)))
        return out

    # ------------------------------------------------------------ a5-a7
    def modup(self, c, out=None, ws=None):
        B = c.shape[0]
        _ptr(c, "c_ntt", (B, self.L, self.n))
        out = self._empty(B, self.dnum, self.L + self.K, self.n) if out is None else out
        ws, wp = self._ws(ws, OP_MODUP, B)
        check("ckks_modup", lib().ckks_modup(self._h, _ptr(c, "c"), _ptr(out, "digits"), B, wp,
                                             _stream(c)))
        return out

    def modup_noalloc(self, c, out):
        """ModUp whose scratch is the library's static device array: nothing
        is allocated (the caller provides `out`, [B][dnum][L+K][n]).  Limit:
        B * L <= 2048."""
        B = c.shape[0]
        _ptr(c, "c_ntt", (B, self.L, self.n))
        _ptr(out, "digits", (B, self.dnum, self.L + self.K, self.n))
        check("ckks_modup_noalloc", lib().ckks_modup_noalloc(self._h, _ptr(c, "c"), _ptr(out, "digits"),
                                                             B, _stream(c)))
        return out

    def key_inner(self, digits, key, galois=1, out=None):
        B = digits.shape[0]
        LK = self.L + self.K
        _ptr(digits, "digits", (B, self.dnum, LK, self.n))
        _ptr(key, "key", self._kshape)
        out = self._empty(B, 2, LK, self.n) if out is None else out
        check("ckks_key_inner", lib().ckks_key_inner(self._h, _ptr(digits, "digits"), _ptr(key, "key"),
                                                     int(galois), _ptr(out, "acc"), B,
                                                     _stream(digits)))
        return out

    def moddown(self, acc, out=None, ws=None):
        B = acc.shape[0]
        _ptr(acc, "acc", (B, 2, self.L + self.K, self.n))
        out = self._empty(B, 2, self.L, self.n) if out is None else out
        ws, wp = self._ws(ws, OP_MODDOWN, B)
        check("ckks_moddown", lib().ckks_moddown(self._h, _ptr(acc, "acc"), _ptr(out, "out"), B, wp,
                                                 _stream(acc)))
        return out

    def keyswitch(self, d, key, out=None, ws=None):
        B = d.shape[0]
        _ptr(d, "d", (B, self.L, self.n))
        _ptr(key, "key", self._kshape)
        out = self._empty(B, 2, self.L, self.n) if out is None else out
        ws, wp = self._ws(ws, OP_KEYSWITCH, B)
        check("ckks_keyswitch", lib().ckks_keyswitch(self._h, _ptr(d, "d"), _ptr(key, "key"),
                                                     _ptr(out, "out"), B, wp, _stream(d)))
        return out

    # ------------------------------------------------------------ a8
    def rotate(self, ct, keys, galois, out=None, ws=None):
        B = ct.shape[0]
        nk = len(keys)
        _ptr(ct, "ct", (B, 2, self.L, self.n))
        kp = (C.c_void_p * max(1, nk))(*[_ptr(k, "key", self._kshape).value
                                        for k in keys])
        gp = (C.c_uint32 * max(1, nk))(*[int(g) for g in galois])
        out = self._empty(nk, B, 2, self.L, self.n) if out is None else out
        ws, wp = self._ws(ws, OP_ROTATE, B, nk)
        check("ckks_rotate", lib().ckks_rotate(self._h, _ptr(ct, "ct"), kp, gp, nk, _ptr(out, "out"),
                                               B, wp, _stream(ct)))
        return out

    def rotate_streamed(self, ct, keys, galois, out=None, ws=None):
        """The hoisted rotations of rotate(), word for word, with ModUp -> NTT -> inner product
        streamed over windows of at most 60 primes (no [B][dnum][L+K][n] digit tensor)."""
        B = ct.shape[0]
        nk = len(keys)
        _ptr(ct, "ct", (B, 2, self.L, self.n))
        kp = (C.c_void_p * max(1, nk))(*[_ptr(k, "key", self._kshape).value
                                        for k in keys])
        gp = (C.c_uint32 * max(1, nk))(*[int(g) for g in galois])
        out = self._empty(nk, B, 2, self.L, self.n) if out is None else out
        ws, wp = self._ws(ws, OP_ROTATE_STREAMED, B, nk)
        check("ckks_rotate_streamed",
              lib().ckks_rotate_streamed(self._h, _ptr(ct, "ct"), kp, gp, nk, _ptr(out, "out"), B, wp,
                                         _stream(ct)))
        return out

    def rotate_unhoisted(self, ct, keys, galois, out=None, ws=None):
        """Rotations in the other order: phi_g before ModUp, one ModUp per key."""
        B = ct.shape[0]
        nk = len(keys)
        _ptr(ct, "ct", (B, 2, self.L, self.n))
        kp = (C.c_void_p * max(1, nk))(*[_ptr(k, "key", self._kshape).value
                                        for k in keys])
        gp = (C.c_uint32 * max(1, nk))(*[int(g) for g in galois])
        out = self._empty(nk, B, 2, self.L, self.n) if out is None else out
        ws, wp = self._ws(ws, OP_ROTATE_UNHOISTED, B)
        check("ckks_rotate_unhoisted",
              lib().ckks_rotate_unhoisted(self._h, _ptr(ct, "ct"), kp, gp, nk, _ptr(out, "out"), B, wp,
                                          _stream(ct)))
        return out

    # ------------------------------------------------------------ a9/a10
    def rescale(self, ct, out=None, ws=None):
        B, _, lp1, _ = ct.shape
        out = self._empty(B, 2, lp1 - 1, self.n) if out is None else out
        ws, wp = self._ws(ws, OP_RESCALE, B, lp1)
        check("ckks_rescale", lib().ckks_rescale(self._h, _ptr(ct, "ct"), _ptr(out, "out"), lp1, B, wp,
                                                 _stream(ct)))
        return out

    def mul_relin_rescale(self, a, b, rlk, out=None, ws=None):
        B = a.shape[0]
        _ptr(a, "a", (B, 2, self.L, self.n))
        _ptr(b, "b", (B, 2, self.L, self.n))
        _ptr(rlk, "rlk", self._kshape)
        out = self._empty(B, 2, self.L - 1, self.n) if out is None else out
        ws, wp = self._ws(ws, OP_MRR, B)
        check("ckks_mul_relin_rescale",
              lib().ckks_mul_relin_rescale(self._h, _ptr(a, "a"), _ptr(b, "b"), _ptr(rlk, "rlk"),
                                           _ptr(out, "out"), B, wp, _stream(a)))
        return out

    # ------------------------------------------------------------ a11
    def bsgs_lintrans(self, x, diags, baby_keys, giant_keys, bb, gg, out=None, ws=None):
        B = x.shape[0]
        _ptr(x, "x", (B, 2, self.L, self.n))
        _ptr(diags, "diags", (gg, bb, self.L, self.n))
        kshape = self._kshape
        if len(baby_keys) != bb - 1 or len(giant_keys) != gg - 1:
            raise ValueError("need bb-1 baby keys and gg-1 giant keys")
        bk = (C.c_void_p * max(1, bb - 1))(*[_ptr(k, "baby key", kshape).value for k in baby_keys])
        gk = (C.c_void_p * max(1, gg - 1))(*[_ptr(k, "giant key", kshape).value for k in giant_keys])
        out = self._empty(B, 2, self.L - 1, self.n) if out is None else out
        ws, wp = self._ws(ws, OP_BSGS, B, bb * 1000 + gg)
        check("ckks_bsgs_lintrans",
              lib().ckks_bsgs_lintrans(self._h, _ptr(x, "x"), _ptr(diags, "diags"), bk, gk, bb, gg,
                                       _ptr(out, "y"), B, wp, _stream(x)))
        return out

    def bsgs_lintrans_plan(self, x, diags, baby_keys, giant_keys, plan, out=None, ws=None):
        """The BSGS transform over a strided window of diagonals, plan =
        (stride, t0, bb, gg): baby_keys rotate by stride b (b = 1..bb-1),
        giant_keys[g] by stride (t0 + bb g) mod n/2 (None where that is 0)."""
        stride, t0, bb, gg = (int(v) for v in plan)
        B = x.shape[0]
        _ptr(x, "x", (B, 2, self.L, self.n))
        _ptr(diags, "diags", (gg, bb, self.L, self.n))
        kshape = self._kshape
        if len(baby_keys) != bb - 1 or len(giant_keys) != gg:
            raise ValueError("need bb-1 baby keys and gg giant keys")
        bk = (C.c_void_p * max(1, bb - 1))(*[_ptr(k, "baby key", kshape).value for k in baby_keys])
        gk = (C.c_void_p * gg)(*[None if k is None else _ptr(k, "giant key", kshape).value
                                 for k in giant_keys])
        out = self._empty(B, 2, self.L - 1, self.n) if out is None else out
        ws, wp = self._ws(ws, OP_BSGS, B, bb * 1000 + gg)
        check("ckks_bsgs_lintrans_plan",
              lib().ckks_bsgs_lintrans_plan(self._h, _ptr(x, "x"), _ptr(diags, "diags"), bk, gk, stride,
                                            t0, bb, gg, _ptr(out, "y"), B, wp, _stream(x)))
        return out

    # ------------------------------------------------------------ refresh building blocks
    def pointwise_scalar(self, op, a, k, out=None, limb_begin=0):
        """out = a op k[limb] over a[..., limbs, n]; k: device int64 tensor of
        `limbs` residues."""
        out = torch.empty_like(a) if out is None else out
        limbs = a.shape[-2]
        batch = a.numel() // (limbs * self.n) if a.numel() else 0
        _ptr(k, "k", (limbs,))
        check("ckks_pointwise_scalar",
              lib().ckks_pointwise_scalar(self._h, PW[op], _ptr(a, "a"), _ptr(k, "k"), _ptr(out, "out"),
                                          batch, limb_begin, limbs, _stream(a)))
        return out

    def add_const_c0(self, ct, k):
        """In place: component 0 of every ciphertext of ct[B][2][L][n] plus k[limb]."""
        B = ct.shape[0]
        _ptr(ct, "ct", (B, 2, self.L, self.n))
        _ptr(k, "k", (self.L,))
        check("ckks_add_const_c0", lib().ckks_add_const_c0(self._h, _ptr(ct, "ct"), _ptr(k, "k"), B,
                                                           _stream(ct)))
        return ct

    def mul_i(self, x, out=None, limb_begin=0):
        """X^{n/2} x (every slot times i) over x[..., limbs, n], NTT domain."""
        out = torch.empty_like(x) if out is None else out
        limbs = x.shape[-2]
        batch = x.numel() // (limbs * self.n) if x.numel() else 0
        check("ckks_mul_i", lib().ckks_mul_i(self._h, _ptr(x, "in"), _ptr(out, "out"), batch, limb_begin,
                                             limbs, _stream(x)))
        return out

    def conj_extract(self, ct, conj_key, ws=None):
        """ct[B][2][L][n] -> (re, im) with slots 2 Re w and 2 Im w."""
        B = ct.shape[0]
        _ptr(ct, "ct", (B, 2, self.L, self.n))
        _ptr(conj_key, "conj_key", self._kshape)
        re, im = self._empty(B, 2, self.L, self.n), self._empty(B, 2, self.L, self.n)
        ws, wp = self._ws(ws, OP_CONJ_EXTRACT, B)
        check("ckks_conj_extract",
              lib().ckks_conj_extract(self._h, _ptr(ct, "ct"), _ptr(conj_key, "conj_key"), _ptr(re, "re"),
                                      _ptr(im, "im"), B, wp, _stream(ct)))
        return re, im

    def restore_merge(self, re, im, out=None):
        """re + X^{n/2} im over [B][2][L][n]: slots a + i b."""
        B = re.shape[0]
        _ptr(re, "re", (B, 2, self.L, self.n))
        _ptr(im, "im", (B, 2, self.L, self.n))
        out = torch.empty_like(re) if out is None else out
        check("ckks_restore_merge", lib().ckks_restore_merge(self._h, _ptr(re, "re"), _ptr(im, "im"),
                                                             _ptr(out, "out"), B, _stream(re)))
        return out

    def modraise(self, x, out=None, ws=None):
        """x[B][2][l][n] over q_0..q_{l-1} -> [B][2][L][n], each coefficient
        lifted to its centred value and reduced modulo every prime."""
        B, _, l, _ = x.shape
        out = self._empty(B, 2, self.L, self.n) if out is None else out
        ws, wp = self._ws(ws, OP_MODRAISE, B, l)
        check("ckks_modraise", lib().ckks_modraise(self._h, _ptr(x, "in"), l, _ptr(out, "out"), B, wp,
                                                   _stream(x)))
        return out

    # ------------------------------------------------------------ measurement
    def bench_intpipe(self, kind, blocks, iters):
        """(ms, ops) of the microbenchmark `kind`: 0 Shoup mulmod, 1 64x64->128
        MAC, 2 64-bit high multiply, 3 / 4 int8 tcgen05.mma at N = 256 / 32,
        5 the forward NTT's butterfly, 6 the key inner product's split-form
        product (primes 2^60 - delta only)."""
        ms, ops = C.c_double(), C.c_double()
        check("ckks_bench_intpipe",
              lib().ckks_bench_intpipe(self._h, kind, blocks, iters, C.byref(ms), C.byref(ops)))
        return ms.value, ops.value
