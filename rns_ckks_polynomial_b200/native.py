"""ctypes declarations for libckks_b200.so (the C ABI in include/ckks.h).

Loading only maps the library (it links the CUDA runtime statically, so this
works on a machine without a GPU); every compute call needs a CUDA device.
There is no fallback: a missing library raises immediately.
"""
import ctypes as C
import os

from . import build as _build

_LIB = None
_u64p = C.POINTER(C.c_uint64)
_vp = C.c_void_p

# every function the header declares: name -> (restype, argtypes)
SIGNATURES = {
    "ckks_primes": (C.c_int, [C.c_int, C.c_int, _u64p]),
    "ckks_ctx_create": (C.c_int, [_u64p, C.c_int, _u64p, C.c_int, C.c_int, C.c_int, C.c_int,
                                  C.POINTER(_vp)]),
    "ckks_ctx_destroy": (None, [_vp]),
    "ckks_last_error": (C.c_char_p, []),
    "ckks_ctx_params": (C.c_int, [_vp] + [C.POINTER(C.c_int)] * 5),
    "ckks_device_status": (C.c_int, [_vp]),
    "ckks_ctx_set_conversion": (C.c_int, [_vp, C.c_int]),
    "ckks_ctx_set_key_chain": (C.c_int, [_vp, C.c_int]),
    "ckks_selftest_wait_expiry": (C.c_int, [_vp]),
    "ckks_workspace_bytes": (C.c_size_t, [_vp, C.c_int, C.c_int, C.c_int]),
    "ckks_ntt_fwd": (C.c_int, [_vp, _vp, C.c_int, C.c_int, C.c_int, _vp]),
    "ckks_ntt_inv": (C.c_int, [_vp, _vp, C.c_int, C.c_int, C.c_int, _vp]),
    "ckks_ntt_fwd_group": (C.c_int, [_vp, C.POINTER(_vp), C.POINTER(C.c_int), C.POINTER(C.c_int),
                                     C.POINTER(C.c_int), C.c_int, _vp]),
    "ckks_ntt_inv_group": (C.c_int, [_vp, C.POINTER(_vp), C.POINTER(C.c_int), C.POINTER(C.c_int),
                                     C.POINTER(C.c_int), C.c_int, _vp]),
    "ckks_pointwise": (C.c_int, [_vp, C.c_int, _vp, _vp, _vp, C.c_int, C.c_int, C.c_int, _vp]),
    "ckks_pointwise_scalar": (C.c_int, [_vp, C.c_int, _vp, _vp, _vp, C.c_int, C.c_int, C.c_int, _vp]),
    "ckks_add_const_c0": (C.c_int, [_vp, _vp, _vp, C.c_int, _vp]),
    "ckks_mul_i": (C.c_int, [_vp, _vp, _vp, C.c_int, C.c_int, C.c_int, _vp]),
    "ckks_conj_extract": (C.c_int, [_vp, _vp, _vp, _vp, _vp, C.c_int, _vp, _vp]),
    "ckks_restore_merge": (C.c_int, [_vp, _vp, _vp, _vp, C.c_int, _vp]),
    "ckks_modraise": (C.c_int, [_vp, _vp, C.c_int, _vp, C.c_int, _vp, _vp]),
    "ckks_automorph": (C.c_int, [_vp, _vp, _vp, C.c_int, C.c_int, C.c_uint32, _vp]),
    "ckks_modup": (C.c_int, [_vp, _vp, _vp, C.c_int, _vp, _vp]),
    "ckks_modup_noalloc": (C.c_int, [_vp, _vp, _vp, C.c_int, _vp]),
    "ckks_key_inner": (C.c_int, [_vp, _vp, _vp, C.c_uint32, _vp, C.c_int, _vp]),
    "ckks_moddown": (C.c_int, [_vp, _vp, _vp, C.c_int, _vp, _vp]),
    "ckks_keyswitch": (C.c_int, [_vp, _vp, _vp, _vp, C.c_int, _vp, _vp]),
    "ckks_rotate": (C.c_int, [_vp, _vp, C.POINTER(_vp), C.POINTER(C.c_uint32), C.c_int, _vp,
                              C.c_int, _vp, _vp]),
    "ckks_rotate_unhoisted": (C.c_int, [_vp, _vp, C.POINTER(_vp), C.POINTER(C.c_uint32), C.c_int, _vp,
                              C.c_int, _vp, _vp]),
    "ckks_rotate_streamed": (C.c_int, [_vp, _vp, C.POINTER(_vp), C.POINTER(C.c_uint32), C.c_int, _vp,
                             C.c_int, _vp, _vp]),
    "ckks_rescale": (C.c_int, [_vp, _vp, _vp, C.c_int, C.c_int, _vp, _vp]),
    "ckks_mul_relin_rescale": (C.c_int, [_vp, _vp, _vp, _vp, _vp, C.c_int, _vp, _vp]),
    "ckks_bsgs_lintrans": (C.c_int, [_vp, _vp, _vp, C.POINTER(_vp), C.POINTER(_vp), C.c_int,
                                     C.c_int, _vp, C.c_int, _vp, _vp]),
    "ckks_bsgs_lintrans_plan": (C.c_int, [_vp, _vp, _vp, C.POINTER(_vp), C.POINTER(_vp), C.c_int,
                                          C.c_int, C.c_int, C.c_int, _vp, C.c_int, _vp, _vp]),
    "ckks_bench_intpipe": (C.c_int, [_vp, C.c_int, C.c_int, C.c_int, C.POINTER(C.c_double),
                                     C.POINTER(C.c_double)]),
}


class CkksError(RuntimeError):
    def __init__(self, name, code, msg):
        super().__init__("%s failed (%d): %s" % (name, code, msg))
        self.code = code


def library_path():
    return _build.LIB


def lib():
    """The loaded library; raises if it has not been built."""
    global _LIB
    if _LIB is None:
        path = _build.LIB
        if not os.path.exists(path):
            raise RuntimeError(
                "libckks_b200.so is not built (expected at %s); run "
                "`python -m rns_ckks_polynomial_b200.build`" % path)
        L = C.CDLL(path)
        for name, (res, args) in SIGNATURES.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _LIB = L
    return _LIB


def check(name, rc):
    if rc != 0:
        msg = lib().ckks_last_error()
        raise CkksError(name, rc, msg.decode() if msg else "")
