"""Host-side checks of the C-ABI library that need no GPU: it loads, exports
every symbol the header declares, and its host logic (prime scan, argument
validation before any launch) behaves as documented."""
import ctypes as C
import os
import re

import pytest

from rns_ckks_polynomial_b200 import native, primes
from rns_ckks_polynomial_b200.native import CkksError

from .helpers import N

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ckks.h")

EINVAL, EUNSUPPORTED = -1, -2


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(ckks_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_hot_path():
    names = declared_functions()
    for must in ["ckks_ntt_fwd", "ckks_ntt_inv", "ckks_automorph", "ckks_modup", "ckks_moddown",
                 "ckks_keyswitch", "ckks_rotate", "ckks_mul_relin_rescale", "ckks_bsgs_lintrans",
                 "ckks_rescale", "ckks_pointwise", "ckks_key_inner"]:
        assert must in names


def test_library_exports_every_declared_symbol():
    lib = native.lib()
    for name in declared_functions():
        assert hasattr(lib, name), name
        assert name in native.SIGNATURES, name


def test_library_path_is_in_tree():
    assert native.library_path().startswith(ROOT)


def test_product_primes_match_oracle(orc):
    assert primes(300) == [int(x) for x in orc.gen_primes(N, 300)]
    # the whole boot chain: 2100 ciphertext and 60 special primes
    assert primes(2160) == [int(x) for x in orc.gen_primes(N, 2160)]


def test_primes_argument_checks():
    with pytest.raises(CkksError) as e:
        primes(3, n=1000)
    assert e.value.code == EINVAL
    assert primes(0) == []


def _create(q, p, alpha, n=N):
    lib = native.lib()
    qa = (C.c_uint64 * max(1, len(q)))(*q)
    pa = (C.c_uint64 * max(1, len(p)))(*p)
    h = C.c_void_p()
    rc = lib.ckks_ctx_create(qa, len(q), pa, len(p), alpha, n, 0, C.byref(h))
    return rc, lib.ckks_last_error().decode()


def test_ctx_create_rejects_bad_parameters():
    good = primes(6)
    # not 2048
    assert _create(good[:4], good[4:5], 1, n=4096)[0] == EUNSUPPORTED
    # alpha out of range, K out of range
    assert _create(good[:4], good[4:5], 5)[0] == EUNSUPPORTED
    assert _create(good[:4], [], 1)[0] == EUNSUPPORTED
    # composite with q = 1 mod 2n
    comp = good[0] + 2 * N
    while all(comp % d for d in (3, 5, 7, 11, 13)):
        comp += 2 * N
    rc, msg = _create([comp] + good[1:4], good[4:5], 1)
    assert rc == EINVAL and "prime 0" in msg
    # prime but not 1 mod 2n
    rc, _ = _create([1152921504606846883] + good[1:4], good[4:5], 1)  # 2^60 - 93
    assert rc == EINVAL
    # at or above 2^60
    rc, _ = _create([2**60 + 1] + good[1:4], good[4:5], 1)
    assert rc == EINVAL
    # duplicates
    rc, msg = _create(good[:4], good[:1], 1)
    assert rc == EINVAL and "distinct" in msg


def test_calls_reject_null_context():
    lib = native.lib()
    assert lib.ckks_ntt_fwd(None, None, 1, 0, 1, None) == EINVAL
    assert lib.ckks_keyswitch(None, None, None, None, 1, None, None) == EINVAL
    assert lib.ckks_workspace_bytes(None, 1, 1, 0) == 0
    assert "null context" in lib.ckks_last_error().decode()
    assert lib.ckks_ctx_set_conversion(None, 1) == EINVAL
    assert lib.ckks_ctx_set_key_chain(None, 5) == EINVAL
    assert lib.ckks_selftest_wait_expiry(None) == EINVAL


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    """Without the compiled library every call raises; nothing falls back to
    a CPU path."""
    from rns_ckks_polynomial_b200 import Context
    ps = primes(4)
    monkeypatch.setattr(native, "_LIB", None)
    monkeypatch.setattr(native._build, "LIB", str(tmp_path / "absent.so"))
    with pytest.raises(RuntimeError, match="not built"):
        native.lib()
    with pytest.raises(RuntimeError, match="not built"):
        Context(ps[:3], ps[3:], 1)
    with pytest.raises(RuntimeError, match="not built"):
        primes(4)
