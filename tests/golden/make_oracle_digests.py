"""Writes oracle_digests.json: SHA-256 digests of the oracle's outputs on small
seeded cases.  It calls only `oracle/` and the seeded generators; the digests
guard against an unnoticed change of the oracle's arithmetic (they are not
pins: the pins in test_oracle_pins.py and test_oracle_boot_pins.py decide
what is correct).

    python tests/golden/make_oracle_digests.py        # rewrite the file
"""
import hashlib
import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from rns_ckks_polynomial_b200 import synth  # noqa: E402

N = 2048
SEED = synth.config_seed(0) + 0x600


def _digest(*arrays):
    h = hashlib.sha256()
    for a in arrays:
        a = np.ascontiguousarray(a)
        h.update(str(a.shape).encode())
        h.update(a.astype(np.uint64).tobytes())
    return h.hexdigest()


def _res(shape, mods, stream):
    return np.ascontiguousarray(synth.uniform_residues(shape, mods, SEED, stream).numpy().astype(np.uint64))


def cases():
    """name -> digest of the oracle's output on that case."""
    out = {}
    mods = oracle.gen_primes(N, 8)
    out["gen_primes_2160"] = _digest(oracle.gen_primes(N, 2160))
    out["find_psi_first_8"] = _digest(np.array([oracle.find_psi(int(q), N) for q in mods],
                                               dtype=np.uint64))
    L, K, alpha = 6, 2, 2
    x = _res((2, 3, N), mods[:3], 1)
    out["ntt_fwd_2x3"] = _digest(oracle.ntt_fwd(x, mods[:3]))
    out["ntt_inv_2x3"] = _digest(oracle.ntt_inv(x, mods[:3]))
    a, b = _res((2, L, N), mods[:L], 2), _res((2, L, N), mods[:L], 3)
    out["pointwise_mul_add_sub"] = _digest(*(oracle.pointwise(op, a, b, mods[:L])
                                             for op in ("mul", "add", "sub")))
    out["automorph_ntt_g5_g4095"] = _digest(oracle.automorph_ntt(a, 5), oracle.automorph_ntt(a, 4095))
    dn = (L + alpha - 1) // alpha
    key = _res((dn, 2, L + K, N), mods, 4)
    key2 = _res((dn, 2, L + K, N), mods, 5)
    d = _res((2, L, N), mods[:L], 6)
    dig = oracle.modup(d, mods, L, K, alpha)
    out["modup_6_2_2"] = _digest(dig)
    acc = oracle.key_inner(dig, key, 5, mods, L, K, alpha)
    out["key_inner_g5"] = _digest(acc)
    out["moddown"] = _digest(oracle.moddown(acc, mods, L, K))
    out["keyswitch"] = _digest(oracle.keyswitch(d, key, mods, L, K, alpha))
    ct = _res((2, 2, L, N), mods[:L], 7)
    gal = np.array([5, 25], dtype=np.uint64)
    out["rotate_hoisted_2_keys"] = _digest(oracle.rotate(ct, [key, key2], gal, mods, L, K, alpha))
    out["rotate_unhoisted_2_keys"] = _digest(oracle.rotate_unhoisted(ct, [key, key2], gal, mods, L, K,
                                                                     alpha))
    out["rescale"] = _digest(oracle.rescale(ct, mods[:L]))
    ct2 = _res((2, 2, L, N), mods[:L], 8)
    out["mul_relin_rescale"] = _digest(oracle.mul_relin_rescale(ct, ct2, key, mods, L, K, alpha))
    bb = gg = 2
    pts = _res((gg, bb, L, N), mods[:L], 9)
    out["bsgs_2x2"] = _digest(oracle.bsgs(ct, pts, [key], [key2], bb, gg, mods, L, K, alpha))
    out["modraise_3_to_6"] = _digest(oracle.modraise(_res((2, 2, 3, N), mods[:3], 10), mods[:L]))
    out["mul_monomial_half"] = _digest(oracle.mul_monomial(a, N // 2, mods[:L]))
    re, im = oracle.conj_extract(ct, key, mods, L, K, alpha)
    out["conj_extract"] = _digest(re, im)
    out["restore_merge"] = _digest(oracle.restore_merge(re, im, mods[:L]))
    s = synth.ternary(N, SEED, 11).numpy()
    e = synth.gaussian((dn, N), SEED, 12).numpy()
    out["keygen_galois_5"] = _digest(oracle.keygen_galois(s, 5, key[:, 1].copy(), e, mods, L, K, alpha))
    m = oracle.encode(synth.uniform_real((N // 2,), -1, 1, SEED, 13).numpy(), N, 2**50)
    out["encode"] = _digest(m.astype(np.int64).view(np.uint64))
    enc = oracle.encrypt(m, s, a[0], synth.gaussian((N,), SEED, 14).numpy(), mods[:L])
    out["encrypt_decrypt"] = _digest(enc, oracle.decrypt(enc, s, mods[:L]))
    return out


if __name__ == "__main__":
    path = os.path.join(HERE, "oracle_digests.json")
    with open(path, "w") as f:
        json.dump(cases(), f, indent=1, sort_keys=True)
        f.write("\n")
    print(path)
