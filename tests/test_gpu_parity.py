"""Bit-exact parity of every C-ABI call against the CPU oracle, on the GPU.

All integer RNS tensors must match word for word.  Keys and ciphertexts for
the small and layer-shaped cases come from the oracle's keygen/encryption so
that decryption can be checked too; at the full boot-level sizes keys and
ciphertexts are seeded uniform residues (the integer function is the same,
and the decryption pins run at the smaller sizes).
"""
import ctypes as C

import numpy as np
import pytest
import torch

from rns_ckks_polynomial_b200 import native, synth
from rns_ckks_polynomial_b200.native import CkksError

from .gpu_common import assert_bits_equal, context, ctx_for, dev, gpu, host, need_gpu
from .helpers import N, SCALE, SLOTS, Params, Scheme, galois_for_rotation, rot_left, u64

pytestmark = gpu

SEED = synth.config_seed(1)


@pytest.fixture(autouse=True)
def _gpu():
    need_gpu()
    yield
    torch.cuda.synchronize()
    torch.cuda.empty_cache()


def _res(shape, mods, stream, seed=SEED):
    return u64(synth.uniform_residues(shape, mods, seed, stream))


# ------------------------------------------------------------------ config 1
def test_config1_tiny_pipeline(orc):
    """4 + 1 primes, alpha = 1: 8 polynomials -> NTT -> pairwise product ->
    INTT, and one rotation key switch with the Galois-5 key."""
    p = Params(4, 1, 1)
    ctx = ctx_for(p)
    sch = Scheme(orc, p, SEED)
    q = sch.q
    polys = _res((8, 4, N), q, 1)
    x = dev(polys)
    ctx.ntt_fwd(x)
    want = orc.ntt_fwd(polys, q)
    assert_bits_equal(host(x), want, "ntt_fwd")
    prod = ctx.pointwise("mul", x[0::2].contiguous(), x[1::2].contiguous())
    want_p = orc.pointwise("mul", want[0::2], want[1::2], q)
    assert_bits_equal(host(prod), want_p, "pointwise mul")
    ctx.ntt_inv(prod)
    assert_bits_equal(host(prod), orc.ntt_inv(want_p, q), "ntt_inv")
    # rotation key switch on (P0, P1) in the NTT domain
    key = sch.keygen_galois(5)
    ct = want[0:2][None]
    out = ctx.rotate(dev(ct), [dev(key)], [5])
    want_r = orc.rotate(ct, [key], np.array([5], dtype=np.uint64), sch.mods, 4, 1, 1)
    assert_bits_equal(host(out), want_r, "rotate")


def test_config1_rotation_decrypts(orc):
    p = Params(4, 1, 1)
    ctx = ctx_for(p)
    sch = Scheme(orc, p, SEED + 1)
    z = synth.uniform_real((SLOTS,), -1, 1, SEED, 3).numpy()
    ct = sch.encrypt_slots(z)
    key = sch.keygen_galois(5)
    out = host(ctx.rotate(dev(ct[None]), [dev(key)], [5]))
    assert np.max(np.abs(sch.decrypt_slots(out[0, 0]) - rot_left(z, 1))) < 1e-8


# ------------------------------------------------------------------ NTT (config 2)
@pytest.mark.parametrize("limbs,batch,begin", [(3, 16, 0), (112, 16, 0), (5, 3, 7), (1, 1, 2159),
                                               (512, 16, 0)])
def test_ntt_roundtrip_and_parity(orc, limbs, batch, begin):
    ctx = context(2100, 60, 60)
    mods = np.array(ctx.mods[begin:begin + limbs], dtype=np.uint64)
    a = _res((batch, limbs, N), mods, 10 + limbs)
    x = dev(a)
    ctx.ntt_fwd(x, limb_begin=begin)
    assert_bits_equal(host(x), orc.ntt_fwd(a, mods), "ntt_fwd")
    ctx.ntt_inv(x, limb_begin=begin)
    assert_bits_equal(host(x), a, "ntt round trip")
    y = dev(a)
    ctx.ntt_inv(y, limb_begin=begin)
    assert_bits_equal(host(y), orc.ntt_inv(a, mods), "ntt_inv")


def test_ntt_full_sweep_2100(orc):
    """The bench's largest sweep entry: 16 x 2100 limbs, every limb checked."""
    ctx = context(2100, 60, 60)
    mods = np.array(ctx.q, dtype=np.uint64)
    a = synth.uniform_residues((16, 2100, N), mods, SEED, 20, device="cuda")
    x = a.clone()
    ctx.ntt_fwd(x)
    want = orc.ntt_fwd(host(a), mods)
    assert_bits_equal(host(x), want, "ntt_fwd 2100")
    ctx.ntt_inv(x)
    assert torch.equal(x, a)


def test_ntt_group_matches_single_launches(orc):
    """One grouped launch over tensors of 3, 112, 512 and 5 limbs (different batches, one at an odd
    limb_begin, one empty) gives every tensor the oracle's forward transform, and the grouped
    inverse brings them back; more than 8 groups is rejected."""
    ctx = context(2100, 60, 60)
    shapes = [(16, 3, 0), (4, 112, 0), (2, 512, 40), (3, 5, 2155), (0, 7, 0)]
    arrs = [_res((b, l, N), np.array(ctx.mods[s0:s0 + l], dtype=np.uint64), 700 + i) if b else
            np.zeros((0, l, N), dtype=np.uint64) for i, (b, l, s0) in enumerate(shapes)]
    xs = [dev(a) for a in arrs]
    begins = [s0 for _, _, s0 in shapes]
    ctx.ntt_fwd_group(xs, begins)
    for (b, l, s0), a, x in zip(shapes, arrs, xs):
        want = orc.ntt_fwd(a, np.array(ctx.mods[s0:s0 + l], dtype=np.uint64)) if b else a
        assert_bits_equal(host(x), want, "grouped ntt_fwd %d x %d at %d" % (b, l, s0))
    ctx.ntt_inv_group(xs, begins)
    for a, x in zip(arrs, xs):
        assert_bits_equal(host(x), a, "grouped round trip")
    lib = native.lib()
    ptrs = (C.c_void_p * 9)(*([xs[0].data_ptr()] * 9))
    ints = (C.c_int * 9)(*([1] * 9))
    assert lib.ckks_ntt_fwd_group(ctx._h, ptrs, ints, (C.c_int * 9)(*([0] * 9)), ints, 9, None) == -1


def test_ntt_empty_and_errors():
    ctx = context(4, 1, 1)
    e = torch.empty((0, 4, N), dtype=torch.int64, device="cuda")
    ctx.ntt_fwd(e)
    x = torch.zeros((1, 4, N), dtype=torch.int64, device="cuda")
    with pytest.raises(CkksError) as err:
        ctx.ntt_fwd(x, limb_begin=2)  # 2 + 4 > L + K = 5
    assert err.value.code == -1
    buf = torch.zeros(4 * N + 1, dtype=torch.int64, device="cuda")
    lib = native.lib()
    rc = lib.ckks_ntt_fwd(ctx._h, C.c_void_p(buf.data_ptr() + 8), 1, 0, 4, None)
    assert rc == -1 and "aligned" in lib.ckks_last_error().decode()



def test_key_switch_calls_accept_empty_inputs():
    """An empty batch (or no keys) is a no-op for every key-switching call: each returns CKKS_OK with
    null data pointers, so it reads, writes and launches nothing; a negative batch is CKKS_EINVAL."""
    ctx = context(20, 3, 7)
    lib = native.lib()
    h, nul = ctx._h, None
    no_keys = (C.c_void_p * 1)()
    no_gal = (C.c_uint32 * 1)()
    calls = {
        "modup": lambda b: lib.ckks_modup(h, nul, nul, b, nul, nul),
        "modup_noalloc": lambda b: lib.ckks_modup_noalloc(h, nul, nul, b, nul),
        "key_inner": lambda b: lib.ckks_key_inner(h, nul, nul, 5, nul, b, nul),
        "moddown": lambda b: lib.ckks_moddown(h, nul, nul, b, nul, nul),
        "keyswitch": lambda b: lib.ckks_keyswitch(h, nul, nul, nul, b, nul, nul),
        "rotate": lambda b: lib.ckks_rotate(h, nul, no_keys, no_gal, 1, nul, b, nul, nul),
        "rotate_unhoisted": lambda b: lib.ckks_rotate_unhoisted(h, nul, no_keys, no_gal, 1, nul, b, nul, nul),
        "rotate_streamed": lambda b: lib.ckks_rotate_streamed(h, nul, no_keys, no_gal, 1, nul, b, nul, nul),
        "rescale": lambda b: lib.ckks_rescale(h, nul, nul, 20, b, nul, nul),
        "mul_relin_rescale": lambda b: lib.ckks_mul_relin_rescale(h, nul, nul, nul, nul, b, nul, nul),
        "bsgs_lintrans": lambda b: lib.ckks_bsgs_lintrans(h, nul, nul, None, None, 1, 1, nul, b, nul, nul),
    }
    for name, call in calls.items():
        assert call(0) == 0, (name, lib.ckks_last_error())
        assert call(-1) == -1, name
    for fn in (lib.ckks_rotate, lib.ckks_rotate_unhoisted, lib.ckks_rotate_streamed):
        assert fn(h, nul, no_keys, no_gal, 0, nul, 3, nul, nul) == 0  # no keys, a non-empty batch
    torch.cuda.synchronize()
    ctx.device_status()

# ------------------------------------------------------------------ pointwise / automorphism
@pytest.mark.parametrize("op", ["mul", "add", "sub"])
def test_pointwise(orc, op):
    ctx = context(112, 8, 8)
    mods = np.array(ctx.mods[:112], dtype=np.uint64)
    a, b = _res((3, 112, N), mods, 30), _res((3, 112, N), mods, 31)
    out = ctx.pointwise(op, dev(a), dev(b))
    assert_bits_equal(host(out), orc.pointwise(op, a, b, mods), op)


@pytest.mark.parametrize("g", [5, 25, 625, 1505, 4095, 3])
def test_automorph(orc, g):
    ctx = context(112, 8, 8)
    mods = np.array(ctx.mods[:7], dtype=np.uint64)
    a = _res((2, 7, N), mods, 40)
    out = ctx.automorph(dev(a), g)
    assert_bits_equal(host(out), orc.automorph_ntt(a, g), "automorph %d" % g)


def test_automorph_rejects_even_and_in_place():
    ctx = context(4, 1, 1)
    x = torch.zeros((1, 4, N), dtype=torch.int64, device="cuda")
    with pytest.raises(CkksError):
        ctx.automorph(x, 4)
    with pytest.raises(CkksError):
        ctx.automorph(x, 5, out=x)


# ------------------------------------------------------------------ key switching stages
@pytest.mark.parametrize("L,K,alpha", [(4, 1, 1), (6, 2, 2), (5, 2, 2), (112, 8, 8), (20, 3, 7),
                                       (40, 20, 20), (70, 33, 33), (130, 64, 64)])
def test_modup_inner_moddown_stages(orc, L, K, alpha):
    """Every stage on every conversion engine (integer pipes, int8 tensor cores,
    and the automatic choice, which takes the tensor cores from 8 source
    primes on); (70, 33, 33) has a ragged 4-prime last digit."""
    p = Params(L, K, alpha)
    ctx = ctx_for(p)
    mods = np.array(ctx.mods, dtype=np.uint64)
    c = _res((2, L, N), mods[:L], 50)
    key = _res((p.dnum, 2, L + K, N), mods, 51)
    want_d = orc.modup(c, mods, L, K, alpha)
    want_a = {g: orc.key_inner(want_d, key, g, mods, L, K, alpha) for g in (1, 5, 4095)}
    want_m = orc.moddown(want_a[4095], mods, L, K)
    want_k = orc.keyswitch(c, key, mods, L, K, alpha)
    try:
        for engine in ("integer", "tensor", "auto"):
            ctx.set_conversion(engine)
            dig = ctx.modup(dev(c))
            assert_bits_equal(host(dig), want_d, "modup (%s)" % engine)
            for g in (1, 5, 4095):
                acc = ctx.key_inner(dig, dev(key), g)
                assert_bits_equal(host(acc), want_a[g], "key_inner g=%d" % g)
            out = ctx.moddown(acc)
            assert_bits_equal(host(out), want_m, "moddown (%s)" % engine)
            ks = ctx.keyswitch(dev(c), dev(key))
            assert_bits_equal(host(ks), want_k, "keyswitch (%s)" % engine)
            ctx.device_status()
    finally:
        ctx.set_conversion("auto")


def test_set_conversion_rejects_unknown_engine():
    ctx = ctx_for(Params(4, 1, 1))
    with pytest.raises(CkksError):
        ctx.set_conversion(7)
    with pytest.raises(CkksError):
        ctx.set_conversion("fast")


def test_hoisted_rotations_match_and_decrypt(orc):
    p = Params(5, 2, 2)
    ctx = ctx_for(p)
    sch = Scheme(orc, p, SEED + 2)
    zs = [synth.uniform_real((SLOTS,), -1, 1, SEED, 60 + i).numpy() for i in range(3)]
    cts = np.stack([sch.encrypt_slots(z) for z in zs])
    rs = [1, 2, 5, 33]
    keys = [sch.keygen_galois(galois_for_rotation(r)) for r in rs]
    gal = [galois_for_rotation(r) for r in rs]
    out = host(ctx.rotate(dev(cts), [dev(k) for k in keys], gal))
    want = orc.rotate(cts, keys, np.array(gal, dtype=np.uint64), sch.mods, p.L, p.K, p.alpha)
    assert_bits_equal(out, want, "rotate")
    for i, r in enumerate(rs):
        for b in range(3):
            assert np.max(np.abs(sch.decrypt_slots(out[i, b]) - rot_left(zs[b], r))) < 1e-8


def test_tensor_core_rotation_decrypts(orc):
    """Rotation with 20-prime digits and 20 special primes (tensor-core ModUp
    and ModDown) decrypts to the slot rotation."""
    p = Params(40, 20, 20)
    ctx = ctx_for(p)
    sch = Scheme(orc, p, SEED + 7)
    z = synth.uniform_real((SLOTS,), -1, 1, SEED, 77).numpy()
    ct = sch.encrypt_slots(z)
    g = galois_for_rotation(3)
    key = sch.keygen_galois(g)
    out = host(ctx.rotate(dev(ct[None]), [dev(key)], [g]))
    ctx.device_status()
    assert_bits_equal(out, orc.rotate(ct[None], [key], np.array([g], dtype=np.uint64), sch.mods,
                                      p.L, p.K, p.alpha), "rotate")
    assert np.max(np.abs(sch.decrypt_slots(out[0, 0]) - rot_left(z, 3))) < 1e-8


def test_rotate_context_owned_workspace(orc):
    """ws = NULL makes the context allocate its own workspace."""
    p = Params(4, 1, 1)
    ctx = ctx_for(p)
    mods = np.array(ctx.mods, dtype=np.uint64)
    ct = _res((2, 2, 4, N), mods[:4], 70)
    key = _res((4, 2, 5, N), mods, 71)
    ref = host(ctx.rotate(dev(ct), [dev(key)], [25]))
    out = torch.empty((1, 2, 2, 4, N), dtype=torch.int64, device="cuda")
    keep = dev(key)
    kp = (C.c_void_p * 1)(keep.data_ptr())
    gp = (C.c_uint32 * 1)(25)
    ctd = dev(ct)
    lib = native.lib()
    rc = lib.ckks_rotate(ctx._h, C.c_void_p(ctd.data_ptr()), kp, gp, 1, C.c_void_p(out.data_ptr()),
                         2, None, None)
    assert rc == 0
    torch.cuda.synchronize()
    assert_bits_equal(host(out), ref, "rotate (own workspace)")


# ------------------------------------------------------------------ rescale, ct x ct
@pytest.mark.parametrize("lp1,batch", [(5, 3), (112, 2), (2, 1)])
def test_rescale(orc, lp1, batch):
    ctx = context(112, 8, 8)
    mods = np.array(ctx.mods[:lp1], dtype=np.uint64)
    ct = _res((batch, 2, lp1, N), mods, 80 + lp1)
    out = ctx.rescale(dev(ct))
    assert_bits_equal(host(out), orc.rescale(ct, mods), "rescale")


def test_mul_relin_rescale_small_decrypts(orc):
    p = Params(6, 2, 2)
    ctx = ctx_for(p)
    sch = Scheme(orc, p, SEED + 3)
    za = [synth.uniform_real((SLOTS,), -1, 1, SEED, 90 + i).numpy() for i in range(2)]
    zb = [synth.uniform_real((SLOTS,), -1, 1, SEED, 95 + i).numpy() for i in range(2)]
    ca = np.stack([sch.encrypt_slots(z) for z in za])
    cb = np.stack([sch.encrypt_slots(z) for z in zb])
    rlk = sch.keygen_relin()
    out = host(ctx.mul_relin_rescale(dev(ca), dev(cb), dev(rlk)))
    assert_bits_equal(out, orc.mul_relin_rescale(ca, cb, rlk, sch.mods, p.L, p.K, p.alpha), "mrr")
    sc = sch.rescaled_scale(SCALE * SCALE, p.L)
    for i in range(2):
        assert np.max(np.abs(sch.decrypt_slots(out[i], sc) - za[i] * zb[i])) < 1e-8


def test_config3_layer_multiply(orc):
    """112 primes, alpha = 8, 8 special primes; 8 ciphertext pairs."""
    p = Params(112, 8, 8)
    ctx = ctx_for(p)
    sch = Scheme(orc, p, synth.config_seed(3))
    za = [synth.uniform_real((SLOTS,), -1, 1, synth.config_seed(3), 100 + i).numpy() for i in range(8)]
    zb = [synth.uniform_real((SLOTS,), -1, 1, synth.config_seed(3), 200 + i).numpy() for i in range(8)]
    ca = np.stack([sch.encrypt_slots(z) for z in za])
    cb = np.stack([sch.encrypt_slots(z) for z in zb])
    rlk = sch.keygen_relin()
    out = host(ctx.mul_relin_rescale(dev(ca), dev(cb), dev(rlk)))
    want = orc.mul_relin_rescale(ca, cb, rlk, sch.mods, p.L, p.K, p.alpha)
    assert_bits_equal(out, want, "config 3")
    sc = sch.rescaled_scale(SCALE * SCALE, p.L)
    for i in (0, 7):
        assert np.max(np.abs(sch.decrypt_slots(out[i], sc) - za[i] * zb[i])) < 1e-8


# ------------------------------------------------------------------ BSGS
def test_bsgs_banded_decrypts(orc):
    from .test_oracle_pins import bsgs_plaintexts
    p = Params(6, 2, 2)
    bb = gg = 4
    ctx = ctx_for(p)
    sch = Scheme(orc, p, SEED + 5)
    rng_m = synth.uniform_real((SLOTS, SLOTS), -1 / 32, 1 / 32, SEED, 110).numpy()
    idx = np.arange(SLOTS)
    M = np.zeros((SLOTS, SLOTS))
    for k in range(bb * gg):
        M[idx, (idx + k) % SLOTS] = rng_m[idx, (idx + k) % SLOTS]
    xs = [synth.uniform_real((SLOTS,), -1, 1, SEED, 111 + i).numpy() for i in range(2)]
    ct = np.stack([sch.encrypt_slots(x) for x in xs])
    diags = bsgs_plaintexts(orc, M, bb, gg, sch.q)
    baby = [sch.keygen_galois(galois_for_rotation(b)) for b in range(1, bb)]
    giant = [sch.keygen_galois(galois_for_rotation(bb * g)) for g in range(1, gg)]
    y = host(ctx.bsgs_lintrans(dev(ct), dev(diags), [dev(k) for k in baby],
                               [dev(k) for k in giant], bb, gg))
    want = orc.bsgs(ct, diags, baby, giant, bb, gg, sch.mods, p.L, p.K, p.alpha)
    assert_bits_equal(y, want, "bsgs")
    sc = sch.rescaled_scale(SCALE * SCALE, p.L)
    for i in range(2):
        assert np.max(np.abs(sch.decrypt_slots(y[i], sc) - M @ xs[i])) < 1e-8


@pytest.mark.parametrize("bb,gg", [(3, 5), (1, 2), (2, 1), (33, 2)])
def test_bsgs_shapes(orc, bb, gg):
    p = Params(5, 2, 2)
    ctx = ctx_for(p)
    mods = np.array(ctx.mods, dtype=np.uint64)
    x = _res((2, 2, 5, N), mods[:5], 120)
    diags = _res((gg, bb, 5, N), mods[:5], 121)
    baby = [_res((3, 2, 7, N), mods, 122 + i) for i in range(bb - 1)]
    giant = [_res((3, 2, 7, N), mods, 140 + i) for i in range(gg - 1)]
    y = host(ctx.bsgs_lintrans(dev(x), dev(diags), [dev(k) for k in baby], [dev(k) for k in giant],
                               bb, gg))
    assert_bits_equal(y, orc.bsgs(x, diags, baby, giant, bb, gg, mods, 5, 2, 2), "bsgs %dx%d" % (bb, gg))


@pytest.mark.parametrize("bb,gg", [(9, 3), (33, 2)])
def test_bsgs_extreme_residues(orc, bb, gg):
    """Every diagonal word, key word and the words of ciphertext 0 at q - 1, ciphertext 1 alternating
    q - 1 with 0: the inner sums over 9 baby values (split sums folded after 8 and after 1 term, 4
    components per CTA) and 33 (2 per CTA) at their largest, bit-exact against the oracle."""
    L, K, alpha = 5, 2, 2
    p = Params(L, K, alpha)
    ctx = ctx_for(p)
    mods = np.array(ctx.mods, dtype=np.uint64)
    ext = _extremes(mods[:L])
    x = np.ascontiguousarray(np.stack([np.stack([ext[1], ext[1]]), np.stack([ext[2], ext[2][:, ::-1]])]))
    top = lambda shape, m: np.ascontiguousarray(np.broadcast_to((m - 1)[:, None], shape), dtype=np.uint64)
    diags = top((gg, bb, L, N), mods[:L])
    key = top((p.dnum, 2, L + K, N), mods)
    y = host(ctx.bsgs_lintrans(dev(x), dev(diags), [dev(key)] * (bb - 1), [dev(key)] * (gg - 1), bb, gg))
    ctx.device_status()
    want = orc.bsgs(x, diags, [key] * (bb - 1), [key] * (gg - 1), bb, gg, mods, L, K, alpha)
    assert_bits_equal(y, want, "bsgs %dx%d, extreme words" % (bb, gg))


def test_config4_bsgs_full_size(orc):
    """112 primes, alpha = 8, bb = gg = 32, 62 keys, 8 ciphertexts of seeded
    uniform residues: the GPU runs the batch, the oracle recomputes every
    ciphertext."""
    p = Params(112, 8, 8)
    ctx = ctx_for(p)
    seed = synth.config_seed(4)
    mods = np.array(ctx.mods, dtype=np.uint64)
    kshape = (p.dnum, 2, 120, N)
    x = synth.uniform_residues((8, 2, 112, N), mods[:112], seed, 1, device="cuda")
    diags = synth.uniform_residues((32, 32, 112, N), mods[:112], seed, 2, device="cuda")
    baby = [synth.uniform_residues(kshape, mods, seed, 100 + i, device="cuda") for i in range(31)]
    giant = [synth.uniform_residues(kshape, mods, seed, 200 + i, device="cuda") for i in range(31)]
    y = ctx.bsgs_lintrans(x, diags, baby, giant, 32, 32)
    ctx.device_status()
    want = orc.bsgs(host(x), host(diags), [host(k) for k in baby], [host(k) for k in giant],
                    32, 32, mods, 112, 8, 8)
    assert_bits_equal(host(y), want, "config 4, all 8 ciphertexts")


def test_config4_dense_matrix_decrypts(orc):
    """Config 4 as stated: a dense 1024 x 1024 matrix with entries uniform in
    [-1, 1]/32, its 1024 diagonals encoded at scale 2^60 (pre-rotated for the
    giant steps), 8 encryptions of slots uniform in [-1, 1], and the 62
    Galois keys of bb = gg = 32 from the oracle's key generation.  All 8
    outputs decrypt to M x within 1e-8 of the float64 product; ciphertexts 0
    and 7 are bit-exact against the oracle."""
    p = Params(112, 8, 8)
    ctx = ctx_for(p)
    seed = synth.config_seed(4) + 500
    sch = Scheme(orc, p, seed)
    bb = gg = 32
    M = synth.uniform_real((SLOTS, SLOTS), -1 / 32, 1 / 32, seed, 1).numpy()
    xs = [synth.uniform_real((SLOTS,), -1, 1, seed, 10 + i).numpy() for i in range(8)]
    ct = np.stack([sch.encrypt_slots(x) for x in xs])
    idx = np.arange(SLOTS)
    rows = np.stack([np.roll(M[idx, (idx + bb * g + b) % SLOTS], bb * g)
                     for g in range(gg) for b in range(bb)])
    diags = orc.encode_ntt_many(rows, sch.q, SCALE, N).reshape(gg, bb, p.L, N)
    baby = [sch.keygen_galois(galois_for_rotation(b)) for b in range(1, bb)]
    giant = [sch.keygen_galois(galois_for_rotation(bb * g)) for g in range(1, gg)]
    y = host(ctx.bsgs_lintrans(dev(ct), dev(diags), [dev(k) for k in baby],
                               [dev(k) for k in giant], bb, gg))
    ctx.device_status()
    sc = sch.rescaled_scale(SCALE * SCALE, p.L)
    for i in range(8):
        err = np.max(np.abs(sch.decrypt_slots(y[i], sc) - M @ xs[i]))
        assert err < 1e-8, (i, err)
    want = orc.bsgs(ct[[0, 7]], diags, baby, giant, bb, gg, sch.mods, p.L, p.K, p.alpha)
    assert_bits_equal(y[[0, 7]], want, "config 4 dense, ciphertexts 0 and 7")


# ------------------------------------------------------------------ config 5
def test_config5_boot_rotation_full_size(orc):
    """2100 primes, alpha = 60, 60 special primes, 4 Galois keys (5^k,
    k in {1, 2, 4, 8}), 8 ciphertexts: the GPU runs all 32 key switches with
    one hoisted ModUp per ciphertext.  The oracle recomputes every one of the
    32 key switches (two ciphertexts at a time, which bounds its memory); the
    integer-pipe conversion then gives the same words for all 32."""
    p = Params(2100, 60, 60)
    ctx = ctx_for(p)
    seed = synth.config_seed(5)
    mods = np.array(ctx.mods, dtype=np.uint64)
    gal = [galois_for_rotation(k) for k in (1, 2, 4, 8)]
    assert gal == [5, 25, 625, 1505]
    ct = synth.uniform_residues((8, 2, 2100, N), mods[:2100], seed, 1, device="cuda")
    keys = [synth.uniform_residues((35, 2, 2160, N), mods, seed, 10 + r, device="cuda")
            for r in range(4)]
    out = ctx.rotate(ct, keys, gal)
    ctx.device_status()
    keys_h = [host(k) for k in keys]
    for pick in ([0, 1], [2, 3], [4, 5], [6, 7]):
        want = orc.rotate(host(ct[pick]), keys_h, np.array(gal, dtype=np.uint64), mods, 2100, 60, 60)
        assert_bits_equal(host(out[:, pick]), want, "config 5, ciphertexts %s, all keys" % pick)
        del want
    del keys_h
    try:
        for engine in ("integer",):
            ctx.set_conversion(engine)
            assert torch.equal(ctx.rotate(ct, keys, gal), out), engine
            ctx.device_status()
    finally:
        ctx.set_conversion("auto")


def test_microbenchmarks_report_counts(orc):
    """The roofline denominators: every kind runs, reports its own operation
    count and leaves the device flag clear; bad kinds are rejected, and the
    split-form kind 6 only runs where every prime is 2^60 - delta."""
    from rns_ckks_polynomial_b200 import Context
    ctx = ctx_for(Params(4, 1, 1))
    for kind, blocks, iters, per in ((0, 16, 64, 256 * 8), (1, 16, 64, 256 * 8), (2, 16, 64, 256 * 8),
                                     (3, 4, 64, 2 * 128 * 256 * 32), (4, 4, 64, 2 * 128 * 32 * 32),
                                     (5, 16, 64, 256 * 4), (6, 16, 8, 256 * 8 * 2 * 8)):
        ms, ops = ctx.bench_intpipe(kind, blocks, iters)
        assert ms > 0
        assert ops == blocks * iters * per
    ctx.device_status()
    with pytest.raises(CkksError) as e:
        ctx.bench_intpipe(7, 1, 1)
    assert e.value.code == -1
    mods = _general_primes(orc, 5)
    gctx = Context(mods[:4], mods[4:], 1)
    with pytest.raises(CkksError) as e:
        gctx.bench_intpipe(6, 1, 1)
    assert e.value.code == -2


def _general_primes(orc, count):
    """Primes q = 1 mod 2n just above 2^59: far from 2^60, so none has the 2^60 - delta form the
    library's cheaper products use."""
    out, c = [], (1 << 59) + 1
    while len(out) < count:
        if orc.is_prime(c):
            out.append(c)
        c += 2 * N
    return out


def test_general_primes_full_stage_parity(orc):
    """The general-prime code paths (full Shoup quotients in the transforms, the generic 128-bit
    reduction in both conversion engines) on every stage, against the oracle."""
    from rns_ckks_polynomial_b200 import Context
    L, K, alpha = 6, 3, 3
    mods_l = _general_primes(orc, L + K)
    assert all((1 << 60) - q >= (1 << 32) for q in mods_l)
    ctx = Context(mods_l[:L], mods_l[L:], alpha)
    mods = np.array(mods_l, dtype=np.uint64)
    x = _res((2, L, N), mods[:L], 300)
    y = ctx.ntt_fwd(dev(x))
    assert_bits_equal(host(y), orc.ntt_fwd(x, mods[:L]), "ntt_fwd")
    assert_bits_equal(host(ctx.ntt_inv(y)), x, "ntt_inv round trip")
    key = _res((2, 2, L + K, N), mods, 301)
    want_d = orc.modup(x, mods, L, K, alpha)
    want_a = orc.key_inner(want_d, key, 5, mods, L, K, alpha)
    want_m = orc.moddown(want_a, mods, L, K)
    want_k = orc.keyswitch(x, key, mods, L, K, alpha)
    try:
        for engine in ("integer", "tensor"):
            ctx.set_conversion(engine)
            dig = ctx.modup(dev(x))
            assert_bits_equal(host(dig), want_d, "modup (%s)" % engine)
            acc = ctx.key_inner(dig, dev(key), 5)
            assert_bits_equal(host(acc), want_a, "key_inner")
            assert_bits_equal(host(ctx.moddown(acc)), want_m, "moddown (%s)" % engine)
            assert_bits_equal(host(ctx.keyswitch(dev(x), dev(key))), want_k, "keyswitch (%s)" % engine)
            ctx.device_status()
    finally:
        ctx.set_conversion("auto")
    ct = _res((2, 2, L, N), mods[:L], 302)
    assert_bits_equal(host(ctx.rescale(dev(ct))), orc.rescale(ct, mods[:L]), "rescale")


def test_bounded_wait_expiry_is_reported_and_recoverable(orc):
    """A device wait that runs out (on a barrier nothing completes) raises the
    context's flag; device_status reports it once, clears it, and the context
    keeps computing correctly."""
    ctx = ctx_for(Params(4, 1, 1))
    ctx.device_status()
    ctx.selftest_wait_expiry()
    with pytest.raises(CkksError) as e:
        ctx.device_status()
    assert e.value.code == -3 and "waiting" in str(e.value)
    ctx.device_status()
    q = np.array(ctx.q, dtype=np.uint64)
    x = _res((2, 4, N), q, 400)
    assert_bits_equal(host(ctx.ntt_fwd(dev(x))), orc.ntt_fwd(x, q), "ntt_fwd after the expiry")


def test_unhoisted_rotation_order(orc):
    """The automorphism-before-ModUp order: bit-exact against the oracle and decrypting to the
    rotated slots (small scheme), and bit-exact with 20-prime digits on the tensor-core path."""
    p = Params(5, 2, 2)
    ctx = ctx_for(p)
    sch = Scheme(orc, p, SEED + 9)
    zs = [synth.uniform_real((SLOTS,), -1, 1, SEED, 90 + i).numpy() for i in range(2)]
    cts = np.stack([sch.encrypt_slots(z) for z in zs])
    rs = [1, 5]
    keys = [sch.keygen_galois(galois_for_rotation(r)) for r in rs]
    gal = [galois_for_rotation(r) for r in rs]
    out = host(ctx.rotate_unhoisted(dev(cts), [dev(k) for k in keys], gal))
    want = orc.rotate_unhoisted(cts, keys, np.array(gal, dtype=np.uint64), sch.mods, p.L, p.K, p.alpha)
    assert_bits_equal(out, want, "rotate_unhoisted")
    for i, r in enumerate(rs):
        for b in range(2):
            assert np.max(np.abs(sch.decrypt_slots(out[i, b]) - rot_left(zs[b], r))) < 1e-8
    p2 = Params(40, 20, 20)
    ctx2 = ctx_for(p2)
    mods = np.array(ctx2.mods, dtype=np.uint64)
    ct = _res((2, 2, 40, N), mods[:40], 91)
    key = _res((2, 2, 60, N), mods, 92)
    got = host(ctx2.rotate_unhoisted(dev(ct), [dev(key)], [25]))
    ctx2.device_status()
    assert_bits_equal(got, orc.rotate_unhoisted(ct, [key], np.array([25], dtype=np.uint64), mods, 40, 20, 20),
                      "rotate_unhoisted, tensor-core conversion")


# ------------------------------------------------------------------ keys of a longer chain
@pytest.mark.parametrize("L,K,alpha,l", [(6, 2, 2, 3), (7, 2, 3, 4), (20, 3, 7, 13), (5, 1, 1, 1)])
def test_key_chain_serves_lower_levels(orc, L, K, alpha, l):
    """A context on q_0..q_{l-1} (with the top chain's special primes) given
    keys made for all L primes (set_key_chain(L)): key switch, rotation and
    relinearised product bit-exact against the oracle run with the keys cut
    down to level l.  (5, 1, 1, 1) is the single-prime chain a refresh starts
    from."""
    from oracle.boot import Chain

    from rns_ckks_polynomial_b200 import Context
    mods = [int(x) for x in orc.gen_primes(N, L + K)]
    m64 = np.array(mods, dtype=np.uint64)
    chain = Chain(m64, L, K, alpha)
    m_l = chain.mods_at(l)
    ctx = Context(mods[:l], mods[L:], alpha)
    try:
        ctx.set_key_chain(L)
        key = _res((Params(L, K, alpha).dnum, 2, L + K, N), m64, 300)
        key_l = chain.key_at(key, l)
        d = _res((2, l, N), m_l[:l], 301)
        assert_bits_equal(host(ctx.keyswitch(dev(d), dev(key))),
                          orc.keyswitch(d, key_l, m_l, l, K, alpha), "keyswitch, level %d" % l)
        ct = _res((2, 2, l, N), m_l[:l], 302)
        assert_bits_equal(host(ctx.rotate(dev(ct), [dev(key)], [5])),
                          orc.rotate(ct, [key_l], np.array([5], dtype=np.uint64), m_l, l, K, alpha),
                          "rotate, level %d" % l)
        if l >= 2:
            a, b = _res((1, 2, l, N), m_l[:l], 303), _res((1, 2, l, N), m_l[:l], 304)
            assert_bits_equal(host(ctx.mul_relin_rescale(dev(a), dev(b), dev(key))),
                              orc.mul_relin_rescale(a, b, key_l, m_l, l, K, alpha),
                              "mul_relin_rescale, level %d" % l)
        with pytest.raises(CkksError):
            ctx.set_key_chain(l - 1)
    finally:
        ctx.close()


# ------------------------------------------------------------------ refresh building blocks
def test_mul_i_scalar_ops_and_c0_constant(orc):
    """X^{n/2} (slots times i) against the oracle's coefficient-domain
    monomial product; products and sums with a per-limb constant; a constant
    added to component 0 only."""
    p = Params(6, 2, 2)
    ctx = ctx_for(p)
    mods = np.array(ctx.mods, dtype=np.uint64)
    LK = p.L + p.K
    x = _res((3, LK, N), mods, 400)
    assert_bits_equal(host(ctx.mul_i(dev(x))), orc.mul_monomial(x, N // 2, mods), "mul_i")
    k = np.ascontiguousarray(_res((LK, 1), mods, 401)[:, 0])
    kb = np.ascontiguousarray(np.broadcast_to(k[:, None], x.shape))
    for op in ("mul", "add", "sub"):
        assert_bits_equal(host(ctx.pointwise_scalar(op, dev(x), dev(k))),
                          orc.pointwise(op, x, kb, mods), "pointwise_scalar %s" % op)
    ct = _res((2, 2, p.L, N), mods[:p.L], 402)
    want = ct.copy()
    want[:, 0] = orc.pointwise("add", ct[:, 0], np.ascontiguousarray(
        np.broadcast_to(k[:p.L, None], ct[:, 0].shape)), mods[:p.L])
    assert_bits_equal(host(ctx.add_const_c0(dev(ct), dev(np.ascontiguousarray(k[:p.L])))), want,
                      "add_const_c0")


def test_conj_extract_and_restore_merge(orc):
    """Bit-exact against the oracle, and the slots decrypt to 2 Re w, 2 Im w,
    then to 2 w after the merge."""
    p = Params(6, 2, 2)
    ctx = ctx_for(p)
    sch = Scheme(orc, p, SEED + 40)
    w = synth.uniform_real((SLOTS,), -1, 1, SEED, 410).numpy() + \
        1j * synth.uniform_real((SLOTS,), -1, 1, SEED, 411).numpy()
    ct = sch.encrypt_slots(w)[None]
    ck = sch.keygen_galois(2 * N - 1)
    re, im = ctx.conj_extract(dev(ct), dev(ck))
    want_re, want_im = orc.conj_extract(ct, ck, sch.mods, p.L, p.K, p.alpha)
    assert_bits_equal(host(re), want_re, "conj_extract re")
    assert_bits_equal(host(im), want_im, "conj_extract im")
    merged = ctx.restore_merge(re, im)
    assert_bits_equal(host(merged), orc.restore_merge(want_re, want_im, sch.q), "restore_merge")
    assert np.max(np.abs(sch.decrypt_slots(host(re)[0], 2 * SCALE) - w.real)) < 1e-8
    assert np.max(np.abs(sch.decrypt_slots(host(merged)[0], 2 * SCALE) - w)) < 1e-8


@pytest.mark.parametrize("L,K,alpha,l", [(6, 2, 2, 1), (6, 2, 2, 3), (6, 2, 2, 6), (40, 4, 4, 19),
                                         (80, 4, 4, 63)])
def test_modraise(orc, L, K, alpha, l):
    """The centred lift onto the whole chain, bit-exact against the oracle;
    coefficients 0, 1, (Q-1)/2, (Q+1)/2 and Q-1 sit at the start of the
    first polynomial, where the sign decision is tightest."""
    ctx = context(L, K, alpha)
    mods = np.array(ctx.mods, dtype=np.uint64)
    q = [int(v) for v in mods[:l]]
    Q = 1
    for v in q:
        Q *= v
    coef = _res((2, 2, l, N), mods[:l], 420)
    for j, X in enumerate([0, 1, (Q - 1) // 2, (Q + 1) // 2, Q - 1]):
        for i in range(l):
            coef[0, 0, i, j] = X % q[i]
    x = orc.ntt_fwd(coef, mods[:l])
    got = host(ctx.modraise(dev(x)))
    assert_bits_equal(got, orc.modraise(x, mods[:L]), "modraise l=%d" % l)


@pytest.mark.parametrize("plan", [(64, -8, 4, 4), (8, -7, 4, 4), (1, -7, 4, 4), (1, 0, 4, 3),
                                  (3, 5, 2, 1)])
def test_bsgs_plan_matches_oracle(orc, plan):
    """Strided-window BSGS (the groups of a three-level factored transform at
    n = 2048, the dense window, and a single rotated giant step) bit-exact
    against the oracle on seeded residues, with the oracle's Galois keys."""
    from oracle.boot import Chain, bsgs_plan_apply
    stride, t0, bb, gg = plan
    S = SLOTS
    p = Params(6, 2, 2)
    ctx = ctx_for(p)
    sch = Scheme(orc, p, SEED + 50)
    chain = Chain(sch.mods, p.L, p.K, p.alpha)
    amounts = {(stride * b) % S for b in range(1, bb)} | {(stride * (t0 + bb * g)) % S for g in range(gg)}
    keys = {a: sch.keygen_galois(galois_for_rotation(a)) for a in amounts if a}
    x = _res((2, 2, p.L, N), sch.q, 430)
    pts = _res((gg, bb, p.L, N), sch.q, 431)
    giants = [(stride * (t0 + bb * g)) % S for g in range(gg)]
    y = host(ctx.bsgs_lintrans_plan(dev(x), dev(pts), [dev(keys[(stride * b) % S]) for b in range(1, bb)],
                                    [dev(keys[G]) if G else None for G in giants], plan))
    for i in range(2):
        want, _ = bsgs_plan_apply(x[i], SCALE, [[pts[g, b] for b in range(bb)] for g in range(gg)],
                                  plan, SCALE, keys, chain)
        assert_bits_equal(y[i], want, "bsgs plan %s, ct %d" % (plan, i))


def test_refresh_matches_oracle(orc):
    """The whole refresh at n = 2048 (16 primes, the plans of two-level
    factored transforms, r = 4: 2 * 2 + 6 + 4 levels) through the per-level
    contexts and one top-level key set, bit-exact against the oracle's
    refresh with the same seeded plaintext residues, and the same tracked
    scale.  (Decryption of the refresh is pinned on the CPU.)"""
    from oracle import boot

    from rns_ckks_polynomial_b200.refresh import Refresh
    L, K, alpha, depth, r = 16, 4, 4, 2, 4
    p = Params(L, K, alpha)
    sch = Scheme(orc, p, SEED + 60)
    chain = boot.Chain(sch.mods, L, K, alpha)
    keys = {"rot": {a: sch.keygen_galois(galois_for_rotation(a))
                    for a in boot.factored_rotation_amounts(N, depth)},
            "conj": sch.keygen_galois(2 * N - 1), "relin": sch.keygen_relin()}
    low = np.ascontiguousarray(_res((2, 1, N), sch.q[:1], 440))

    def levels(factors, top, stream):
        out = []
        for i, F in enumerate(factors):
            plan = orc.bsgs_plan(F, SLOTS)
            _, _, bb, gg = plan
            out.append((plan, _res((gg, bb, top - i, N), sch.q[:top - i], stream + i)))
        return out

    cts = levels(orc.factored_coeff_to_slot(N, depth), L, 450)
    stc = levels(orc.factored_slot_to_coeff(N, depth), L - depth - 6 - r, 460)
    want, s_want = boot.refresh_with_levels(low, r, [(pl, list(a)) for pl, a in cts],
                                            [(pl, list(a)) for pl, a in stc], keys, chain)
    dkeys = {"rot": {a: dev(k) for a, k in keys["rot"].items()}, "conj": dev(keys["conj"]),
             "relin": dev(keys["relin"])}
    rf = Refresh(sch.q, sch.mods[L:], alpha, dkeys)
    try:
        got, s_got = rf.refresh(dev(low[None]), r, [(pl, dev(a)) for pl, a in cts],
                                [(pl, dev(a)) for pl, a in stc])
        assert s_got == s_want
        assert_bits_equal(host(got)[0], want, "refresh")
    finally:
        rf.close()


def _extremes(q):
    """All zeros, all q - 1, and q - 1 alternating with 0, over limbs with primes q: [3][len(q)][n]."""
    q = np.asarray(q, dtype=np.uint64)
    top = np.broadcast_to((q - 1)[:, None], (q.size, N))
    alt = np.where(np.arange(N) % 2 == 0, top, 0).astype(np.uint64)
    return np.stack([np.zeros((q.size, N), np.uint64), np.ascontiguousarray(top, dtype=np.uint64), alt])


def test_extreme_residues_ntt_2100(orc):
    """Inputs at the ends of [0, q) through the forward and inverse NTT on all
    2100 limbs of the boot chain (the lazy butterflies see their largest
    operands)."""
    ctx = context(2100, 60, 60)
    q = np.array(ctx.q, dtype=np.uint64)
    x = _extremes(q)
    y = dev(x)
    ctx.ntt_fwd(y)
    assert_bits_equal(host(y), orc.ntt_fwd(x, q), "ntt_fwd extremes, 2100 limbs")
    ctx.ntt_inv(y)
    assert_bits_equal(host(y), x, "ntt round trip extremes, 2100 limbs")
    z = dev(x)
    ctx.ntt_inv(z)
    assert_bits_equal(host(z), orc.ntt_inv(x, q), "ntt_inv extremes, 2100 limbs")


@pytest.mark.parametrize("L,K,alpha", [(6, 2, 2), (24, 8, 8), (120, 60, 60)])
def test_extreme_residues_key_switch_stages(orc, L, K, alpha):
    """Extreme inputs (all zeros, all q - 1, alternating) and an all-(q - 1)
    key through ModUp, the key inner product (g = 1 and 5) and ModDown on
    both conversion engines, where the exact 128-bit sums and the tensor
    cores' byte planes reach their largest values; ModDown also on an
    all-(q - 1) accumulator.  Each stage bit-exact against the oracle."""
    p = Params(L, K, alpha)
    ctx = ctx_for(p)
    mods = np.array(ctx.mods, dtype=np.uint64)
    c = _extremes(mods[:L])
    key = np.ascontiguousarray(np.broadcast_to((mods - 1)[None, None, :, None], (p.dnum, 2, L + K, N)),
                               dtype=np.uint64)
    acc_top = np.ascontiguousarray(np.broadcast_to((mods - 1)[None, None, :, None], (1, 2, L + K, N)),
                                   dtype=np.uint64)
    want_d = orc.modup(c, mods, L, K, alpha)
    want_a = {g: orc.key_inner(want_d, key, g, mods, L, K, alpha) for g in (1, 5)}
    want_m = orc.moddown(want_a[5], mods, L, K)
    want_top = orc.moddown(acc_top, mods, L, K)
    try:
        for engine in ("integer", "tensor"):
            ctx.set_conversion(engine)
            dig = ctx.modup(dev(c))
            assert_bits_equal(host(dig), want_d, "modup extremes (%s)" % engine)
            for g in (1, 5):
                acc = ctx.key_inner(dig, dev(key), g)
                assert_bits_equal(host(acc), want_a[g], "key_inner extremes g=%d (%s)" % (g, engine))
            assert_bits_equal(host(ctx.moddown(acc)), want_m, "moddown extremes (%s)" % engine)
            assert_bits_equal(host(ctx.moddown(dev(acc_top))), want_top, "moddown all q-1 (%s)" % engine)
            ctx.device_status()
    finally:
        ctx.set_conversion("auto")


@pytest.mark.parametrize("lp1", [2, 112])
def test_extreme_residues_rescale(orc, lp1):
    ctx = context(112, 8, 8)
    q = np.array(ctx.mods[:lp1], dtype=np.uint64)
    x = _extremes(q)
    ct = np.ascontiguousarray(np.stack([x, x[::-1]], axis=1))  # [3][2][lp1][n]
    assert_bits_equal(host(ctx.rescale(dev(ct))), orc.rescale(ct, q), "rescale extremes, %d limbs" % lp1)


def _top_general_primes(orc, count):
    """Primes q = 1 mod 2n just below 2^60 - 2^32: close enough to 2^60 that 260 (q - 1)^2 passes
    2^128, yet not of the 2^60 - delta (delta < 2^32) form."""
    out, c = [], ((1 << 60) - (1 << 32)) // (2 * N) * (2 * N) + 1
    while len(out) < count:
        if orc.is_prime(c):
            out.append(c)
        c -= 2 * N
    return out


@pytest.mark.parametrize("form", ["special", "general"])
def test_key_inner_more_than_256_digits(orc, form):
    """260 single-prime digits (L = 260, alpha = 1): with every digit word and
    key word at q - 1 the exact sum 260 (q - 1)^2 passes 2^128.  Primes of the
    2^60 - delta form take the split sums (three 64-bit partial sums, folded
    every 8 digits: this input drives each of them to its largest value);
    other primes take 128-bit sums, which must be reduced between blocks of
    256 digits.  Each output word is the closed form 260 (q - 1)^2 = 260 mod q."""
    from rns_ckks_polynomial_b200 import Context
    L, K = 260, 1
    if form == "special":
        ctx = context(L, K, 1)
    else:
        mods_l = _top_general_primes(orc, L + K)
        assert all((1 << 60) - q >= (1 << 32) and 260 * (q - 1) ** 2 >= 1 << 128 for q in mods_l)
        ctx = Context(mods_l[:L], mods_l[L:], 1)
    mods = torch.tensor(np.array(ctx.mods, dtype=np.uint64).view(np.int64), device="cuda")
    LK = L + K
    top = (mods - 1).view(1, 1, LK, 1)
    digits = top.expand(1, L, LK, N).contiguous()
    key = top.expand(L, 2, LK, N).contiguous()
    acc = host(ctx.key_inner(digits, key, 1))
    ctx.device_status()
    want = np.broadcast_to((260 % np.array(ctx.mods, dtype=np.uint64))[None, None, :, None], (1, 2, LK, N))
    assert_bits_equal(acc, want, "key inner product over 260 digits")


def test_key_inner_wide_chunks(orc):
    """From 8 ciphertexts per key the split-form inner product gives each thread 8 ciphertexts
    (4 digits of prefetch); below that, 4.  Ragged chunks (10 = 8 + 2 and 9 = 8 + 1 ciphertexts)
    through the direct call, the hoisted rotation and the per-key digits of the unhoisted order,
    bit-exact against the oracle; all-(q - 1) words over 40 one-prime digits against the closed
    form 40 (q - 1)^2 = 40 mod q, which drives every split sum to its largest value."""
    L, K, alpha = 20, 3, 7
    p = Params(L, K, alpha)
    ctx = ctx_for(p)
    mods = np.array(ctx.mods, dtype=np.uint64)
    B = 10
    dig = _res((B, p.dnum, L + K, N), mods, 700)
    key = _res((p.dnum, 2, L + K, N), mods, 701)
    for g in (1, 5, 4095):
        got = host(ctx.key_inner(dev(dig), dev(key), g))
        assert_bits_equal(got, orc.key_inner(dig, key, g, mods, L, K, alpha), "key_inner, 10 ct, g=%d" % g)
    ctx.device_status()
    ct = _res((B, 2, L, N), mods[:L], 702)
    keys = [_res((p.dnum, 2, L + K, N), mods, 703 + r) for r in range(2)]
    gal = np.array([5, 4095], dtype=np.uint64)
    want = orc.rotate(ct, keys, gal, mods, L, K, alpha)
    assert_bits_equal(host(ctx.rotate(dev(ct), [dev(k) for k in keys], list(gal))), want, "rotate, 10 ct")
    want_u = orc.rotate_unhoisted(ct, keys, gal, mods, L, K, alpha)
    assert_bits_equal(host(ctx.rotate_unhoisted(dev(ct), [dev(k) for k in keys], list(gal))), want_u,
                      "rotate_unhoisted, 10 ct")
    ctx.device_status()
    ctx1 = context(40, 1, 1)
    m1 = torch.tensor(np.array(ctx1.mods, dtype=np.uint64).view(np.int64), device="cuda")
    top = (m1 - 1).view(1, 1, 41, 1)
    acc = host(ctx1.key_inner(top.expand(9, 40, 41, N).contiguous(), top.expand(40, 2, 41, N).contiguous(), 5))
    ctx1.device_status()
    want_top = np.broadcast_to((40 % np.array(ctx1.mods, dtype=np.uint64))[None, None, :, None], (9, 2, 41, N))
    assert_bits_equal(acc, want_top, "key inner product of all-(q - 1) words, 9 ct")


def test_refresh_n2048_decodes_to_the_sine_form(orc):
    """The refresh as the oracle's n = 2048 pin runs it (23 + 4 primes, a
    dense ternary secret, three-level factored transforms with their encoded
    plaintexts, r = 9: 21 levels) through the per-level contexts on the GPU:
    bit-exact against the oracle's refresh over the same plaintexts, and the
    decrypted coefficients within 1e-5 of the sine form
    (q_0 / 2 pi) sin(2 pi m_k / q_0) / Delta of the input's coefficients m."""
    import math
    from fractions import Fraction

    from oracle import boot

    from rns_ckks_polynomial_b200.refresh import Refresh
    n, depth, r, L, K, alpha = N, 3, 9, 23, 4, 4
    delta = 2**50
    p = Params(L, K, alpha)
    sch = Scheme(orc, p, SEED + 80)
    chain = boot.Chain(sch.mods, L, K, alpha)
    keys = {"rot": {a: sch.keygen_galois(galois_for_rotation(a, n))
                    for a in boot.factored_rotation_amounts(n, depth)},
            "conj": sch.keygen_galois(2 * n - 1), "relin": sch.keygen_relin()}
    z = synth.uniform_real((SLOTS,), -1, 1, SEED, 810).numpy() + \
        1j * synth.uniform_real((SLOTS,), -1, 1, SEED, 811).numpy()
    low = np.ascontiguousarray(sch.encrypt_slots(z, delta)[:, :1])
    q0 = int(sch.mods[0])

    def levels(factors, scalar, top, pt_scale):
        out = []
        for i, F in enumerate(factors):
            if i == 0:
                F = {k: scalar * d for k, d in F.items()}
            plan = orc.bsgs_plan(F, SLOTS)
            pts, _ = orc.plan_plaintexts(F, plan, SLOTS, sch.mods[:top - i], pt_scale, n)
            out.append((plan, np.stack([np.stack([np.zeros((top - i, n), np.uint64) if v is None else v
                                                  for v in row]) for row in pts])))
        return out

    cts = levels(orc.factored_coeff_to_slot(n, depth), 0.5, L, 2**60)
    stc = levels(orc.factored_slot_to_coeff(n, depth), q0 / (2 * math.pi * delta), L - depth - 6 - r, 2**50)
    want, s_want = boot.refresh_with_levels(low, r, [(pl, list(a)) for pl, a in cts],
                                            [(pl, list(a)) for pl, a in stc], keys, chain)
    dkeys = {"rot": {a: dev(k) for a, k in keys["rot"].items()}, "conj": dev(keys["conj"]),
             "relin": dev(keys["relin"])}
    rf = Refresh(sch.q, sch.mods[L:], alpha, dkeys)
    try:
        got, s_got = rf.refresh(dev(low[None]), r, [(pl, dev(a)) for pl, a in cts],
                                [(pl, dev(a)) for pl, a in stc])
        torch.cuda.synchronize()
    finally:
        rf.close()
    assert s_got == s_want
    out = host(got)[0]
    assert out.shape == (2, L - 2 * depth - 6 - r, n)
    assert_bits_equal(out, want, "refresh at n = 2048")
    res = orc.decrypt(low, sch.s, sch.mods[:1])
    m = orc.crt_centered(res, sch.mods[:1])
    res_o = orc.decrypt(out, sch.s, sch.mods[:out.shape[-2]])
    got_c = np.array([float(Fraction(c) / s_got) for c in orc.crt_centered(res_o, sch.mods[:out.shape[-2]])])
    sine = np.array([q0 / (2 * math.pi) * math.sin(2 * math.pi * v / q0) / delta for v in m])
    assert np.max(np.abs(got_c - sine)) < 1e-5


def test_coeff_to_slot_level_at_2100_primes(orc):
    """One level of the three-level factored coeff_to_slot at the boot chain's
    full size (2100 + 60 primes, alpha = 60): the plan (stride 64, t0 = -8,
    bb = gg = 4) with its 6 Galois keys over 8 ciphertexts of seeded uniform
    residues and seeded plaintext diagonals, as the refresh bench runs it.
    The oracle recomputes ciphertext 5 (3 hoisted baby rotations, 3 rotated
    giant steps and the unrotated one, rescale)."""
    import psutil

    from oracle.boot import Chain, bsgs_plan_apply
    if psutil.virtual_memory().available < 64 << 30:
        pytest.skip("needs 64 GB of free host memory for the oracle's keys")
    p = Params(2100, 60, 60)
    ctx = ctx_for(p)
    seed = synth.config_seed(5) + 90
    mods = np.array(ctx.mods, dtype=np.uint64)
    stride, t0, bb, gg = plan = (64, -8, 4, 4)
    S = SLOTS
    amounts = sorted({(stride * b) % S for b in range(1, bb)} |
                     {(stride * (t0 + bb * g)) % S for g in range(gg)} - {0})
    assert amounts == [64, 128, 192, 256, 512, 768]
    keys = {a: synth.uniform_residues((35, 2, 2160, N), mods, seed, 10 + a, device="cuda") for a in amounts}
    x = synth.uniform_residues((8, 2, 2100, N), mods[:2100], seed, 1, device="cuda")
    pts = synth.uniform_residues((gg, bb, 2100, N), mods[:2100], seed, 2, device="cuda")
    giants = [(stride * (t0 + bb * g)) % S for g in range(gg)]
    y = ctx.bsgs_lintrans_plan(x, pts, [keys[(stride * b) % S] for b in range(1, bb)],
                               [keys[G] if G else None for G in giants], plan)
    ctx.device_status()
    chain = Chain(mods, 2100, 60, 60)
    hp = host(pts)
    want, _ = bsgs_plan_apply(host(x[5]), SCALE, [[hp[g, b] for b in range(bb)] for g in range(gg)], plan,
                              SCALE, {a: host(k) for a, k in keys.items()}, chain)
    assert_bits_equal(host(y[5]), want, "coeff_to_slot level (64, -8, 4, 4) at 2100 primes, ciphertext 5")
