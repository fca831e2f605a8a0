"""The streamed rotation (ModUp -> NTT -> key inner product over windows of at most 60 primes, no
[B][dnum][L+K][n] digit tensor) against the oracle's hoisted rotation and, word for word, against
the library's own hoisted rotation (which keeps the whole digit tensor)."""
import numpy as np
import pytest
import torch

from rns_ckks_polynomial_b200 import synth
from rns_ckks_polynomial_b200.api import OP_ROTATE, OP_ROTATE_STREAMED
from rns_ckks_polynomial_b200.native import CkksError

from .gpu_common import assert_bits_equal, context, ctx_for, dev, gpu, host, need_gpu
from .helpers import N, Params, galois_for_rotation, u64

pytestmark = gpu

SEED = synth.config_seed(7)


@pytest.fixture(autouse=True)
def _gpu():
    need_gpu()
    yield
    torch.cuda.synchronize()
    torch.cuda.empty_cache()


def _res(shape, mods, stream):
    return u64(synth.uniform_residues(shape, mods, SEED, stream))


# (4, 1, 1): one-prime digits and windows; (20, 3, 7): a ragged last digit (7 + 7 + 6);
# (112, 8, 8): the layer chain; (70, 33, 33): 33-prime windows (two blocks of targets), a 4-prime
# last digit; (130, 64, 64): 64-source conversions, two 32-prime windows per digit; (120, 30, 30):
# one 30-prime window per digit and one for the special primes.
@pytest.mark.parametrize("L,K,alpha", [(4, 1, 1), (20, 3, 7), (112, 8, 8), (70, 33, 33), (130, 64, 64),
                                       (120, 30, 30)])
def test_streamed_rotation_matches_oracle(orc, L, K, alpha):
    p = Params(L, K, alpha)
    ctx = ctx_for(p)
    mods = np.array(ctx.mods, dtype=np.uint64)
    B = 3
    ct = _res((B, 2, L, N), mods[:L], 100 + L)
    keys = [_res((p.dnum, 2, L + K, N), mods, 200 + L + r) for r in range(2)]
    gal = [5, 4095]
    out = ctx.rotate_streamed(dev(ct), [dev(k) for k in keys], gal)
    ctx.device_status()
    want = orc.rotate(ct, keys, np.array(gal, dtype=np.uint64), mods, L, K, alpha)
    assert_bits_equal(host(out), want, "streamed rotation (%d, %d, %d)" % (L, K, alpha))
    hoisted = ctx.rotate(dev(ct), [dev(k) for k in keys], gal)
    assert torch.equal(out, hoisted)


def test_streamed_rotation_boot_size_equals_hoisted():
    """2100 + 60 primes, alpha = 60, 8 ciphertexts x 4 Galois keys (config 5): every word equals
    the hoisted rotation's, which its own test checks against the oracle; the streamed call's
    workspace lacks the 9.9 GB digit tensor and holds two 275 MB windows of it instead."""
    ctx = context(2100, 60, 60)
    mods = np.array(ctx.mods, dtype=np.uint64)
    gal = [galois_for_rotation(k) for k in (1, 2, 4, 8)]
    ct = synth.uniform_residues((8, 2, 2100, N), mods[:2100], SEED, 1, device="cuda")
    keys = [synth.uniform_residues((35, 2, 2160, N), mods, SEED, 10 + r, device="cuda") for r in range(4)]
    out = ctx.rotate_streamed(ct, keys, gal)
    ctx.device_status()
    want = ctx.rotate(ct, keys, gal)
    ctx.device_status()
    assert torch.equal(out, want)
    # the hoisted call holds the digit tensor (and ModUp's sources inside ModDown's larger scratch);
    # the streamed one holds ModUp's sources and two windows of digits (one per stream) instead
    limb = N * 8
    digits, sources, window = 8 * 35 * 2160 * limb, 8 * 2100 * limb, 8 * 35 * 60 * limb
    ws_h = ctx.workspace_bytes(OP_ROTATE, 8, 4)
    ws_s = ctx.workspace_bytes(OP_ROTATE_STREAMED, 8, 4)
    assert ws_h - ws_s == digits - sources - 2 * window, (ws_h, ws_s)


def test_streamed_rotation_extreme_residues(orc):
    """Every input word at q - 1 (the largest residue) through every window, against the oracle."""
    L, K, alpha = 20, 3, 7
    ctx = context(L, K, alpha)
    mods = np.array(ctx.mods, dtype=np.uint64)
    dnum = (L + alpha - 1) // alpha
    ct = np.broadcast_to((mods[:L] - 1)[None, None, :, None], (2, 2, L, N)).copy()
    key = np.broadcast_to((mods - 1)[None, None, :, None], (dnum, 2, L + K, N)).copy()
    out = ctx.rotate_streamed(dev(ct), [dev(key)], [25])
    ctx.device_status()
    want = orc.rotate(ct, [key], np.array([25], dtype=np.uint64), mods, L, K, alpha)
    assert_bits_equal(host(out), want, "streamed rotation of all-(q - 1) words")


def test_streamed_rotation_errors():
    """An even Galois element is CKKS_EINVAL, before any launch."""
    ctx = context(4, 1, 1)
    ct = torch.zeros((1, 2, 4, N), dtype=torch.int64, device="cuda")
    key = torch.zeros((4, 2, 5, N), dtype=torch.int64, device="cuda")
    with pytest.raises(CkksError) as e:
        ctx.rotate_streamed(ct, [key], [4])
    assert e.value.code == -1


def test_streamed_rotation_in_a_cuda_graph():
    """Captured into a CUDA graph the call keeps every window on the capturing stream (one lane,
    one window buffer); replays give the hoisted rotation's words."""
    L, K, alpha = 20, 3, 7
    ctx = context(L, K, alpha)
    mods = np.array(ctx.mods, dtype=np.uint64)
    dnum = (L + alpha - 1) // alpha
    ct = dev(_res((2, 2, L, N), mods[:L], 300))
    keys = [dev(_res((dnum, 2, L + K, N), mods, 301 + r)) for r in range(3)]
    gal = [5, 25, 4095]
    want = ctx.rotate(ct, keys, gal)
    out = torch.empty_like(want)
    ws = torch.empty(ctx.workspace_bytes(OP_ROTATE_STREAMED, 2, 3), dtype=torch.uint8, device="cuda")
    ctx.rotate_streamed(ct, keys, gal, out=out, ws=ws)  # tables built outside the capture
    torch.cuda.synchronize()
    out.zero_()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=side):
            ctx.rotate_streamed(ct, keys, gal, out=out, ws=ws)
    torch.cuda.current_stream().wait_stream(side)
    for _ in range(2):
        out.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(out, want)
    ctx.device_status()
    del g


def test_streamed_rotation_more_than_64_keys(orc):
    """66 keys: the call works through them in chunks of 64, each repeating the windows' work;
    every output equals the hoisted rotation's, and two of them the oracle's."""
    L, K, alpha = 4, 1, 1
    ctx = context(L, K, alpha)
    mods = np.array(ctx.mods, dtype=np.uint64)
    ct_h = _res((1, 2, L, N), mods[:L], 400)
    keys_h = [_res((L, 2, L + K, N), mods, 401 + r) for r in range(66)]
    gal = [galois_for_rotation(r + 1) for r in range(66)]
    ct = dev(ct_h)
    keys = [dev(k) for k in keys_h]
    out = ctx.rotate_streamed(ct, keys, gal)
    ctx.device_status()
    assert torch.equal(out, ctx.rotate(ct, keys, gal))
    pick = [0, 65]
    want = orc.rotate(ct_h, [keys_h[r] for r in pick], np.array([gal[r] for r in pick], dtype=np.uint64),
                      mods, L, K, alpha)
    assert_bits_equal(host(out[pick]), want, "keys 0 and 65")
