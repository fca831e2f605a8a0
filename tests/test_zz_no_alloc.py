"""The allocation-free ModUp entry point (ckks_modup_noalloc).

Some callers cannot call cudaMalloc. Examples are a host framework whose
caching allocator already owns the device memory under a fixed budget, and a
latency-critical loop that cannot absorb the device-wide synchronisation an
allocation can imply. For them the library offers ModUp with its scratch in a
static device array. This test calls it through the C ABI twice in a row and
checks both results word for word against ckks_modup, whose own parity with the
CPU oracle is covered by the other GPU tests. It lives in a file of its own that
pytest collects last, and it passes alone in a fresh process as well as after
the other tests.
"""
import ctypes as C

import pytest
import torch

from rns_ckks_polynomial_b200 import native, synth

from .gpu_common import context, need_gpu

pytestmark = pytest.mark.gpu

N = 2048


@pytest.mark.parametrize("L,K,alpha,batch", [(112, 8, 8, 8), (5, 2, 2, 3)])
def test_modup_noalloc_matches_modup_twice(L, K, alpha, batch):
    need_gpu()
    ctx = context(L, K, alpha)
    lib = native.lib()
    mods = ctx.mods
    stream = C.c_void_p(torch.cuda.current_stream().cuda_stream)
    ref = torch.empty((batch, ctx.dnum, L + K, N), dtype=torch.int64, device="cuda")
    out = torch.empty_like(ref)
    for call in range(2):
        c = synth.uniform_residues((batch, L, N), mods[:L], synth.config_seed(9), 300 + call,
                                   device="cuda")
        ws = torch.empty(ctx.workspace_bytes(1, batch), dtype=torch.uint8, device="cuda")
        rc = lib.ckks_modup(ctx._h, C.c_void_p(c.data_ptr()), C.c_void_p(ref.data_ptr()), batch,
                            C.c_void_p(ws.data_ptr()), stream)
        assert rc == 0, lib.ckks_last_error()
        out.fill_(-1)
        rc = lib.ckks_modup_noalloc(ctx._h, C.c_void_p(c.data_ptr()), C.c_void_p(out.data_ptr()),
                                    batch, stream)
        assert rc == 0, lib.ckks_last_error()
        torch.cuda.synchronize()
        assert torch.equal(out, ref), "call %d differs from ckks_modup" % call
    ctx.device_status()
    # with the address resolved, calls of the entry point alone leave the
    # device's free memory as it was
    del ws
    torch.cuda.synchronize()
    free_before, _ = torch.cuda.mem_get_info()
    for _ in range(2):
        rc = lib.ckks_modup_noalloc(ctx._h, C.c_void_p(c.data_ptr()), C.c_void_p(out.data_ptr()),
                                    batch, stream)
        assert rc == 0, lib.ckks_last_error()
    torch.cuda.synchronize()
    free_after, _ = torch.cuda.mem_get_info()
    assert free_after == free_before
    assert torch.equal(out, ref)
    ctx.device_status()


def test_modup_noalloc_rejects_oversized_batch():
    need_gpu()
    ctx = context(112, 8, 8)
    lib = native.lib()
    rc = lib.ckks_modup_noalloc(ctx._h, None, None, 19, None)  # 19 * 112 > 2048 limbs
    assert rc == -2
    assert b"2048-limb" in lib.ckks_last_error()


def test_modup_noalloc_refuses_before_the_folded_tables_exist():
    """On a fresh context whose digits of 8 primes convert on the folded tensor-core engine, the
    tables do not exist until a converting call builds them (with cudaMalloc). Until then the entry
    point returns CKKS_EUNSUPPORTED, launches nothing and leaves the device's free memory as it
    was; after one ckks_modup it gives ckks_modup's words."""
    need_gpu()
    import oracle
    from rns_ckks_polynomial_b200 import Context
    L, K, alpha, batch = 24, 8, 8, 2
    mods = [int(x) for x in oracle.gen_primes(N, L + K)]
    ctx = Context(mods[:L], mods[L:], alpha)  # not the shared cached context: no call has run on it
    lib = native.lib()
    stream = C.c_void_p(torch.cuda.current_stream().cuda_stream)
    c = synth.uniform_residues((batch, L, N), mods[:L], synth.config_seed(9), 400, device="cuda")
    out = torch.full((batch, ctx.dnum, L + K, N), -1, dtype=torch.int64, device="cuda")
    torch.cuda.synchronize()
    free_before, _ = torch.cuda.mem_get_info()
    rc = lib.ckks_modup_noalloc(ctx._h, C.c_void_p(c.data_ptr()), C.c_void_p(out.data_ptr()), batch, stream)
    torch.cuda.synchronize()
    free_after, _ = torch.cuda.mem_get_info()
    assert rc == -2
    assert b"folded conversion tables" in lib.ckks_last_error()
    assert free_after == free_before
    assert bool((out == -1).all()), "a refused call wrote its output"
    ref = ctx.modup(c)
    rc = lib.ckks_modup_noalloc(ctx._h, C.c_void_p(c.data_ptr()), C.c_void_p(out.data_ptr()), batch, stream)
    assert rc == 0, lib.ckks_last_error()
    torch.cuda.synchronize()
    assert torch.equal(out, ref)
    ctx.device_status()
