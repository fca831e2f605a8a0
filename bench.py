#!/usr/bin/env python
"""Benchmark of the RNS-CKKS hot path on B200.

Workload (one step): the NTT/INTT throughput sweep at n = 2048 -- a batch of
16 polynomials with seeded uniform residues at each of 3, 112, 512 and 2100
limbs of 60-bit NTT-friendly primes, forward NTT then inverse NTT, in place,
each direction one grouped launch over the four tensors (ckks_ntt_fwd_group /
ckks_ntt_inv_group); the round trip is checked to be the identity after the
timed steps.  The metric is limb-NTTs per second (forward and inverse both
count).

Next to it, the key-switch rates of the three key-switching workloads are
measured once in the same run (not part of the step): the layer-shaped
ct x ct multiply (112 primes, alpha 8, 8 pairs), the BSGS matrix-vector
product (112 primes, bb = gg = 32, 8 ciphertexts) and the boot-level hoisted
rotation (2100 primes, alpha 60, 4 Galois keys, 8 ciphertexts).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
                    [--no-ks]

Under torchrun each rank runs its own batch (weak scaling, no data-path
collective); the step time is the max over ranks.
"""
import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

N = 2048
SWEEP = (3, 112, 512, 2100)
BATCH = 16
METRIC = "limb-NTTs/s at n=2048 (NTT+INTT sweep, limbs 3/112/512/2100, batch 16)"
WORKLOAD = "ntt_sweep_n2048_b16_limbs3-112-512-2100"
L2_FLUSH_BYTES = 256 << 20


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=60)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="b200", choices=["b200", "reference"])
    ap.add_argument("--no-ks", action="store_true", help="skip the key-switch measurements")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU oracle baseline")
    ap.add_argument("--refresh-only", action="store_true",
                    help="time only the bootstrapping refresh at 2100 + 60 primes")
    ap.add_argument("--ks-only", action="store_true",
                    help="run only the key-switch measurements (for profiling)")
    ap.add_argument("--ks-batch", type=int, default=8,
                    help="ciphertexts per key-switch workload (8 = the configs; smaller only for profiling)")
    ap.add_argument("--ks-keys", type=int, default=4,
                    help="Galois keys of the boot-level rotation (4 = the config; smaller only for profiling)")
    ap.add_argument("--ks-entries", default=",".join(KS_ENTRIES),
                    help="key-switching workloads to build and time (with --ks-only: only these)")
    ap.add_argument("--sweep", default=",".join(str(x) for x in SWEEP),
                    help="limb counts of the step (a smaller case for profiling only)")
    return ap.parse_args()


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


# ---------------------------------------------------------------- clocks
class ClockSampler:
    """Samples the SM clock and the clock-event reasons through NVML every
    `period` seconds while active (the same counters nvidia-smi reports)."""

    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
               0x4: "sw_power_cap", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, torch_device, period=0.002):
        self.dev = torch_device
        self.period = period
        self.samples = []
        self.max_mhz = None
        self.handle = None
        self._stop = threading.Event()

    def _open(self):
        import pynvml
        import torch
        pynvml.nvmlInit()
        p = torch.cuda.get_device_properties(self.dev)
        bus = "%08x:%02x:%02x.0" % (p.pci_domain_id, p.pci_bus_id, p.pci_device_id)
        self.handle = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
        self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.handle, pynvml.NVML_CLOCK_SM)
        return pynvml

    def __enter__(self):
        try:
            nv = self._open()
        except Exception as e:  # noqa: BLE001 - clocks are reported as unsampled
            self.error = repr(e)
            return self

        def run():
            get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                nv.nvmlDeviceGetCurrentClocksThrottleReasons
            while not self._stop.is_set():
                try:
                    mhz = nv.nvmlDeviceGetClockInfo(self.handle, nv.NVML_CLOCK_SM)
                    self.samples.append((mhz, int(get_reasons(self.handle))))
                except Exception:  # noqa: BLE001
                    pass
                time.sleep(self.period)

        self.thread = threading.Thread(target=run, daemon=True)
        self.thread.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if getattr(self, "thread", None):
            self.thread.join(timeout=2)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unsampled"],
                    "error": getattr(self, "error", None)}
        reasons = sorted({name for _, r in self.samples for bit, name in self.REASONS.items()
                          if r & bit})
        return {"sm_mhz": statistics.median(m for m, _ in self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(self.samples), "source": "nvml"}


# ---------------------------------------------------------------- distributed plumbing
def dist_init(args, backend=None):
    """One process per GPU: rank, world size, local rank and the process group
    (None for a single process).  The backend is NCCL when CUDA is present,
    gloo otherwise (or as given)."""
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    pg = None
    if world > 1:
        import datetime

        import torch.distributed as dist
        if backend is None:
            backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
        pg = dist
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return rank, world, local, pg


def max_over_ranks(value, pg):
    """The maximum of a per-rank value over all ranks (device timing is taken
    as the slowest rank's)."""
    if pg is None:
        return value
    import torch
    dev = "cuda" if pg.get_backend() == "nccl" else "cpu"
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


def barrier(pg):
    if pg is not None:
        pg.barrier()


def weak_scaling_value(per_step_units, steps, world, total_ms):
    """Whole-job throughput: every rank processes per_step_units per step (its
    own batch), and the job takes the slowest rank's time."""
    return per_step_units * steps * world / (total_ms * 1e-3)


# ---------------------------------------------------------------- roofline bits
def ntt_launch_work(limbs, batch=BATCH):
    """Algorithmic bytes and butterflies of one forward-NTT launch over `batch` polynomials at each
    limb count in `limbs` (one int, or a tuple for a grouped launch); the twiddle table of a prime
    is counted once per tensor."""
    if isinstance(limbs, int):
        limbs = (limbs,)
    bytes_ = mm = 0
    for l in limbs:
        jobs = l * batch
        bytes_ += jobs * 2 * N * 8 + l * N * 16  # data in+out, {w, w'} per prime
        mm += jobs * (N // 2) * 11
    return bytes_, mm


def traffic_for(kernel_key):
    """DRAM bytes per launch from the committed ncu summary, if the kernel's
    sources are unchanged since the capture (else None)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    e = json.load(open(p)).get(kernel_key)
    if not e:
        return None
    blob = b"".join(open(os.path.join(ROOT, f), "rb").read() for f in e["sources"])
    if hashlib.sha256(blob).hexdigest()[:16] != e.get("sources_sha256_16"):
        return None
    return e["dram_bytes_per_launch"]


def intpipe_peaks(ctx):
    """Same-run microbenchmarks over the whole GPU: Shoup multiplies/s,
    64x64->128 MACs/s and 64-bit high multiplies/s on the integer pipes, the
    forward NTT's own butterfly (kind 5), the key inner product's split-form
    product (kind 6, for primes 2^60 - delta), and int8 tcgen05.mma ops/s at
    N = 256 (dense rate) and N = 32 (the basis conversion's tile), one
    issuing thread per SM."""
    out = {}
    kinds = [(0, "shoup_mulmod_per_s", 2048), (1, "mac128_per_s", 2048), (2, "mulhi64_per_s", 2048),
             (5, "ntt_butterfly_per_s", 2048)]
    if all(q < 1 << 60 and (1 << 60) - q < 1 << 32 for q in ctx.mods):  # every prime 2^60 - delta
        kinds.append((6, "split_mac_per_s", 256))
    for kind, name, iters in kinds:
        best = 0.0
        for _ in range(3):
            ms, ops = ctx.bench_intpipe(kind, 148 * 8, iters)
            best = max(best, ops / (ms * 1e-3))
        out[name] = best
    for kind, name in ((3, "int8_mma_n256_ops_per_s"), (4, "int8_mma_n32_ops_per_s")):
        best = 0.0
        for _ in range(3):
            ms, ops = ctx.bench_intpipe(kind, 148, 4096)
            best = max(best, ops / (ms * 1e-3))
        out[name] = best
    return out


def rates_from(ipeak):
    """Per-operation rates of the roofline model (operations per second)."""
    return {"bfly": ipeak["ntt_butterfly_per_s"], "mm": ipeak["shoup_mulmod_per_s"],
            "mac": ipeak["mac128_per_s"], "int8_mac": ipeak["int8_mma_n256_ops_per_s"] / 2,
            "kmac": ipeak.get("split_mac_per_s", ipeak["mac128_per_s"])}


def ntt_roofline(limbs, k_ms, hbm_peak, peak_src, ipeak):
    """Roofline object of one forward-NTT launch over BATCH x limbs (or the grouped launch over a
    tuple of limb counts): the
    slower of its bytes at the measured HBM copy rate and its butterflies at
    the same-run rate of the kernel's own butterfly (microbenchmark kind 5).
    The generic Shoup rate (kind 0) is reported beside it."""
    bytes_, mm = ntt_launch_work(limbs)
    t = k_ms * 1e-3
    t_hbm = bytes_ / (hbm_peak * 1e9)
    t_alu = mm / ipeak["ntt_butterfly_per_s"]
    if t_alu > t_hbm:
        roof = {"bound": "alu", "achieved": mm / t / 1e9, "peak": ipeak["ntt_butterfly_per_s"] / 1e9,
                "unit": "G butterflies/s",
                "peak_source": "same-run microbenchmark of the kernel's own butterfly (kind 5)"}
    else:
        roof = {"bound": "hbm", "achieved": bytes_ / t / 1e9, "peak": hbm_peak, "unit": "GB/s",
                "peak_source": "%s MEASURED_PEAKS.json hbm_gbs" % peak_src}
    roof["frac"] = roof["achieved"] / roof["peak"]
    key = "ntt_fwd_group_" + "-".join(str(l) for l in limbs) if isinstance(limbs, tuple) else "ntt_fwd_%d" % limbs
    roof["traffic"] = traffic_for(key)
    roof["kernel"] = ("ntt_fwd_kernel<GroupJob> (%d x {%s} limbs, one launch)" % (BATCH, ", ".join(map(str, limbs)))
                      if isinstance(limbs, tuple) else "ntt_fwd_kernel<BatchJob> (%d x %d limbs)" % (BATCH, limbs))
    roof["launch_ms"] = k_ms
    roof["algorithmic_bytes"] = bytes_
    roof["butterflies"] = mm
    roof["hbm_frac_of_%s" % peak_src] = (bytes_ / t / 1e9) / hbm_peak
    roof["alu_frac_of_butterfly_microbench"] = (mm / t) / ipeak["ntt_butterfly_per_s"]
    roof["alu_frac_of_generic_shoup_microbench"] = (mm / t) / ipeak["shoup_mulmod_per_s"]
    return roof


# ---------------------------------------------------------------- GPU arm
def run_b200(args):
    import torch

    from rns_ckks_polynomial_b200 import Context, primes, synth

    rank, world, local, pg = dist_init(args)
    dev = torch.device("cuda", local)
    hbm_peak, peak_src = peaks()
    seed = synth.config_seed(2) + 1000 * rank
    top = max(max(SWEEP), 60)
    mods = primes(top + 60)
    ctx = Context(mods[:top], mods[top:top + 60], 60, device=local)

    xs = [synth.uniform_residues((BATCH, l, N), mods[:l], seed, l, device=dev) for l in SWEEP]
    refs = [x.clone() for x in xs]
    flush = torch.empty(L2_FLUSH_BYTES // 8, dtype=torch.int64, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(ev=None):
        # every sweep entry in one grouped launch per direction
        if ev is not None:
            ev[0].record(stream)
        ctx.ntt_fwd_group(xs)
        if ev is not None:
            ev[1].record(stream)
        ctx.ntt_inv_group(xs)

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()

    ipeak = intpipe_peaks(ctx)
    barrier(pg)
    torch.cuda.synchronize()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    kev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    with ClockSampler(dev) as clk:
        for s in range(args.steps):
            flush.zero_()  # L2 flush between steps, outside the timed events
            starts[s].record(stream)
            step(kev[s])
            ends[s].record(stream)
        torch.cuda.synchronize()
    barrier(pg)
    step_ms = [a.elapsed_time(b) for a, b in zip(starts, ends)]
    total_ms = max_over_ranks(sum(step_ms), pg)
    k_ms = statistics.mean(a.elapsed_time(b) for a, b in kev)
    # round trip must be the identity after W + K steps
    ok = all(torch.equal(x, r) for x, r in zip(xs, refs))
    ok = bool(max_over_ranks(0.0 if ok else 1.0, pg) == 0.0)

    per_step = 2 * BATCH * sum(SWEEP)
    value = weak_scaling_value(per_step, args.steps, world, total_ms)

    # roofline of the dominant kernel: the grouped forward NTT over every sweep entry
    roof = ntt_roofline(SWEEP, k_ms, hbm_peak, peak_src, ipeak)

    line = {
        "metric": METRIC, "value": value, "unit": "limb-NTTs/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "u64",
        "data": "synthetic (seeded uniform residues)",
        "config": {"workload": WORKLOAD, "n": N, "batch_per_gpu": BATCH, "limbs": list(SWEEP),
                   "primes": "60-bit, q = 1 mod 4096, descending from 2^60",
                   "l2": "flushed between steps (256 MiB write, outside the timed events)",
                   "parallelism": "replicas" if world > 1 else "single"},
        "roundtrip_identity": ok,
        "gpu_launches": 2 * args.steps,
        "roofline": roof,
        "intpipe_peaks": ipeak,
        "clocks": clk.summary(),
    }

    if not args.no_e2e:
        line["e2e"] = run_e2e(ctx, xs, refs, args, dev, stream, pg, world)
    # the key-switch rates come from the single-GPU run; under torchrun every
    # rank leaves together instead of waiting on rank 0's extra minutes
    if not args.no_ks and rank == 0 and world == 1:
        del xs, refs
        torch.cuda.empty_cache()
        line["keyswitch"] = run_keyswitch(dev, hbm_peak, ipeak,
                                          entries=tuple(e for e in args.ks_entries.split(",") if e))
    if rank == 0 and world == 1 and not args.no_cpu:
        line["cpu_baseline"] = cpu_baseline()
    if rank == 0:
        print(json.dumps(line), flush=True)
    if pg is not None:
        pg.destroy_process_group()


def run_e2e(ctx, xs, refs, args, dev, stream, pg, world):
    """Same metric through the public API from pinned host buffers: each step
    copies its inputs host->device, runs NTT then INTT, and reads the result
    back.  The inputs go in chunks of 2 polynomials through three streams, so
    the upload of a chunk, the transforms of the previous one and the download
    of the one before that overlap (PCIe is full duplex)."""
    import torch
    hosts = [r.cpu().pin_memory() for r in refs]
    backs = [torch.empty_like(h).pin_memory() for h in hosts]
    steps = max(3, min(args.steps, 10))
    chunks = [(h[c:c + 2], x[c:c + 2], bk[c:c + 2]) for h, x, bk in zip(hosts, xs, backs)
              for c in range(0, x.shape[0], 2)]
    s_in, s_cmp, s_out = (torch.cuda.Stream(dev) for _ in range(3))
    e_in = [torch.cuda.Event() for _ in chunks]
    e_cmp = [torch.cuda.Event() for _ in chunks]
    e_out = [torch.cuda.Event() for _ in chunks]

    def step():
        for i, (h, x, bk) in enumerate(chunks):
            with torch.cuda.stream(s_in):
                s_in.wait_event(e_out[i])  # the previous step's download of this buffer is done
                x.copy_(h, non_blocking=True)
                e_in[i].record(s_in)
            with torch.cuda.stream(s_cmp):
                s_cmp.wait_event(e_in[i])
                ctx.ntt_fwd(x)
                ctx.ntt_inv(x)
                e_cmp[i].record(s_cmp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(e_cmp[i])
                bk.copy_(x, non_blocking=True)
                e_out[i].record(s_out)

    for _ in range(2):
        step()
    torch.cuda.synchronize()
    barrier(pg)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(s_in)
    for _ in range(steps):
        step()
    b.record(s_out)
    torch.cuda.synchronize()
    ms = max_over_ranks(a.elapsed_time(b), pg)
    ok = all(torch.equal(bk, h) for bk, h in zip(backs, hosts))
    nbytes = sum(h.numel() * 8 for h in hosts)
    return {"value": 2 * BATCH * sum(SWEEP) * steps * world / (ms * 1e-3), "unit": "limb-NTTs/s",
            "h2d_bytes_per_step": nbytes, "d2h_bytes_per_step": nbytes, "steps": steps,
            "roundtrip_identity": ok, "pipelining": "chunks of 2 polynomials on 3 streams"}


def _time_call(fn, reps, stream, dev=None):
    """Mean device milliseconds of fn() over `reps` calls after 2 warm-up
    calls (CUDA events on the launching stream), and the clocks sampled while
    the timed calls ran."""
    import torch
    for _ in range(2):
        fn()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(dev if dev is not None else torch.device("cuda", torch.cuda.current_device())) as clk:
        a.record(stream)
        for _ in range(reps):
            fn()
        b.record(stream)
        torch.cuda.synchronize()
    return a.elapsed_time(b) / reps, clk.summary()


def _time_graph(fn, reps, stream, dev):
    """The same as _time_call for fn() captured once in a CUDA graph and replayed (the library
    calls take torch's current stream, which is the capture stream while capturing; their
    one-time tables are built by the eager warm-up calls first)."""
    import torch
    for _ in range(2):
        fn()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    torch.cuda.synchronize()
    ms, clk = _time_call(g.replay, reps, torch.cuda.current_stream(dev), dev)
    del g
    return ms, clk


KS_ENTRIES = ("tiny", "boot_rotation", "boot_rotation_integer", "boot_rotation_byteplanes",
              "boot_rotation_streamed", "layer", "layer_byteplanes", "bsgs", "bsgs_byteplanes", "refresh")


def run_keyswitch(dev, hbm_peak, ipeak, B=8, R=4, entries=KS_ENTRIES, refresh_batch=8):
    """Key switches per second of the key-switching workloads (B ciphertexts
    each; the boot-level rotation with R Galois keys), each with its roofline
    fraction and the clocks sampled while it ran.  `entries` selects which
    workloads are built at all (a smaller set for profiling)."""
    import torch

    from rns_ckks_polynomial_b200 import Context, primes, synth
    stream = torch.cuda.current_stream(dev)
    rates = rates_from(ipeak)
    out = {}
    if "tiny" in entries:
        # 4 + 1 primes, alpha = 1; 8 polynomials -> NTT -> pairwise product -> INTT, and one
        # rotation key switch of (P0, P1) with the Galois-5 key
        seed = synth.config_seed(1)
        m1 = primes(5)
        ctx = Context(m1[:4], m1[4:], 1, device=dev.index)
        polys = synth.uniform_residues((8, 4, N), m1[:4], seed, 1, device=dev)
        key = synth.uniform_residues((4, 2, 5, N), m1, seed, 2, device=dev)
        x = polys.clone()
        prod = torch.empty((4, 4, N), dtype=torch.int64, device=dev)
        rot = torch.empty((1, 1, 2, 4, N), dtype=torch.int64, device=dev)
        ws = torch.empty(ctx.workspace_bytes(4, 1, 1), dtype=torch.uint8, device=dev)

        def tiny():
            x.copy_(polys)
            ctx.ntt_fwd(x)
            ctx.pointwise("mul", x[0::2].contiguous(), x[1::2].contiguous(), out=prod)
            ctx.ntt_inv(prod)
            ctx.rotate(x[0:2].reshape(1, 2, 4, N), [key], [5], out=rot, ws=ws)

        ms, clk = _time_call(tiny, 50, stream, dev)
        w = work_sum(work(bfly=(8 + 4) * 4 * NTT_BFLY, mm=4 * 4 * N + 4 * 4 * N),
                     work_rotation(4, 1, 1, 1, 1))
        w["bytes"] = (8 * 4 + 4 * 4 + 2 * 4) * N * 8 + 4 * 2 * 5 * N * 8
        out["tiny_pipeline_L4"] = ks_entry(1, ms, w, hbm_peak, rates, clk)
        out["tiny_pipeline_L4"]["note"] = ("one call: 8 limb-4 NTTs, 4 products, 4 INTTs and one rotation; "
                                           "launch-bound at this size")
        ms, clk = _time_graph(tiny, 200, stream, dev)
        out["tiny_pipeline_L4_graph"] = ks_entry(1, ms, w, hbm_peak, rates, clk)
        out["tiny_pipeline_L4_graph"]["note"] = "the same call captured once in a CUDA graph and replayed"
        ctx.device_status()
        del ctx, polys, key, x, prod, rot, ws
    if any(e.startswith("boot_rotation") for e in entries):
        # boot-level hoisted rotation: L = 2100, K = 60, alpha = 60, R keys, B cts
        seed = synth.config_seed(5)
        mods = primes(2160)
        ctx = Context(mods[:2100], mods[2100:], 60, device=dev.index)
        ct = synth.uniform_residues((B, 2, 2100, N), mods[:2100], seed, 1, device=dev)
        keys = [synth.uniform_residues((35, 2, 2160, N), mods, seed, 10 + r, device=dev) for r in range(R)]
        gal = [5, 25, 625, 1505][:R]
        res = torch.empty((R, B, 2, 2100, N), dtype=torch.int64, device=dev)
        ws = torch.empty(ctx.workspace_bytes(4, B, R), dtype=torch.uint8, device=dev)
        if "boot_rotation" in entries:
            ms, clk = _time_call(lambda: ctx.rotate(ct, keys, gal, out=res, ws=ws), 10, stream, dev)
            out["boot_rotation_L2100"] = ks_entry(B * R, ms, work_rotation(2100, 60, 60, B, R), hbm_peak,
                                                  rates, clk)
            ctx.device_status()
        if "boot_rotation_integer" in entries:
            # the same call with both conversions on the integer pipes (bit-identical output)
            ctx.set_conversion("integer")
            ms, clk = _time_call(lambda: ctx.rotate(ct, keys, gal, out=res, ws=ws), 10, stream, dev)
            out["boot_rotation_L2100_integer_pipes"] = ks_entry(
                B * R, ms, work_rotation(2100, 60, 60, B, R, engine="integer"), hbm_peak, rates, clk)
            ctx.set_conversion("auto")
            ctx.device_status()
        if "boot_rotation_byteplanes" in entries:
            # the same call with both conversions on the byte-plane tensor-core form (bit-identical output)
            ctx.set_conversion("tensor")
            ms, clk = _time_call(lambda: ctx.rotate(ct, keys, gal, out=res, ws=ws), 10, stream, dev)
            out["boot_rotation_L2100_byteplanes"] = ks_entry(B * R, ms, work_rotation(2100, 60, 60, B, R),
                                                             hbm_peak, rates, clk)
            out["boot_rotation_L2100_byteplanes"]["conversion"] = "int8 tensor cores, byte planes"
            ctx.set_conversion("auto")
            ctx.device_status()
        if "boot_rotation_streamed" in entries:
            # the same rotations with ModUp -> NTT -> inner product streamed over windows of at most
            # 60 primes, without the [B][dnum][L+K][n] digit tensor (bit-identical output); the first
            # call builds the windows' conversion tables, outside the timing
            ws_s = torch.empty(ctx.workspace_bytes(11, B, R), dtype=torch.uint8, device=dev)
            ctx.rotate_streamed(ct, keys, gal, out=res, ws=ws_s)
            torch.cuda.synchronize(dev)
            ms, clk = _time_call(lambda: ctx.rotate_streamed(ct, keys, gal, out=res, ws=ws_s), 10, stream, dev)
            e = ks_entry(B * R, ms, work_rotation(2100, 60, 60, B, R), hbm_peak, rates, clk)
            e["workspace_bytes"] = int(ws_s.numel())
            e["hoisted_workspace_bytes"] = int(ws.numel())
            e["note"] = ("ModUp -> NTT -> key inner product per window of at most 60 primes (folded "
                         "conversion, two window buffers of B x 35 x 60 limbs on two streams); ModDown "
                         "as in the hoisted call")
            out["boot_rotation_L2100_streamed"] = e
            ctx.device_status()
            del ws_s
        del ct, keys, res, ws, ctx
        torch.cuda.empty_cache()
    if any(e.startswith("layer") or e.startswith("bsgs") for e in entries):
        mods = primes(120)
        ctx = Context(mods[:112], mods[112:], 8, device=dev.index)
    if "layer" in entries:
        # layer ct x ct multiply: L = 112, K = 8, alpha = 8, B pairs
        seed = synth.config_seed(3)
        a = synth.uniform_residues((B, 2, 112, N), mods[:112], seed, 1, device=dev)
        b = synth.uniform_residues((B, 2, 112, N), mods[:112], seed, 2, device=dev)
        rlk = synth.uniform_residues((14, 2, 120, N), mods, seed, 3, device=dev)
        res = torch.empty((B, 2, 111, N), dtype=torch.int64, device=dev)
        ws = torch.empty(ctx.workspace_bytes(6, B), dtype=torch.uint8, device=dev)
        ms, clk = _time_call(lambda: ctx.mul_relin_rescale(a, b, rlk, out=res, ws=ws), 20, stream, dev)
        out["layer_mul_relin_L112"] = ks_entry(B, ms, work_mrr(112, 8, 8, B), hbm_peak, rates, clk)
        ms, clk = _time_graph(lambda: ctx.mul_relin_rescale(a, b, rlk, out=res, ws=ws), 50, stream, dev)
        out["layer_mul_relin_L112_graph"] = ks_entry(B, ms, work_mrr(112, 8, 8, B), hbm_peak, rates, clk)
        out["layer_mul_relin_L112_graph"]["note"] = "the same call captured once in a CUDA graph and replayed"
        if "layer_byteplanes" in entries:
            ctx.set_conversion("tensor")
            ms, clk = _time_call(lambda: ctx.mul_relin_rescale(a, b, rlk, out=res, ws=ws), 20, stream, dev)
            out["layer_mul_relin_L112_byteplanes"] = ks_entry(B, ms, work_mrr(112, 8, 8, B), hbm_peak, rates, clk)
            out["layer_mul_relin_L112_byteplanes"]["conversion"] = "int8 tensor cores, byte planes"
            ctx.set_conversion("auto")
        del a, b, rlk, res, ws
    if "bsgs" in entries:
        # BSGS: bb = gg = 32, 62 keys, B cts
        seed = synth.config_seed(4)
        x = synth.uniform_residues((B, 2, 112, N), mods[:112], seed, 1, device=dev)
        diags = synth.uniform_residues((32, 32, 112, N), mods[:112], seed, 2, device=dev)
        bk = [synth.uniform_residues((14, 2, 120, N), mods, seed, 100 + i, device=dev) for i in range(31)]
        gk = [synth.uniform_residues((14, 2, 120, N), mods, seed, 200 + i, device=dev) for i in range(31)]
        y = torch.empty((B, 2, 111, N), dtype=torch.int64, device=dev)
        ws = torch.empty(ctx.workspace_bytes(7, B, 32032), dtype=torch.uint8, device=dev)
        ms, clk = _time_call(lambda: ctx.bsgs_lintrans(x, diags, bk, gk, 32, 32, out=y, ws=ws), 10, stream, dev)
        out["bsgs_L112_32x32"] = ks_entry(B * 62, ms, work_bsgs(112, 8, 8, B, 32, 32), hbm_peak, rates, clk)
        if "bsgs_byteplanes" in entries:
            ctx.set_conversion("tensor")
            ms, clk = _time_call(lambda: ctx.bsgs_lintrans(x, diags, bk, gk, 32, 32, out=y, ws=ws), 10, stream,
                                 dev)
            out["bsgs_L112_32x32_byteplanes"] = ks_entry(B * 62, ms, work_bsgs(112, 8, 8, B, 32, 32), hbm_peak,
                                                         rates, clk)
            out["bsgs_L112_32x32_byteplanes"]["conversion"] = "int8 tensor cores, byte planes"
            ctx.set_conversion("auto")
        del x, diags, bk, gk, y, ws
    if any(e.startswith("layer") or e.startswith("bsgs") for e in entries):
        ctx.device_status()
        del ctx
        torch.cuda.empty_cache()
    if "refresh" in entries:
        try:
            out["refresh_L2100"] = run_refresh(dev, hbm_peak, rates, B=refresh_batch)
        except Exception as e:  # noqa: BLE001 - reported in the line, the other entries stand
            out["refresh_L2100"] = {"error": repr(e)[:400]}
        torch.cuda.empty_cache()
    return out


# ---------------------------------------------------------------- algorithmic work model
NTT_BFLY = (N // 2) * 11  # butterflies per limb transform, one modular product each
TC_MIN_SOURCES = 8        # conversions with this many source primes run on the int8 tensor cores


def work(bfly=0, mm=0, mac=0, conv_tc=0, kmac=0, bytes=0):
    """Algorithmic work: NTT butterflies, other modular products, 60x60-bit
    multiply-adds (mac), of which conv_tc run as basis conversions on the int8
    tensor cores and kmac are the key inner product's, and the minimum bytes
    that cross HBM."""
    return {"bfly": bfly, "mm": mm, "mac": mac, "conv_tc": conv_tc, "kmac": kmac, "bytes": bytes}


def work_sum(*parts, times=1):
    out = work()
    for p in parts:
        for k in out:
            out[k] += p[k] * times
    return out


def ks_work_keyswitch_parts(L, K, alpha, engine="auto"):
    """Work of the parts of one hybrid key switch at n = 2048 (ModUp of one
    polynomial, the key inner product, ModDown of the two components)."""
    dnum = (L + alpha - 1) // alpha
    LK = L + K
    new_limbs = dnum * LK - L
    tc = engine != "integer"
    conv_up = conv_up_tc = 0
    for j in range(dnum):
        S = min(alpha, L - j * alpha)
        conv_up += S * (LK - S) * N
        if tc and S >= TC_MIN_SOURCES:
            conv_up_tc += S * (LK - S) * N
    conv_dn = 2 * K * L * N
    modup = work(bfly=(L + new_limbs) * NTT_BFLY, mm=L * N, mac=conv_up, conv_tc=conv_up_tc)
    inner = work(mac=2 * dnum * LK * N, kmac=2 * dnum * LK * N)
    moddown = work(bfly=2 * (K + L) * NTT_BFLY, mm=2 * (K + L) * N, mac=conv_dn,
                   conv_tc=conv_dn if tc and K >= TC_MIN_SOURCES else 0)
    return modup, inner, moddown


def work_rescale(l, B):
    """Rescale of B ciphertexts from l primes: INTT of the dropped limb, NTT of
    the l - 1 kept ones with the subtraction and q_l^-1 in the store."""
    return work(bfly=B * 2 * l * NTT_BFLY, mm=B * 2 * (l - 1) * N,
                bytes=B * 2 * (2 * l - 1) * N * 8)


def work_rotation(L, K, alpha, B, nkeys, engine="auto"):
    up, inner, down = ks_work_keyswitch_parts(L, K, alpha, engine)
    w = work_sum(work_sum(up, times=B), work_sum(inner, down, times=B * nkeys))
    dnum = (L + alpha - 1) // alpha
    w["bytes"] = nkeys * dnum * 2 * (L + K) * N * 8 + B * 2 * L * N * 8 * (1 + nkeys)
    return w


def work_mrr(L, K, alpha, B):
    up, inner, down = ks_work_keyswitch_parts(L, K, alpha)
    w = work_sum(up, inner, down, times=B)
    w = work_sum(w, work(mm=B * 4 * L * N), work_rescale(L, B))
    dnum = (L + alpha - 1) // alpha
    w["bytes"] = dnum * 2 * (L + K) * N * 8 + B * (4 * L + 2 * (L - 1)) * N * 8
    return w


def work_bsgs_plan(l, K, alpha, B, bb, gg, rotated_giants):
    """BSGS over bb x gg plaintext diagonals at l primes: one hoisted ModUp and
    bb - 1 baby key switches, the inner sums (one multiply-add per diagonal
    word and ciphertext component), `rotated_giants` full key switches and a
    rescale."""
    up, inner, down = ks_work_keyswitch_parts(l, K, alpha)
    w = work()
    if bb > 1:
        w = work_sum(w, up, work_sum(inner, down, times=bb - 1))
    w = work_sum(w, work_sum(up, inner, down, times=rotated_giants))
    w = work_sum(work_sum(w, times=B), work(mac=B * gg * bb * 2 * l * N), work_rescale(l, B))
    dnum = (l + alpha - 1) // alpha
    w["bytes"] = ((bb - 1 + rotated_giants) * dnum * 2 * (l + K) * N * 8 + gg * bb * l * N * 8
                  + B * (2 * l + 2 * (l - 1)) * N * 8)
    return w


def work_bsgs(L, K, alpha, B, bb, gg):
    return work_bsgs_plan(L, K, alpha, B, bb, gg, gg - 1)


def model_seconds(w, rates, hbm_peak, engine_tc=True):
    """(ALU seconds, HBM seconds) of a work dict.  The key inner product's
    multiply-adds (kmac) are charged at the same-run rate of its own split-form
    product (rates["kmac"]).  With engine_tc the conversions counted in conv_tc
    are charged as 64 int8 byte-plane multiply-adds per 60-bit multiply-add at
    the same-run dense int8 rate; otherwise they too run at the 128-bit MAC
    rate, as do the other multiply-adds."""
    t = w["bfly"] / rates["bfly"] + w["mm"] / rates["mm"] + w["kmac"] / rates.get("kmac", rates["mac"])
    rest = w["mac"] - w["kmac"]
    if engine_tc:
        t += (rest - w["conv_tc"]) / rates["mac"] + w["conv_tc"] * 64 / rates["int8_mac"]
    else:
        t += rest / rates["mac"]
    return t, w["bytes"] / (hbm_peak * 1e9)


def ks_entry(nks, ms, w, hbm_peak, rates, clocks=None):
    """One key-switching workload: rate, and roofline_frac = (the slower of
    its bytes at the measured HBM rate and its operations at the same-run
    rates of the engines that actually ran) / measured time.  NTT butterflies
    are charged at the kernel's own butterfly rate, other modular products at
    the Shoup rate, the key inner product's multiply-adds at the rate of its
    own split-form product, other multiply-adds at the 128-bit MAC rate, and
    conversions on the tensor cores at the dense int8 rate.  integer_pipe_model_frac charges
    every multiply-add to the integer pipes instead: a model the tensor-core
    path can exceed, so it is reported, not used as the bound."""
    t = ms * 1e-3
    t_alu, t_hbm = model_seconds(w, rates, hbm_peak, engine_tc=True)
    bound = "alu" if t_alu >= t_hbm else "hbm"
    out = {"keyswitches_per_s": nks / t, "ms_per_call": ms, "keyswitches_per_call": nks,
           "butterflies": w["bfly"], "mulmods": w["mm"], "macs": w["mac"], "macs_on_tensor_cores": w["conv_tc"],
           "macs_key_inner": w["kmac"],
           "min_bytes": w["bytes"], "bound": bound, "roofline_frac": max(t_alu, t_hbm) / t,
           "alu_frac": t_alu / t, "hbm_frac": t_hbm / t,
           "conversion": "int8 tensor cores, folded form" if w["conv_tc"] else "integer pipes"}
    if w["conv_tc"]:
        t_int, _ = model_seconds(w, rates, hbm_peak, engine_tc=False)
        out["integer_pipe_model_frac"] = max(t_int, t_hbm) / t
    if clocks is not None:
        out["clocks"] = clocks
    return out


# ---------------------------------------------------------------- CPU baselines
def cpu_model():
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def cpu_baseline(min_seconds=10.0):
    """The oracle as it stands, timed on this host's cores on bounded samples.

    - value: the bench step itself (16 polynomials at each of the sweep's limb
      counts, forward + inverse) on all cores, repeated until at least
      `min_seconds` have elapsed;
    - single_thread: one polynomial of each limb count on one thread (>= 3 s);
    - keyswitch: the key-switching workloads on all cores, each on a subset
      scaled linearly to the GPU workload: the boot-level rotation from one
      ciphertext's hoisted ModUp and one key's inner product + ModDown (then
      8 ModUps + 32 key switches), the layer multiply from one ciphertext
      pair, BSGS from one ciphertext."""
    import numpy as np

    import oracle
    from rns_ckks_polynomial_b200 import synth
    mods = oracle.gen_primes(N, max(SWEEP))
    xs = [synth.uniform_residues((BATCH, l, N), mods[:l], synth.config_seed(2), l).numpy().astype(np.uint64)
          for l in SWEEP]
    reps, t0 = 0, time.perf_counter()
    while True:
        for x in xs:
            oracle.ntt_inv(oracle.ntt_fwd(x, mods[:x.shape[1]]), mods[:x.shape[1]])
        reps += 1
        el = time.perf_counter() - t0
        if el >= min_seconds:
            break
    cores = oracle.num_threads()
    per_step = 2 * BATCH * sum(SWEEP)
    out = {"value": reps * per_step / el, "unit": "limb-NTTs/s", "cores": cores, "kind": "oracle",
           "sample": "%d repetitions of the bench step, 16 x {%s}-limb NTT + INTT (%.1f s)" % (
               reps, ", ".join(str(l) for l in SWEEP), el),
           "cpu_model": cpu_model()}
    # one thread
    oracle.set_num_threads(1)
    try:
        x1 = [np.ascontiguousarray(x[:1]) for x in xs]
        reps, t0 = 0, time.perf_counter()
        while True:
            for x in x1:
                oracle.ntt_inv(oracle.ntt_fwd(x, mods[:x.shape[1]]), mods[:x.shape[1]])
            reps += 1
            el = time.perf_counter() - t0
            if el >= 3.0:
                break
    finally:
        oracle.set_num_threads(cores)
    out["single_thread"] = {"value": reps * 2 * sum(SWEEP) / el, "unit": "limb-NTTs/s", "cores": 1,
                            "sample": "%d repetitions of 1 x {%s}-limb NTT + INTT (%.1f s)" % (
                                reps, ", ".join(str(l) for l in SWEEP), el)}
    del xs, x1
    ks = {}
    # boot-level rotation: L = 2100, K = 60, alpha = 60; the oracle's hoisted rotation of one
    # ciphertext under the 4 Galois elements of the GPU call (one ModUp, 4 key switches; one key
    # array serves all four, the work does not depend on its values); the GPU call's 8 ciphertexts
    # are independent of one another
    m5 = np.array(oracle.gen_primes(N, 2160), dtype=np.uint64)
    seed = synth.config_seed(5)
    c5 = synth.uniform_residues((1, 2, 2100, N), [int(x) for x in m5[:2100]], seed, 1).numpy().astype(np.uint64)
    key = synth.uniform_residues((35, 2, 2160, N), [int(x) for x in m5], seed, 10).numpy().astype(np.uint64)
    t0 = time.perf_counter()
    oracle.rotate(c5, [key] * 4, np.array([5, 25, 625, 1505], dtype=np.uint64), m5, 2100, 60, 60)
    t_rot = time.perf_counter() - t0
    ks["boot_rotation_L2100"] = {
        "keyswitches_per_s": 4 / t_rot, "unit": "key switches/s",
        "sample": "1 ciphertext rotated under 4 Galois elements (one hoisted ModUp, 4 key switches) in "
                  "%.1f s" % t_rot}
    del c5, key
    # layer multiply: L = 112, K = 8, alpha = 8, one ciphertext pair
    m3 = np.array(oracle.gen_primes(N, 120), dtype=np.uint64)
    seed = synth.config_seed(3)
    q3 = [int(x) for x in m3[:112]]
    ca = synth.uniform_residues((1, 2, 112, N), q3, seed, 1).numpy().astype(np.uint64)
    cb = synth.uniform_residues((1, 2, 112, N), q3, seed, 2).numpy().astype(np.uint64)
    rlk = synth.uniform_residues((14, 2, 120, N), [int(x) for x in m3], seed, 3).numpy().astype(np.uint64)
    t0 = time.perf_counter()
    oracle.mul_relin_rescale(ca, cb, rlk, m3, 112, 8, 8)
    t3 = time.perf_counter() - t0
    ks["layer_mul_relin_L112"] = {"keyswitches_per_s": 1 / t3, "unit": "key switches/s",
                                  "sample": "1 ciphertext pair (%.2f s)" % t3}
    # BSGS 32 x 32 at 112 primes: one ciphertext (62 key switches)
    seed = synth.config_seed(4)
    x4 = synth.uniform_residues((1, 2, 112, N), q3, seed, 1).numpy().astype(np.uint64)
    d4 = synth.uniform_residues((32, 32, 112, N), q3, seed, 2).numpy().astype(np.uint64)
    bk = [synth.uniform_residues((14, 2, 120, N), [int(x) for x in m3], seed, 100 + i).numpy().astype(np.uint64)
          for i in range(31)]
    gk = [synth.uniform_residues((14, 2, 120, N), [int(x) for x in m3], seed, 200 + i).numpy().astype(np.uint64)
          for i in range(31)]
    t0 = time.perf_counter()
    oracle.bsgs(x4, d4, bk, gk, 32, 32, m3, 112, 8, 8)
    t4 = time.perf_counter() - t0
    ks["bsgs_L112_32x32"] = {"keyswitches_per_s": 62 / t4, "unit": "key switches/s",
                             "sample": "1 ciphertext (62 key switches, %.1f s)" % t4}
    out["keyswitch"] = ks
    return out


def run_reference(args):
    """The CPU oracle as it stands, on the same workload, metric and unit:
    every step is the bench step itself (16 polynomials at each of the
    sweep's limb counts, forward NTT then inverse), on the host's cores."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import numpy as np

    import oracle
    from rns_ckks_polynomial_b200 import synth
    mods = oracle.gen_primes(N, max(SWEEP))
    xs = [synth.uniform_residues((BATCH, l, N), mods[:l], synth.config_seed(2), l).numpy().astype(np.uint64)
          for l in SWEEP]

    def step():
        for x in xs:
            oracle.ntt_inv(oracle.ntt_fwd(x, mods[:x.shape[1]]), mods[:x.shape[1]])

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    el = time.perf_counter() - t0
    per_step = 2 * BATCH * sum(SWEEP)
    value = per_step * args.steps / el
    cores = oracle.num_threads()
    sample = "the whole bench step per step: 16 x {%s}-limb NTT + INTT" % ", ".join(str(l) for l in SWEEP)
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": "limb-NTTs/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": el * 1e3 / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "u64", "data": "synthetic (seeded uniform residues)",
        "config": {"workload": WORKLOAD, "n": N, "batch_per_gpu": BATCH, "limbs": list(SWEEP),
                   "sample": sample},
        "cpu_baseline": {"value": value, "unit": "limb-NTTs/s", "cores": cores, "kind": "oracle",
                         "sample": sample, "cpu_model": cpu_model()},
        "e2e": {"value": value, "unit": "limb-NTTs/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }), flush=True)


def run_refresh(dev, hbm_peak, rates, B=8, L=2100, K=60, alpha=60, depth=3, r=9, reps=3):
    """The bootstrapping refresh of B ciphertexts on the boot chain (2100 + 60
    primes): modraise from q_0, `depth`-level factored coeff_to_slot and
    slot_to_coeff, conj_extract, two sin_folds of 6 + r levels, restore_merge.
    Each step is timed with CUDA events between its calls; coeff_to_slot and
    slot_to_coeff also get key switches/s and a roofline fraction.  Keys and
    plaintext diagonals are seeded uniform residues: the kernels' time does
    not depend on the values (the parity test runs the same schedule on the
    oracle's keys)."""
    import torch

    from rns_ckks_polynomial_b200 import primes, synth
    from rns_ckks_polynomial_b200.refresh import Refresh, factored_plans, plan_rotations
    seed = synth.config_seed(5) + 77
    mods = primes(L + K)
    q, p = mods[:L], mods[L:]
    dnum = (L + alpha - 1) // alpha
    cts_plans, stc_plans = factored_plans(N, depth)
    amounts = plan_rotations(cts_plans + stc_plans, N)

    def key(stream):
        return synth.uniform_residues((dnum, 2, L + K, N), mods, seed, stream, device=dev)

    keys = {"rot": {a: key(100 + i) for i, a in enumerate(amounts)}, "conj": key(90), "relin": key(91)}

    def levels(plans, top, stream):
        return [(pl, synth.uniform_residues((pl[3], pl[2], top - i, N), q[:top - i], seed, stream + i,
                                            device=dev)) for i, pl in enumerate(plans)]

    stc_top = L - depth - 6 - r
    cts = levels(cts_plans, L, 200)
    stc = levels(stc_plans, stc_top, 300)
    ct = synth.uniform_residues((B, 2, 1, N), q[:1], seed, 1, device=dev)
    rf = Refresh(q, p, alpha, keys, device=dev.index)
    stream = torch.cuda.current_stream(dev)
    steps = ["modraise", "coeff_to_slot", "conj_extract", "sin_fold_re", "sin_fold_im", "restore_merge",
             "slot_to_coeff"]
    per = {k: 0.0 for k in steps}
    try:
        for _ in range(2):
            rf.refresh(ct, r, cts, stc)
        torch.cuda.synchronize()
        total = 0.0
        with ClockSampler(dev) as clk:
            for _ in range(reps):
                evs = []

                def mark(name):
                    e = torch.cuda.Event(enable_timing=True)
                    e.record(stream)
                    evs.append((name, e))

                start = torch.cuda.Event(enable_timing=True)
                start.record(stream)
                rf.refresh(ct, r, cts, stc, mark=mark)
                torch.cuda.synchronize()
                prev = start
                for name, e in evs:
                    per[name] += prev.elapsed_time(e) / reps
                    prev = e
                total += start.elapsed_time(evs[-1][1]) / reps
    finally:
        rf.close()
    S = N // 2

    def transform(plans, top):
        ks, w = 0, work()
        for i, (stride, t0, bb, gg) in enumerate(plans):
            rotated = sum(1 for g in range(gg) if (stride * (t0 + bb * g)) % S)
            ks += (bb - 1) + rotated
            w = work_sum(w, work_bsgs_plan(top - i, K, alpha, B, bb, gg, rotated))
        return ks, w

    out = {"workload": "refresh of %d ciphertexts, %d + %d primes, alpha %d, factored transforms of "
                       "depth %d, sin_fold r = %d (%d levels)" % (B, L, K, alpha, depth, r, 2 * depth + 6 + r),
           "ms_per_call": total, "ciphertext_refreshes_per_s": B / (total * 1e-3),
           "ms_per_step": per, "share_per_step": {k: v / total for k, v in per.items()},
           "keys": len(amounts) + 2, "clocks": clk.summary(),
           "pages_cpu_s_for_8_ciphertexts": 4393.5,
           "data": "seeded uniform residues for keys, plaintexts and the input ciphertexts"}
    for name, plans, top in (("coeff_to_slot", cts_plans, L), ("slot_to_coeff", stc_plans, stc_top)):
        ks, w = transform(plans, top)
        e = ks_entry(B * ks, per[name], w, hbm_peak, rates)
        e["plans"] = [list(pl) for pl in plans]
        e["key_switches_per_ciphertext"] = ks
        e["pages_cpu_s_for_8_ciphertexts"] = 1737.20 if name == "coeff_to_slot" else 1736.19
        out[name] = e
    return out


def run_ks_only(args):
    """Only the selected key-switching workloads (--ks-entries), for
    profiling: nothing else is built, so a capture holds only that workload's
    keys and workspace on the device."""
    import torch
    dev = torch.device("cuda", 0)
    hbm_peak, _ = peaks()
    from rns_ckks_polynomial_b200 import Context, primes
    ctx = Context(primes(60), primes(61)[60:], 60)
    ipeak = intpipe_peaks(ctx)
    ctx.close()
    entries = tuple(e for e in args.ks_entries.split(",") if e)
    print(json.dumps({"keyswitch": run_keyswitch(dev, hbm_peak, ipeak, args.ks_batch, args.ks_keys,
                                                 entries, refresh_batch=args.ks_batch),
                      "intpipe_peaks": ipeak}), flush=True)


def main():
    args = parse()
    if args.refresh_only:
        args.ks_only, args.ks_entries = True, "refresh"
    if args.ks_only:
        run_ks_only(args)
        return
    global SWEEP
    SWEEP = tuple(int(x) for x in args.sweep.split(","))
    if args.impl == "reference":
        run_reference(args)
    else:
        run_b200(args)


if __name__ == "__main__":
    main()
