"""The multi-process path of bench.py on CPU: two gloo ranks (one process
each, as torchrun starts them) exercise the rank setup, the barrier, the
max-over-ranks timing reduction, the whole-job (weak-scaling) throughput and
the reference arm, which runs on rank 0 only.  No GPU is involved."""
import contextlib
import io
import json
import os
import socket
import sys
from types import SimpleNamespace

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, outdir):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    if ROOT not in sys.path:
        sys.path.insert(0, ROOT)
    import bench
    r, w, _, pg = bench.dist_init(None, backend="gloo")
    # each rank reports its own elapsed time; the job takes the slowest
    slowest = bench.max_over_ranks(10.0 * (rank + 1), pg)
    bench.barrier(pg)
    # the plumbing is under test, not the oracle's speed: a two-size sweep keeps rank 0's reference
    # run far inside the process group's timeout on a busy host
    bench.SWEEP, bench.BATCH = (3, 112), 2
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        bench.run_reference(SimpleNamespace(gpus=world, steps=1, warmup=0))
    bench.barrier(pg)
    with open(os.path.join(outdir, "rank%d.json" % rank), "w") as f:
        json.dump({"rank": r, "world": w, "slowest": slowest, "reference": buf.getvalue()}, f)
    pg.destroy_process_group()


def test_two_gloo_ranks(tmp_path):
    import torch.multiprocessing as mp

    import oracle
    oracle.num_threads()  # builds the oracle once, before the ranks start
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       start_method="spawn", join=True)
    res = [json.load(open(tmp_path / ("rank%d.json" % r))) for r in range(world)]
    assert [(x["rank"], x["world"]) for x in res] == [(0, 2), (1, 2)]
    assert all(x["slowest"] == 20.0 for x in res)
    # the reference arm prints one JSON line on rank 0 and nothing elsewhere
    assert res[1]["reference"] == ""
    lines = res[0]["reference"].strip().splitlines()
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2
    assert line["unit"] == "limb-NTTs/s" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0


def test_weak_scaling_value():
    if ROOT not in sys.path:
        sys.path.insert(0, ROOT)
    import bench
    # 2 ranks x 100 units per step x 5 steps in 0.5 s (slowest rank) = 2000 units/s
    assert bench.weak_scaling_value(100, 5, 2, 500.0) == pytest.approx(2000.0)
    assert bench.weak_scaling_value(100, 5, 1, 500.0) == pytest.approx(1000.0)
