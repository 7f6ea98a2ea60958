"""Host-side checks of the multi-rank bench path on CPU: two ``gloo`` ranks.

The decode path shards whole sequences across ranks with no collective; the
only cross-rank step is the max-over-ranks reduction of the timings, and the
reference arm runs on rank 0 alone.
"""

import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import bench
    from mla_latent_kv_45_b200 import synth
    import torch.distributed as dist
    r, w, _ = bench.setup_dist(None, backend="gloo")
    wl = bench.workload("v2_batch64", r)
    lens = synth.make_prior_lengths(wl)
    # every rank reports different timings; all must see the slowest
    got = bench.max_over_ranks([1.0 + r, 10.0 * (w - r), 3.0], w, "cpu")
    # the reference arm: rank 0 alone does work
    calls = []
    real = bench.workload
    bench.workload = lambda *a, **k: calls.append(1) or real(*a, **k)
    if r != 0:
        bench.run_reference(type("A", (), {"workload": "v2_batch64", "steps": 1, "warmup": 0})())
    bench.workload = real
    out.put((r, w, wl.wid, lens.tolist(), got, len(calls)))
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks_shard_and_reduce():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=240) for _ in procs)
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    (r0, w0, wid0, lens0, got0, c0), (r1, w1, wid1, lens1, got1, c1) = res
    assert (r0, r1, w0, w1) == (0, 1, 2, 2)
    # distinct shards of sequences with the same shape
    assert wid0 != wid1 and len(lens0) == len(lens1)
    assert not np.array_equal(lens0, lens1)
    # max over ranks, identical on both
    assert got0 == got1 == [2.0, 20.0, 3.0]
    # rank 1 returned from the reference arm without building its workload
    assert c1 == 0


def test_stored_traffic_only_for_the_captured_sources(tmp_path):
    import json
    import bench
    f = tmp_path / "t.json"
    f.write_text(json.dumps({"workload": "v2_batch64", "kernel_rev": bench.kernel_revision(),
                             "dram_bytes_per_launch": 123}))
    assert bench.stored_traffic("v2_batch64", str(f)) == 123
    assert bench.stored_traffic("v2_step128", str(f)) is None
    f.write_text(json.dumps({"workload": "v2_batch64", "kernel_rev": "0" * 16,
                             "dram_bytes_per_launch": 123}))
    assert bench.stored_traffic("v2_batch64", str(f)) is None
    assert bench.stored_traffic("v2_batch64", str(tmp_path / "missing.json")) is None


def test_bench_gpus_flag_starts_ranks():
    """``bench.py --gpus 2`` outside torchrun starts two ranks itself; the
    plumbing check runs them on CPU (gloo) through the same max-over-ranks
    reduction, and rank 0 alone prints one line with n_gpus = 2."""
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--gpus", "2",
                        "--rank-check"], capture_output=True, text=True, timeout=300,
                       env={**os.environ, "OMP_NUM_THREADS": "1"})
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [json.loads(x) for x in r.stdout.splitlines() if x.startswith("{")]
    assert len(lines) == 1, r.stdout
    # the max over ranks of 1 + rank, and of the ranks' workload seeds (base + 100 rank)
    import bench
    assert lines[0] == {"n_gpus": 2, "max_ms": 2.0,
                        "max_wid": float(bench.workload("v2_batch64", 1).wid)}
