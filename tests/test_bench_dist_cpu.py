"""The multi-rank plumbing of bench.py on CPU: two gloo ranks (spawned
processes, rendezvous on 127.0.0.1) exercise the per-rank batches, the
max-over-ranks timing and the whole-job throughput that the GPU run uses
under torchrun.  The path shards by utterance, so there is no data-path
collective to test: only the timing reduction crosses ranks."""
import os
import socket
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import datetime
    import torch
    import torch.distributed as dist
    import bench

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        pcm, off = bench.rank_batch(rank, world, n_clips=2)
        local_ms = 10.0 + 5.0 * rank                     # rank 1 is the slow one
        total_ms = bench.reduce_max(dist, local_ms, torch.device("cpu"))
        frames = 2 * bench.FRAMES_PER_CLIP
        value = bench.job_throughput(frames, world, 4, total_ms)
        q.put((rank, float(pcm[:1000].sum()), int(off[-1]), total_ms, value))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_two_gloo_ranks_time_as_the_slowest_rank():
    import torch.multiprocessing as mp

    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=240) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, sum0, n0, t0, v0), (r1, sum1, n1, t1, v1) = res
    assert (r0, r1) == (0, 1)
    assert n0 == n1 == 2 * 480000                       # weak scaling: the same work per rank
    assert sum0 != sum1                                 # ...on different clips
    assert t0 == t1 == 15.0                             # both report the slowest rank's time
    expect = 2 * 2998 * 2 * 4 / (15.0 / 1e3)
    assert v0 == v1 and abs(v0 - expect) < 1e-6 * expect


def test_single_rank_helpers_without_a_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.reduce_max(None, 3.5, None) == 3.5
    assert bench.job_throughput(2998, 1, 10, 1000.0) == pytest.approx(29980.0)
    w, r, l = bench.dist_env()
    assert (w, r, l) == (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
                         int(os.environ.get("LOCAL_RANK", "0")))


def test_reference_arm_under_torchrun_prints_one_line():
    # launched the way a multi-GPU run is: rank 0 times the oracle and prints
    # the line; the other rank exits 0 without work (the arm needs no GPU)
    import json
    import subprocess
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()),
           os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2", "--steps", "3", "--warmup", "3"]
    res = subprocess.run(cmd, capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [json.loads(s) for s in res.stdout.splitlines() if s.startswith("{")]
    assert len(lines) == 1
    line = lines[0]
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["e2e"]["h2d_bytes_per_step"] == 0
