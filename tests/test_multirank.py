"""The multi-rank host path of bench.py on CPU: two gloo ranks.

bench.py runs one independent chunk stream per GPU and reports the whole
job's throughput over the slowest rank's device time; these tests run that
plumbing (per-rank workload, max over ranks, job throughput, the reference
arm's rank handling) as two processes on the gloo backend.
"""
import os
import socket
import subprocess
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import datetime
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    from gated_deltanet_linear_chunked_b200 import workloads as wl
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        w = wl.stream_chunk("fwd")
        wr = bench.rank_workload(w, rank)
        ms = 10.0 + 5.0 * rank                      # this rank's "device time"
        mx = bench.max_over_ranks(ms, world)
        val = bench.job_throughput(world, 4, w.head_tokens, mx)
        # a small slice of this rank's inputs, to compare streams across ranks
        x = wl.make_inputs(wl.Workload("probe", 1, 64, 2, 16, 16, "bf16", 64, "fwd",
                                       wr.gate, wr.beta, wr.state, wr.seed))
        out.put((rank, wr.seed, mx, val, x["q"].ravel()[:32].tolist()))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_max_time_and_independent_streams():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    seeds = [r[1] for r in res]
    assert len(set(seeds)) == world                     # independent chunk streams
    assert all(r[2] == 15.0 for r in res)               # every rank sees the slowest time
    from gated_deltanet_linear_chunked_b200 import workloads as wl
    ht = wl.stream_chunk("fwd").head_tokens
    assert all(r[3] == pytest.approx(2 * 4 * ht / 0.015) for r in res)
    assert not np.allclose(res[0][4], res[1][4])         # different inputs per rank


def test_job_throughput_and_single_rank_max():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.job_throughput(1, 10, 1000, 2.0) == pytest.approx(5e6)
    assert bench.job_throughput(8, 10, 1000, 2.0) == pytest.approx(4e7)


def test_reference_arm_other_ranks_exit_without_work():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--steps", "1", "--warmup", "0"],
                       env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0
    assert r.stdout.strip() == ""
