"""The multi-rank host logic of bench.py on CPU (gloo, world size 2).

The scan shards by (b, h) pairs with no data-path collective, so the only
multi-process logic is plumbing: every rank gets its own data, and the job's
time is the slowest rank's.  The reference arm runs on rank 0 only.
"""
import datetime
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    import bench
    import synth
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world, timeout=datetime.timedelta(seconds=60))
    t = bench.max_over_ranks(0.5 + rank, device="cpu")
    spec = bench.rank_spec(synth.workload("gdn_720p_60s"), rank)
    first = synth.slice_storage(spec.with_(F=1, H=1), "q", 0, 0).tobytes()[:64]
    q.put((rank, t, spec.seed, first))
    dist.barrier()
    dist.destroy_process_group()


def test_two_ranks_take_the_max_time_and_own_data():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, t0, s0, d0), (r1, t1, s1, d1) = res
    assert t0 == t1 == 1.5                      # max over ranks, seen by every rank
    assert s0 != s1 and d0 != d1                # each rank scans its own batch


def test_single_process_max_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(2.25) == 2.25


def test_reference_arm_other_ranks_exit_quietly():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--steps", "1", "--warmup", "0"], env=env,
                       capture_output=True,
                       text=True, timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == ""
