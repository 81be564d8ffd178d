"""The N > 1 host path of the benchmark on CPU: two ranks over gloo (no GPU needed).

The gated prefill shards by request, so N GPUs run N independent replicas, each on its
own seeded batch, with no collective on the data path; the only collectives are the
timing's max over ranks (and barriers).  These tests run that host logic in two spawned
processes: per-rank batches differ while shapes and weights do not, every rank sees the
slowest rank's time, and the whole-job rate counts every rank's tokens.
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
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch
    import torch.distributed as dist

    import bench
    import synthetic_inputs as S

    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        base = S.pr1_ref()
        wl = bench.replica_workload(base, rank, world)
        h = S.hidden_rows(wl)
        w = S.layer_weights(wl, 0)
        slowest = bench.max_over_ranks(10.0 + 5.0 * rank, world, "cpu")
        dist.barrier()
        rate = bench.whole_job_rate(wl.total_tokens, world, 4, slowest)
        q.put((rank, tuple(wl.seeds), wl.lengths, float(h.float().sum()),
               float(w["Wqkv"].float().sum()), slowest, rate))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_run_independent_replicas():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = {}
    try:
        for _ in range(2):
            r = q.get(timeout=120)
            out[r[0]] = r
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert all(p.exitcode == 0 for p in procs)
    r0, r1 = out[0], out[1]
    assert r0[1] != r1[1]                  # each rank draws its own batch ...
    assert r0[2] == r1[2]                  # ... of the same shape
    assert r0[3] != r1[3]
    assert r0[4] == r1[4]                  # same weights on every replica
    assert r0[5] == r1[5] == 15.0          # both see the slowest rank's time
    tokens = 1024
    assert r0[6] == pytest.approx(tokens * 2 * 4 / 15.0e-3)


def test_single_rank_helpers_are_identity():
    sys.path.insert(0, ROOT)
    import bench
    import synthetic_inputs as S
    wl = S.pr1_ref()
    assert bench.replica_workload(wl, 0, 1) is wl
    assert bench.max_over_ranks(3.5, 1, "cpu") == 3.5


def test_reference_arm_prints_only_on_rank_zero():
    """Under torchrun the reference arm (the CPU oracle) runs on rank 0 alone; any other
    rank exits 0 at once without output."""
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "0"], env=env, capture_output=True,
                       text=True, timeout=120)
    assert r.returncode == 0 and r.stdout.strip() == ""
