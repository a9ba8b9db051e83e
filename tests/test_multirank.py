"""The multi-rank plumbing of bench.py on CPU: two gloo ranks, each with its own seeded shard
of the same shape (weak scaling, no data-path collective), the job time taken as the max over
ranks, and the reference arm printing on rank 0 only."""
import contextlib
import datetime
import hashlib
import io
import os
import socket
import sys

import pytest

torch = pytest.importorskip("torch")
import torch.multiprocessing as mp  # noqa: E402

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    w = bench.WORKLOADS["tiny"](rank)
    digest = hashlib.sha256(w.W_bits.tobytes() + w.X_bits.tobytes()).hexdigest()
    t_local = 0.001 * (rank + 1)
    t_max = bench.max_over_ranks(t_local, dist, torch.device("cpu"))
    value = bench.job_value(2.0 * w.M * w.K * w.N, world, t_max)
    dist.barrier()
    dist.destroy_process_group()
    # the reference arm: rank 0 prints one JSON line, the others exit 0 without work
    out = io.StringIO()
    args = type("A", (), dict(steps=1, warmup=0, gpus=world))()
    with contextlib.redirect_stdout(out):
        rc = bench.run_reference(args, w)
    q.put((rank, t_max, value, digest, (w.M, w.K, w.N, w.T), rc, out.getvalue()))


def test_two_gloo_ranks_shards_max_timing_and_reference_arm():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = {}
    try:
        for _ in range(2):
            r = q.get(timeout=240)
            res[r[0]] = r
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert all(p.exitcode == 0 for p in procs)
    r0, r1 = res[0], res[1]
    assert r0[1] == r1[1] == pytest.approx(0.002)          # max over ranks, seen by both
    assert r0[2] == r1[2]                                    # same job value on every rank
    M, K, N, T = r0[4]
    assert r0[2] == pytest.approx(2 * (2.0 * M * K * N) / 0.002 / 1e12)
    assert r0[4] == r1[4]                                    # same shape (weak scaling) ...
    assert r0[3] != r1[3]                                    # ... different seeded shard
    assert r0[5] == 0 and r1[5] == 0
    import json
    line = json.loads(r0[6].strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["cpu_baseline"]["kind"] == "oracle"
    assert r1[6].strip() == ""                               # rank 1 prints nothing
