"""The multi-rank plumbing of bench.py on CPU (gloo ranks): every rank draws the same problem
and takes its tiles of it, the job time is the max over ranks and the job value the whole
problem's FLOPs over it, the reference arm prints on rank 0 only; and the tile-sharded split
itself (ranges, and the per-rank results against the unsharded run)."""
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
    w = bench.WORKLOADS["tiny"]()
    digest = hashlib.sha256(w.W_bits.tobytes() + w.X_bits.tobytes()).hexdigest()
    t_local = 0.001 * (rank + 1)
    t_max = bench.max_over_ranks(t_local, dist, torch.device("cpu"))
    value = bench.job_value(2.0 * w.M * w.K * w.N, t_max)
    dist.barrier()
    dist.destroy_process_group()
    # the reference arm: rank 0 prints one JSON line, the others exit 0 without work
    out = io.StringIO()
    args = type("A", (), dict(steps=1, warmup=0, gpus=world))()
    with contextlib.redirect_stdout(out):
        rc = bench.run_reference(args, w)
    q.put((rank, t_max, value, digest, (w.M, w.K, w.N, w.T), rc, out.getvalue()))


def test_two_gloo_ranks_same_problem_max_timing_and_reference_arm():
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
    assert r0[2] == pytest.approx((2.0 * M * K * N) / 0.002 / 1e12)  # whole problem / max time
    assert r0[4] == r1[4] and r0[3] == r1[3]                 # one problem, split by tiles
    assert r0[5] == 0 and r1[5] == 0
    import json
    line = json.loads(r0[6].strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["cpu_baseline"]["kind"] == "oracle"
    assert r1[6].strip() == ""                               # rank 1 prints nothing


# ---------------------------------------------------------------- tile-sharded split
def test_shard_tiles_cover_rows_exactly():
    """Contiguous runs of whole tiles, in rank order, covering [0, M) exactly; sizes differ by
    at most one tile; ranks beyond the tile count get empty ranges."""
    import pruning_hinm_spmm_b200 as H
    for M, T in ((11008, 128), (4096, 128), (256, 64), (640, 64), (128, 128)):
        nt = M // T
        for world in (1, 2, 3, 4, 7, 8, 16):
            rng = [H.shard_tiles(M, T, world, r) for r in range(world)]
            assert rng[0][0] == 0 and rng[-1][1] == M
            for (a0, a1), (b0, b1) in zip(rng, rng[1:]):
                assert a1 == b0
            sizes = [(r1 - r0) // T for r0, r1 in rng]
            assert all((r1 - r0) % T == 0 and r1 >= r0 for r0, r1 in rng)
            assert max(sizes) - min(sizes) <= 1 and sum(sizes) == nt
    with pytest.raises(ValueError):
        H.shard_tiles(200, 64, 2, 0)


def _shard_worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import numpy as np
    import torch.distributed as dist
    import bench
    import hinm_inputs as hi
    import pruning_hinm_spmm_b200 as H
    from oracle import hinm_oracle as O
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    # 10 tiles of 64 rows over the ranks; X (and the permutation) replicated
    w = hi.custom(640, 256, 24, 64, seed=11, t_s=0.625, v_s=None, random_perm=True)
    r0, r1 = H.shard_tiles(w.M, w.T, world, rank)
    part = O.hot_path(w.W_bits[r0:r1], w.X_bits, w.perm, w.T, w.t_s, w.alpha)
    L = part["layout"]
    blocks = []
    for t in range(L.tile_info.shape[0]):
        nd, ns, d0, s0 = (int(x) for x in L.tile_info[t])
        blocks.append((L.vals_dense[d0:d0 + nd].tobytes(), L.vals_sparse[s0:s0 + ns].tobytes(),
                       L.meta[s0:s0 + ns].tobytes(), L.idx_dense[d0:d0 + nd].tobytes(),
                       L.idx_sparse[s0:s0 + ns].tobytes()))
    Y = bench.gather_rows(torch.from_numpy(part["y"]), w.M, w.T, world, dist, H.shard_tiles)
    gathered = [None] * world
    dist.all_gather_object(gathered, dict(rows=(r0, r1), counts=part["counts"],
                                          bitmask=part["bitmask"], region=part["region"],
                                          blocks=blocks))
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, Y.numpy(), gathered))


def test_tile_sharded_run_equals_unsharded():
    """Two gloo ranks each run the oracle's whole path on their tile shard of one W (X
    replicated); concatenated in rank order, their counts, masks, regions, per-tile layout
    bytes and Y rows (the Y rows through the same all-gather the benchmark uses) equal the
    unsharded run's."""
    import numpy as np
    import hinm_inputs as hi
    from oracle import hinm_oracle as O
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    world = 2
    procs = [ctx.Process(target=_shard_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = {}
    try:
        for _ in range(world):
            r = q.get(timeout=300)
            res[r[0]] = r
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert all(p.exitcode == 0 for p in procs)
    w = hi.custom(640, 256, 24, 64, seed=11, t_s=0.625, v_s=None, random_perm=True)
    full = O.hot_path(w.W_bits, w.X_bits, w.perm, w.T, w.t_s, w.alpha)
    parts = res[0][2]
    assert [p["rows"] for p in parts] == [(0, 320), (320, 640)]
    np.testing.assert_array_equal(np.concatenate([p["counts"] for p in parts]), full["counts"])
    np.testing.assert_array_equal(np.concatenate([p["bitmask"] for p in parts]), full["bitmask"])
    np.testing.assert_array_equal(np.concatenate([p["region"] for p in parts]), full["region"])
    L = full["layout"]
    blocks = [b for p in parts for b in p["blocks"]]
    for t in range(L.tile_info.shape[0]):
        nd, ns, d0, s0 = (int(x) for x in L.tile_info[t])
        want = (L.vals_dense[d0:d0 + nd].tobytes(), L.vals_sparse[s0:s0 + ns].tobytes(),
                L.meta[s0:s0 + ns].tobytes(), L.idx_dense[d0:d0 + nd].tobytes(),
                L.idx_sparse[s0:s0 + ns].tobytes())
        assert blocks[t] == want, f"tile {t}"
    for r in range(world):  # the gathered Y on every rank: the unsharded rows
        np.testing.assert_allclose(res[r][1], full["y"], rtol=1e-13, atol=1e-13)
