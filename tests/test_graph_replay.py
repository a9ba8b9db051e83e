"""The five calls of the path captured in a CUDA graph (as bench.py times them) give the same
bytes as the same calls launched eagerly, on the benchmark workload's shape family, with and
without a materialized importance.  The kernels are launched with programmatic stream
serialization, which a capture turns into programmatic graph edges; back-to-back replays
check that every kernel still sees its predecessors' writes."""
import numpy as np
import pytest

import hinm_inputs as hi

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def H():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import pruning_hinm_spmm_b200 as H
    return H


def dev_bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


@pytest.mark.parametrize("materialize", [True, False], ids=["with_I", "from_W"])
@pytest.mark.parametrize("fixed", [True, False], ids=["fixed_counts", "searched"])
def test_graph_replay_matches_eager(H, fixed, materialize):
    w = hi.custom(512, 1024, 256, 128, seed=77, t_s=0.5, v_s=0.25 if fixed else None,
                  random_perm=True)
    M, K, N, T = w.M, w.K, w.N, w.T
    W, X = dev_bf16(w.W_bits), dev_bf16(w.X_bits)
    perm = torch.from_numpy(w.perm).cuda()
    counts = None
    if fixed:
        c = H.hinm_counts_from_vs(K, w.t_s, w.v_s)
        counts = torch.tensor([c] * (M // T), dtype=torch.int32, device="cuda")
    hp = H.HotPath(M, K, N, T, w.t_s, w.alpha, materialize_importance=materialize)
    hp.layout.vals_sparse.zero_()  # blocks beyond those in use are never written
    hp.run(W, X, perm, fixed_counts=counts)  # eager; also every one-time set-up
    torch.cuda.synchronize()
    keys = ("I", "counts", "vs", "rank", "bitmask", "region", "Y") if materialize else \
        ("counts", "vs", "rank", "bitmask", "region", "Y")
    ref = {k: getattr(hp, k).clone() for k in keys}
    ref_vals = hp.layout.vals_sparse.clone()
    for k in ("I", "Y", "bitmask") if materialize else ("Y", "bitmask"):
        getattr(hp, k).zero_()
    hp.layout.vals_sparse.zero_()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        hp.run(W, X, perm, fixed_counts=counts)
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    assert H.hinm_device_status() == 0
    for k, v in ref.items():
        assert torch.equal(getattr(hp, k), v), k
    assert torch.equal(hp.layout.vals_sparse, ref_vals)
    del g
