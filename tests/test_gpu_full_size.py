"""GPU parity at full size: every output row, every mask bit.

The benchmark workloads (pure 2:4 4096x4096x2048, HiNM up-proj 11008x4096x4096 with a
random permutation, decode down-proj 4096x11008x16) in the launch configuration the
benchmark times, and layer 0 of the LLaMA-2-7B-shaped sweep in all 27 (linear shape, N,
t_s) cases with the boundary from the search.  Against the CPU oracle:

* I (every element, bit for bit);
* the benchmark's path does not materialize I (the search and the mask recompute it from W
  and the channel energies); the sweep runs both ways and they agree bit for bit;
* the boundary search (counts, v_s, rank and every candidate's R(m), bit for bit) on
  sampled tiles -- the oracle's exact scan costs about a second per tile;
* the mask and the regions of every tile (bit for bit), with the counts the GPU used (its
  own search's, checked where sampled, or the workload's fixed boundary);
* the compressed layout's bytes on the sampled tiles (the oracle packs in Python loops);
* Y, every element: |y - y_ref| <= 1e-3 * sum|w||x| + 1e-5 (fp64 masked product).
"""
import numpy as np
import pytest

import hinm_inputs as hi
from oracle import hinm_oracle as O

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

from test_gpu_parity import check_y, dev_bf16, dev_i32, layout_equal, status_ok  # noqa: E402


@pytest.fixture(scope="module")
def H():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import pruning_hinm_spmm_b200 as H
    return H


def _check_against_oracle(H, w, hp, Y, counts_used, tiles, R_gpu=None, search_counts=None,
                          search_vs=None, search_rank=None, I=None):
    M, K, T = w.M, w.K, w.T
    I_ref = O.importance(w.W_bits, w.X_bits)
    I_gpu = (hp.I if I is None else I).cpu().numpy()
    np.testing.assert_array_equal(I_gpu.view(np.uint32), I_ref.view(np.uint32))
    del I_gpu
    sr = O.boundary_search(I_ref, w.perm, T, w.t_s, w.alpha, tiles=tiles)
    np.testing.assert_array_equal(search_counts[tiles], sr.counts[tiles])
    np.testing.assert_array_equal(search_rank[tiles], sr.rank[tiles])
    if search_vs is not None:
        np.testing.assert_array_equal(search_vs[tiles], np.asarray(sr.v_s)[tiles])
    if R_gpu is not None:
        for t in tiles:
            np.testing.assert_array_equal(R_gpu[t], np.array(sr.R[t], dtype=np.float64))
    bm_ref, reg_ref = O.mask(I_ref, w.perm, T, counts_used)
    del I_ref
    np.testing.assert_array_equal(hp.bitmask.cpu().numpy().view(np.uint32), bm_ref)
    np.testing.assert_array_equal(hp.region.cpu().numpy(), reg_ref)
    L_ref = O.compress(w.W_bits, bm_ref, reg_ref, w.perm, counts_used, T, tiles=tiles)
    layout_equal(hp.layout, L_ref, tiles=tiles)
    y_ref, bound = O.spmm_reference(w.W_bits, bm_ref, w.X_bits)
    check_y(Y.cpu().numpy(), y_ref, bound)


FULL = [("pure24_4096x4096x2048", hi.pure24, 0.0),
        ("hinm_up_11008x4096x4096", hi.hinm_up_proj, 0.6),
        ("decode_down_4096x11008x16", hi.decode_down_proj, 0.4)]


@pytest.mark.parametrize("name,make,v_s", FULL, ids=[f[0] for f in FULL])
def test_benchmark_workloads_full(H, name, make, v_s):
    """The benchmark's launch configuration (fixed boundary, the tile-pair hint where the
    benchmark passes it); the GPU's own search is checked on three tiles."""
    w = make()
    M, K, N, T = w.M, w.K, w.N, w.T
    nt = M // T
    W, X, perm = dev_bf16(w.W_bits), dev_bf16(w.X_bits), dev_i32(w.perm)
    hp = H.HotPath(M, K, N, T, w.t_s, w.alpha, materialize_importance=False)
    c = np.array(H.hinm_counts_from_vs(K, w.t_s, v_s), dtype=np.int32)
    counts = np.tile(c, (nt, 1))
    Y = hp.run(W, X, perm, fixed_counts=dev_i32(counts),
               tile_pairs=H.tile_pairs_hint(c, w.perm, K))
    I = H.hinm_importance(W, X)        # for the element-wise check of the importance alone
    torch.cuda.synchronize()
    status_ok(H)
    tiles = sorted({0, nt // 2, nt - 1})
    _check_against_oracle(H, w, hp, Y, counts, tiles, search_counts=hp.counts.cpu().numpy(),
                          search_rank=hp.rank.cpu().numpy(), search_vs=hp.vs.cpu().numpy(), I=I)


# Layer 0 of the sweep: the three linear shapes (q/k/v/o 4096x4096, gate/up 11008x4096,
# down 4096x11008) x N in {16, 512, 4096} x t_s in {0.5, 0.625, 0.75}, boundary searched.
SWEEP = [(lin, t_s, N) for lin in ("q", "gate", "down") for t_s in (0.5, 0.625, 0.75)
         for N in (16, 512, 4096)]


@pytest.mark.parametrize("linear,t_s,N", SWEEP, ids=[f"{l}_ts{t}_N{n}" for l, t, n in SWEEP])
def test_llama_sweep_layer0_full(H, linear, t_s, N):
    w = hi.llama_sweep_layer(0, linear, N, t_s)
    M, K, T = w.M, w.K, w.T
    nt = M // T
    W, X, perm = dev_bf16(w.W_bits), dev_bf16(w.X_bits), dev_i32(w.perm)
    hp = H.HotPath(M, K, N, T, w.t_s, w.alpha)
    Y = hp.run(W, X, perm)  # counts from the search
    n_c = H.hinm_search_num_candidates(K, t_s, w.alpha)
    R_gpu = torch.empty((nt, n_c), dtype=torch.float64, device="cuda")
    H.hinm_boundary_search(hp.I, perm, T, t_s, w.alpha, want_rank=False, retained_out=R_gpu)
    # the same pass without materializing I: every result bit for bit
    hq = H.HotPath(M, K, N, T, w.t_s, w.alpha, materialize_importance=False)
    Yq = hq.run(W, X, perm)
    torch.cuda.synchronize()
    status_ok(H)
    for a, b in ((hp.counts, hq.counts), (hp.vs, hq.vs), (hp.rank, hq.rank),
                 (hp.bitmask, hq.bitmask), (hp.region, hq.region),
                 *zip(H.tile_stats_views(hp.stats, M, K, T), H.tile_stats_views(hq.stats, M, K, T))):
        assert torch.equal(a, b)
    assert torch.equal(Y.view(torch.int32), Yq.view(torch.int32))
    del hq, Yq
    counts = hp.counts.cpu().numpy()
    _check_against_oracle(H, w, hp, Y, counts, [0, nt - 1], R_gpu=R_gpu.cpu().numpy(),
                          search_counts=counts, search_vs=hp.vs.cpu().numpy(),
                          search_rank=hp.rank.cpu().numpy())
