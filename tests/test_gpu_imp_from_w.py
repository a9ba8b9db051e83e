"""GPU tests of the search and the mask reading W instead of a materialized importance.

The importance of one weight is fl32(fl32(w^2) * s_c), s_c the channel energy of its input
channel (the FlexHiNM-GP page, 关键设计 1 and 2: second-order weight importance and the
importance matrix).  With
hinm_importance_stats(..., materialize=False) the channel energies stay in the statistics
buffer and no M x K importance is written; the search and the mask recompute every
importance from W (2 bytes per weight) with the same two roundings.  The results must be
the same bits as the materialized path's and the oracle's:

* counts, v_s, rank and every candidate's R(m); the mask bits and the regions; the layout
  bytes and Y (within the product tolerance), on the small parity cases (ragged K, T = 64
  and 128, searched and fixed boundaries, the degenerate t_s = 0 and t_s = 1);
* the same with one working order per tile;
* HotPath(materialize_importance=False) against HotPath(): every buffer and Y bit for bit.
"""
import numpy as np
import pytest

import hinm_inputs as hi
from oracle import hinm_oracle as O

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

from test_gpu_parity import CASES, check_y, dev_bf16, dev_i32, layout_equal, status_ok  # noqa: E402


@pytest.fixture(scope="module")
def H():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import pruning_hinm_spmm_b200 as H
    return H


def _w_path(H, w, perm_np, v_s):
    """importance statistics without I, then search / mask / compress / spmm from W."""
    M, K, N, T = w.M, w.K, w.N, w.T
    nt = M // T
    W, X, perm = dev_bf16(w.W_bits), dev_bf16(w.X_bits), dev_i32(perm_np)
    I_none, stats = H.hinm_importance_stats(W, X, T, materialize=False)
    assert I_none is None
    nc = H.hinm_search_num_candidates(K, w.t_s, w.alpha)
    R = torch.empty((nt, nc), dtype=torch.float64, device="cuda")
    cnt, vs, rank = H.hinm_boundary_search(None, perm, T, w.t_s, w.alpha, retained_out=R,
                                           stats=stats, W=W)
    if v_s is None:
        use = cnt
    else:
        use = dev_i32(np.tile(np.array(H.hinm_counts_from_vs(K, w.t_s, v_s), dtype=np.int32),
                              (nt, 1)))
    bm, region = H.hinm_mask(None, perm, use, T, rank if v_s is None else None, W=W,
                             stats=stats)
    L = H.hinm_compress(W, bm, region, perm, use, T)
    Y = H.hinm_spmm(L, X)
    torch.cuda.synchronize()
    status_ok(H)
    return dict(counts=cnt.cpu().numpy(), vs=vs.cpu().numpy(), rank=rank.cpu().numpy(),
                R=R.cpu().numpy(), used=use.cpu().numpy(),
                bitmask=bm.cpu().numpy().view(np.uint32), region=region.cpu().numpy(), L=L,
                Y=Y.cpu().numpy(), stats=stats, W=W, X=X)


def _against_oracle(w, perm_np, g):
    I_ref = O.importance(w.W_bits, w.X_bits)
    sr = O.boundary_search(I_ref, perm_np, w.T, w.t_s, w.alpha)
    np.testing.assert_array_equal(g["counts"], sr.counts)
    np.testing.assert_array_equal(g["vs"], np.asarray(sr.v_s))
    np.testing.assert_array_equal(g["rank"], sr.rank)
    np.testing.assert_array_equal(g["R"], np.array(sr.R))
    bm_ref, reg_ref = O.mask(I_ref, perm_np, w.T, g["used"])
    np.testing.assert_array_equal(g["region"], reg_ref)
    np.testing.assert_array_equal(g["bitmask"], bm_ref)
    layout_equal(g["L"], O.compress(w.W_bits, bm_ref, reg_ref, perm_np, g["used"], w.T))
    y_ref, bound = O.spmm_reference(w.W_bits, bm_ref, w.X_bits)
    check_y(g["Y"], y_ref, bound)


@pytest.mark.parametrize("searched", [True, False], ids=["searched", "fixed"])
@pytest.mark.parametrize("name,make,v_s", CASES, ids=[c[0] for c in CASES])
def test_w_path_matches_oracle(H, name, make, v_s, searched):
    w = make()
    g = _w_path(H, w, w.perm, None if searched else v_s)
    _against_oracle(w, w.perm, g)
    # the statistics written without I equal those written with it
    I, stats = H.hinm_importance_stats(g["W"], g["X"], w.T)
    torch.cuda.synchronize()
    for a, b in zip(H.tile_stats_views(stats, w.M, w.K, w.T),
                    H.tile_stats_views(g["stats"], w.M, w.K, w.T)):
        assert torch.equal(a, b)


@pytest.mark.parametrize("M,K,N,T,t_s,seed", [(512, 256, 24, 128, 0.625, 1),
                                              (384, 640, 72, 64, 0.75, 2),
                                              (256, 200, 16, 64, 0.5, 3)])
def test_w_path_per_tile_orders(H, M, K, N, T, t_s, seed):
    w = hi.custom(M, K, N, T, seed=seed, t_s=t_s, v_s=None)
    rng = np.random.default_rng(seed + 200)
    perm_tiles = np.stack([rng.permutation(K) for _ in range(M // T)]).astype(np.int32)
    g = _w_path(H, w, perm_tiles, None)
    _against_oracle(w, perm_tiles, g)


@pytest.mark.parametrize("name,make,v_s", CASES[2:5], ids=[c[0] for c in CASES[2:5]])
def test_hot_path_without_materialized_importance(H, name, make, v_s):
    w = make()
    M, K, N, T = w.M, w.K, w.N, w.T
    W, X, perm = dev_bf16(w.W_bits), dev_bf16(w.X_bits), dev_i32(w.perm)
    fixed = dev_i32(np.tile(np.array(H.hinm_counts_from_vs(K, w.t_s, v_s), dtype=np.int32),
                            (M // T, 1)))
    for counts in (None, fixed):
        a = H.HotPath(M, K, N, T, w.t_s, w.alpha)
        b = H.HotPath(M, K, N, T, w.t_s, w.alpha, materialize_importance=False)
        assert b.I is None
        Ya = a.run(W, X, perm, fixed_counts=counts)
        Yb = b.run(W, X, perm, fixed_counts=counts)
        torch.cuda.synchronize()
        status_ok(H)
        for x, y in ((a.counts, b.counts), (a.vs, b.vs), (a.rank, b.rank),
                     (a.bitmask, b.bitmask), (a.region, b.region)):
            assert torch.equal(x, y)
        assert torch.equal(Ya.view(torch.int32), Yb.view(torch.int32))
        _same_used_blocks(a.layout, b.layout)


def _same_used_blocks(La, Lb):
    """Two layouts hold the same bytes in every block their tiles use (blocks past the
    last tile's are never written)."""
    assert torch.equal(La.tile_info, Lb.tile_info)
    info = La.tile_info.cpu().numpy()
    nd_used = int((info[:, 2] + info[:, 0]).max(initial=0))
    ns_used = int((info[:, 3] + info[:, 1]).max(initial=0))
    for f, n in (("vals_dense", nd_used), ("idx_dense", nd_used), ("run_dense", nd_used),
                 ("vals_sparse", ns_used), ("meta", ns_used), ("idx_sparse", ns_used),
                 ("run_sparse", ns_used)):
        assert torch.equal(getattr(La, f)[:n], getattr(Lb, f)[:n]), f


def test_w_path_extreme_dynamic_range(H):
    """Importances spanning more than 2^100 within a tile (weights near 1e-20): the values
    below the column sums' two fp64 levels and below band_sum's fast path take the exact
    128-bit and exponent-bucket paths, recomputed from W, and every R(m), the counts, the
    ranks and the mask still match the oracle bit for bit."""
    rng = np.random.default_rng(5)
    M, K, N, T = 256, 256, 16, 128
    scale = np.where(rng.random(K) < 0.3, 1e-20, 1.0).astype(np.float32)
    Wf = (rng.standard_normal((M, K)).astype(np.float32) * scale[None, :])
    Wf[:, :8] *= np.float32(1e-19)  # a few columns entirely in the tiny range
    Wf[::7, 8:40] *= np.float32(1e-15)  # scattered values below the tile's window
    Wf[::5, 40:72] *= np.float32(1e-9)  # and some 2^50-2^80 below the largest: 128-bit path
    w = hi.Workload(name="extreme_w", M=M, K=K, N=N, T=T, W_bits=hi.f32_to_bf16_bits(Wf),
                    X_bits=hi.f32_to_bf16_bits(rng.standard_normal((K, N)).astype(np.float32)),
                    perm=rng.permutation(K).astype(np.int32), t_s=0.5, v_s=None)
    I_ref = O.importance(w.W_bits, w.X_bits)
    nz = I_ref[I_ref > 0].astype(np.float64)
    assert np.log2(nz.max() / nz.min()) > 100   # really exercises the slow paths
    g = _w_path(H, w, w.perm, None)
    _against_oracle(w, w.perm, g)
