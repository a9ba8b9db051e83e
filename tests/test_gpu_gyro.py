"""GPU tests of the gyro-permutation and of per-tile working orders, against the CPU oracle.

* Per-tile working orders (perm [M/T, K]) through the search, the mask, compress and the
  SpMM: counts, ranks, R(m), masks, regions and layout bytes bit for bit, Y within the
  product tolerance.
* The input rounds' cost matrices of every tile on the GPU, bit for bit against the oracle.
* The whole flow for M/T > 1: search, refine every tile's 2:4 band with the library's
  in-tile rounds, rebuild the per-tile orders, run the path again with them: parity with
  the oracle, and every tile's 2:4 pruning cost no higher than before.
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


def _path(H, w, perm_tiles, counts=None):
    M, K, T = w.M, w.K, w.T
    W, X = dev_bf16(w.W_bits), dev_bf16(w.X_bits)
    P = dev_i32(perm_tiles)
    I = H.hinm_importance(W, X)
    nc = H.hinm_search_num_candidates(K, w.t_s, w.alpha)
    R = torch.empty((M // T, nc), dtype=torch.float64, device="cuda")
    cnt, vs, rank = H.hinm_boundary_search(I, P, T, w.t_s, w.alpha, retained_out=R)
    use = dev_i32(counts) if counts is not None else cnt
    bm, region = H.hinm_mask(I, P, use, T, rank if counts is None else None)
    L = H.hinm_compress(W, bm, region, P, use, T)
    Y = H.hinm_spmm(L, X)
    torch.cuda.synchronize()
    status_ok(H)
    return dict(I=I.cpu().numpy(), counts=cnt.cpu().numpy(), vs=vs.cpu().numpy(),
                rank=rank.cpu().numpy(), R=R.cpu().numpy(), used=use.cpu().numpy(),
                bitmask=bm.cpu().numpy().view(np.uint32), region=region.cpu().numpy(), L=L,
                Y=Y.cpu().numpy())


@pytest.mark.parametrize("M,K,N,T,t_s,seed", [(512, 256, 24, 128, 0.625, 1),
                                              (384, 640, 72, 64, 0.75, 2),
                                              (256, 200, 16, 64, 0.5, 3)])
def test_per_tile_orders_match_oracle(H, M, K, N, T, t_s, seed):
    w = hi.custom(M, K, N, T, seed=seed, t_s=t_s, v_s=None)
    rng = np.random.default_rng(seed + 100)
    perm_tiles = np.stack([rng.permutation(K) for _ in range(M // T)]).astype(np.int32)
    g = _path(H, w, perm_tiles)
    I_ref = O.importance(w.W_bits, w.X_bits)
    np.testing.assert_array_equal(g["I"].view(np.uint32), I_ref.view(np.uint32))
    sr = O.boundary_search(I_ref, perm_tiles, T, t_s, w.alpha)
    np.testing.assert_array_equal(g["counts"], sr.counts)
    np.testing.assert_array_equal(g["vs"], sr.v_s)
    np.testing.assert_array_equal(g["rank"], sr.rank)
    np.testing.assert_array_equal(g["R"], np.array(sr.R))
    bm_ref, reg_ref = O.mask(I_ref, perm_tiles, T, sr.counts)
    np.testing.assert_array_equal(g["region"], reg_ref)
    np.testing.assert_array_equal(g["bitmask"], bm_ref)
    L_ref = O.compress(w.W_bits, bm_ref, reg_ref, perm_tiles, sr.counts, T)
    layout_equal(g["L"], L_ref)
    y_ref, bound = O.spmm_reference(w.W_bits, bm_ref, w.X_bits)
    check_y(g["Y"], y_ref, bound)
    # one shared order given as identical rows equals the shared-order call
    shared = np.tile(perm_tiles[0], (M // T, 1))
    g2 = _path(H, w, shared)
    g1 = _path(H, w, perm_tiles[0])
    np.testing.assert_array_equal(g2["bitmask"], g1["bitmask"])
    np.testing.assert_array_equal(g2["Y"].view(np.uint32), g1["Y"].view(np.uint32))


def test_per_tile_order_bad_row_reported(H):
    w = hi.custom(256, 128, 16, 64, seed=5, t_s=0.5, v_s=0.25)
    W, X = dev_bf16(w.W_bits), dev_bf16(w.X_bits)
    I = H.hinm_importance(W, X)
    c = dev_i32(np.array([H.hinm_counts_from_vs(w.K, w.t_s, w.v_s)] * 4, dtype=np.int32))
    good = np.tile(np.arange(w.K, dtype=np.int32), (4, 1))
    H.hinm_mask(I, dev_i32(good), c, w.T)
    torch.cuda.synchronize()
    assert H.hinm_device_status() == 0
    bad = good.copy()
    bad[3, 7] = bad[3, 9]          # tile 3 repeats a channel
    H.hinm_mask(I, dev_i32(bad), c, w.T)
    torch.cuda.synchronize()
    assert H.hinm_device_status() == H.HINM_ERR_INVALID_ARG
    assert H.hinm_device_status() == 0


def test_gyro_cost_matrix_matches_oracle(H):
    """The input rounds' G x G cost matrices of all tiles in one launch, bit for bit."""
    rng = np.random.default_rng(7)
    M, K, T, nb, G, k = 512, 384, 128, 256, 12, 2
    nt = M // T
    I = rng.exponential(1.0, (M, K)).astype(np.float32)
    bands = np.stack([rng.permutation(K)[:nb] for _ in range(nt)]).astype(np.int32)
    groups = np.stack([rng.choice(nb // 4, G, replace=False) for _ in range(nt)]).astype(np.int32)
    slots = np.stack([np.stack([rng.choice(4, k, replace=False) for _ in range(G)])
                      for _ in range(nt)]).astype(np.int32)
    clusters = []
    for t in range(nt):
        vecs = [int(bands[t][4 * g + s]) for g, ss in zip(groups[t], slots[t]) for s in ss]
        F = I[t * T:(t + 1) * T][:, vecs].T.astype(np.float64)
        clusters.append(O.balanced_kmeans(F, k, 8))
    clusters = np.array(clusters, dtype=np.int32)
    got = H.hinm_gyro_cost_matrix(torch.from_numpy(I).cuda(), T, dev_i32(bands), dev_i32(groups),
                                  dev_i32(slots), dev_i32(clusters))
    torch.cuda.synchronize()
    status_ok(H)
    got = got.cpu().numpy()
    for t in range(nt):
        want = O.gyro_input_cost_matrix(I[t * T:(t + 1) * T], bands[t], groups[t], slots[t],
                                        [list(c) for c in clusters[t]])
        np.testing.assert_array_equal(got[t], want)


def test_gyro_refined_orders_flow_through_the_path(H):
    """M/T = 4 tiles with fixed counts: refine each tile's 2:4 band with three in-tile rounds
    (the library's host code), rebuild the per-tile working orders, run the whole path with
    them on the GPU: every result equals the oracle's with the same orders, every tile's
    groups are the refined band, and no tile's 2:4 pruning cost rose."""
    M, K, N, T = 512, 256, 32, 128
    w = hi.custom(M, K, N, T, seed=12, t_s=0.625, v_s=0.4, random_perm=True)
    nt = M // T
    counts = np.tile(np.array(H.hinm_counts_from_vs(K, w.t_s, w.v_s), dtype=np.int32), (nt, 1))
    base = _path(H, w, np.tile(w.perm, (nt, 1)), counts)
    I_ref = O.importance(w.W_bits, w.X_bits)
    rng = np.random.default_rng(3)
    bands, before, after = [], [], []
    for t in range(nt):
        pt = w.perm
        band = np.array([c for c in pt if base["region"][t][c] == O.REGION_24], dtype=np.int32)
        I_tile = I_ref[t * T:(t + 1) * T]
        before.append(O.band_pruning_cost(I_tile, band))
        for _ in range(3):
            groups = rng.choice(band.size // 4, 8, replace=False).astype(np.int32)
            slots = np.stack([rng.choice(4, 2, replace=False) for _ in range(8)]).astype(np.int32)
            band, _ = H.hinm_gyro_input_round_host(I_tile, band, groups, slots)
        after.append(O.band_pruning_cost(I_tile, band))
        bands.append(band)
    assert all(a <= b for a, b in zip(after, before))
    assert sum(after) < sum(before)                    # the rounds found something
    orders = H.tile_orders_with_bands(w.perm, base["region"], bands)
    g = _path(H, w, orders, counts)
    bm_ref, reg_ref = O.mask(I_ref, orders, T, counts)
    np.testing.assert_array_equal(g["region"], reg_ref)
    np.testing.assert_array_equal(g["region"], base["region"])   # regions do not move
    np.testing.assert_array_equal(g["bitmask"], bm_ref)
    L_ref = O.compress(w.W_bits, bm_ref, reg_ref, orders, counts, T)
    layout_equal(g["L"], L_ref)
    y_ref, bound = O.spmm_reference(w.W_bits, bm_ref, w.X_bits)
    check_y(g["Y"], y_ref, bound)
    # the 2:4 pruning cost of each tile under the new mask is the refined band's
    for t in range(nt):
        keep = O.unpack_bits(g["bitmask"][t * T:(t + 1) * T], K)
        I_tile = I_ref[t * T:(t + 1) * T].astype(np.float64)
        in_band = reg_ref[t] == O.REGION_24
        pruned = float(I_tile[:, in_band][~keep[:, in_band]].sum())
        assert abs(pruned - after[t]) <= 1e-9 * max(after[t], 1.0)
