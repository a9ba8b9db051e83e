"""Host-only checks of the C ABI: the library loads without a GPU, exports every entry
point include/hinm.h declares, computes the closed-form counts and layout sizes the
oracle predicts, and rejects bad arguments before launching anything."""
import ctypes
import os
import re

import numpy as np
import pytest

from oracle import hinm_oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def H():
    from conftest import build_library
    build_library()
    import pruning_hinm_spmm_b200 as H
    return H


def declared_functions():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"\b(hinm_\w+)\s*\(", src))
    return names


def test_exports_every_declared_symbol(H):
    names = declared_functions()
    assert {"hinm_importance", "hinm_boundary_search", "hinm_mask", "hinm_compress",
            "hinm_spmm"} <= names
    lib = ctypes.CDLL(H.LIB_PATH)
    for n in sorted(names):
        assert hasattr(lib, n), f"{n} declared in include/ but not exported"


def test_every_export_is_declared(H):
    """The other direction: every hinm_ function the library exports is declared (and so
    documented) in include/ -- no undocumented entry points."""
    import shutil
    import subprocess
    if not shutil.which("nm"):
        pytest.skip("nm not available")
    out = subprocess.run(["nm", "-D", "--defined-only", H.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = {ln.split()[-1] for ln in out.splitlines()
                if len(ln.split()) >= 3 and ln.split()[1] == "T" and ln.split()[-1].startswith("hinm_")}
    assert exported, "no hinm_ exports found"
    assert exported <= declared_functions(), sorted(exported - declared_functions())


def test_versions_and_strings(H):
    lib = H.lib()
    assert lib.hinm_abi_version() == 1
    assert lib.hinm_status_string(0) == b"HINM_OK"
    assert lib.hinm_status_string(7) == b"HINM_ERR_BAD_MASK"


@pytest.mark.parametrize("K", [64, 100, 200, 256, 4096, 11008])
@pytest.mark.parametrize("t_s", [0.0, 0.5, 0.625, 0.75, 1.0])
def test_counts_match_oracle(H, K, t_s):
    for m in range(0, 40):
        v_s = t_s - m / 32
        if v_s < 0:
            break
        try:
            want = O.counts_from_vs(K, t_s, v_s)
        except ValueError:
            with pytest.raises(H.HinmError):
                H.hinm_counts_from_vs(K, t_s, v_s)
            continue
        assert H.hinm_counts_from_vs(K, t_s, v_s) == want


def test_compress_size_matches_oracle(H):
    for K, t_s, v_s in [(256, 0.5, 0.2), (4096, 0.75, 0.6), (11008, 0.625, 0.4), (4096, 0.5, 0.0)]:
        c = np.array(O.counts_from_vs(K, t_s, v_s), dtype=np.int32)
        counts = np.tile(c, (4, 1))
        sz = H.hinm_compress_size(512, K, 128, counts)
        info = O.tile_blocks(counts)
        assert sz.max_dense_blocks == max(1, info[:, 0].sum())
        assert sz.max_sparse_blocks == max(1, info[:, 1].sum())
        worst = H.hinm_compress_size(512, K, 128, None)
        assert worst.max_dense_blocks >= sz.max_dense_blocks
        assert worst.max_sparse_blocks >= sz.max_sparse_blocks
        assert worst.vals_dense_bytes == worst.max_dense_blocks * 16384


def test_validation_rejects_before_launch(H):
    lib = H.lib()
    fake = 0x10000  # never dereferenced: every call below fails its host checks first
    ws = ctypes.c_size_t(0)
    # bad tile height / shapes
    assert lib.hinm_search_workspace_size(256, 256, 32, 0.5, 1 / 32, ctypes.byref(ws)) == H.HINM_ERR_SHAPE
    assert lib.hinm_search_workspace_size(200, 256, 64, 0.5, 1 / 32, ctypes.byref(ws)) == H.HINM_ERR_SHAPE
    assert lib.hinm_search_workspace_size(256, 258, 64, 0.5, 1 / 32, ctypes.byref(ws)) == H.HINM_ERR_SHAPE
    assert lib.hinm_search_workspace_size(256, 256, 64, 1.5, 1 / 32, ctypes.byref(ws)) == H.HINM_ERR_INVALID_ARG
    assert lib.hinm_search_workspace_size(256, 256, 64, 0.5, 0.0, ctypes.byref(ws)) == H.HINM_ERR_INVALID_ARG
    assert lib.hinm_search_workspace_size(256, 256, 64, 0.5, 1 / 32, ctypes.byref(ws)) == H.HINM_OK
    assert ws.value > 0
    # null / misaligned pointers
    assert lib.hinm_importance(None, fake, 64, 64, 16, fake, fake, 1 << 20, None) == H.HINM_ERR_INVALID_ARG
    assert lib.hinm_importance(fake + 2, fake, 64, 64, 16, fake, fake, 1 << 20, None) == H.HINM_ERR_ALIGNMENT
    assert lib.hinm_importance(fake, fake, 64, 64, 12, fake, fake, 1 << 20, None) == H.HINM_ERR_SHAPE
    assert lib.hinm_importance(fake, fake, 64, 64, 16, fake, fake, 0, None) == H.HINM_ERR_WORKSPACE
    assert b"workspace" in lib.hinm_last_error()
    # workspace too small for the search
    cnt = ctypes.c_void_p(fake)
    assert lib.hinm_boundary_search(fake, None, 256, 256, 64, 0.5, 1 / 32, fake, fake, None, None,
                                    fake, 16, None) == H.HINM_ERR_WORKSPACE
    # t_s * K not whole
    assert lib.hinm_boundary_search(fake, None, 256, 100, 64, 0.333, 1 / 32, fake, fake, None, None,
                                    fake, 1 << 30, None) == H.HINM_ERR_INVALID_ARG
    n = ctypes.c_int32(0)
    assert lib.hinm_search_num_candidates(4096, 0.75, 1 / 32, ctypes.byref(n)) == H.HINM_OK
    assert n.value == len(O.search_candidates(4096, 0.75, 1 / 32))
    # layout checks
    L = H.hinm_layout(H.HINM_LAYOUT_VERSION + 1, 256, 256, 64, 4, 1, 1, fake, fake, fake, fake, fake, fake, fake, fake)
    assert lib.hinm_spmm(ctypes.byref(L), fake, 16, fake, None) == H.HINM_ERR_INVALID_ARG
    L = H.hinm_layout(H.HINM_LAYOUT_VERSION, 256, 256, 64, 3, 1, 1, fake, fake, fake, fake, fake, fake, fake, fake)
    assert lib.hinm_spmm(ctypes.byref(L), fake, 16, fake, None) == H.HINM_ERR_SHAPE
    L = H.hinm_layout(H.HINM_LAYOUT_VERSION, 256, 256, 64, 4, 1, 1, fake, fake, fake, fake, fake, fake, fake, fake)
    assert lib.hinm_spmm(ctypes.byref(L), fake, 20, fake, None) == H.HINM_ERR_SHAPE
    assert lib.hinm_spmm(ctypes.byref(L), fake + 8, 16, fake, None) == H.HINM_ERR_ALIGNMENT
    # the fused importance statistics: T checked, stats buffer required and large enough
    sz = ctypes.c_size_t(0)
    assert lib.hinm_tile_stats_size(256, 256, 96, ctypes.byref(sz)) == H.HINM_ERR_SHAPE
    assert lib.hinm_tile_stats_size(256, 256, 128, ctypes.byref(sz)) == H.HINM_OK
    assert sz.value >= 2 * 256 * 8 + 2 * 4
    assert lib.hinm_importance_stats(fake, fake, 256, 256, 16, 128, fake, None, sz.value, fake,
                                     1 << 20, None) == H.HINM_ERR_INVALID_ARG
    assert lib.hinm_importance_stats(fake, fake, 256, 256, 16, 128, fake, fake, sz.value - 1,
                                     fake, 1 << 20, None) == H.HINM_ERR_INVALID_ARG
    assert lib.hinm_importance_stats(fake, fake, 256, 256, 16, 96, fake, fake, sz.value, fake,
                                     1 << 20, None) == H.HINM_ERR_SHAPE
    assert lib.hinm_boundary_search_stats(fake, None, sz.value, None, 256, 256, 128, 0.5,
                                          1 / 32, fake, fake, None, None, fake, 1 << 30,
                                          None) == H.HINM_ERR_INVALID_ARG
    assert lib.hinm_boundary_search_stats(fake, fake, 8, None, 256, 256, 128, 0.5, 1 / 32, fake,
                                          fake, None, None, fake, 1 << 30,
                                          None) == H.HINM_ERR_INVALID_ARG
    # importance recomputed from W: without I, both W and stats are needed, stats must be
    # large enough, W aligned
    def search_ex(I, W, st, st_bytes):
        return lib.hinm_boundary_search_ex(I, W, st, st_bytes, None, 0, 256, 256, 128, 0.5,
                                           1 / 32, fake, fake, None, None, fake, 1 << 30, None)
    assert search_ex(None, None, fake, sz.value) == H.HINM_ERR_INVALID_ARG
    assert search_ex(None, fake, None, sz.value) == H.HINM_ERR_INVALID_ARG
    assert search_ex(None, fake, fake, sz.value - 1) == H.HINM_ERR_INVALID_ARG
    assert search_ex(None, fake + 2, fake, sz.value) == H.HINM_ERR_ALIGNMENT

    def mask_ex(I, W, st, st_bytes, per_tile=0):
        return lib.hinm_mask_ex(I, W, st, st_bytes, None, per_tile, fake, None, 256, 256, 128,
                                fake, fake, fake, 1 << 30, None)
    assert mask_ex(None, None, fake, sz.value) == H.HINM_ERR_INVALID_ARG
    assert mask_ex(None, fake, None, sz.value) == H.HINM_ERR_INVALID_ARG
    assert mask_ex(None, fake, fake, sz.value - 1) == H.HINM_ERR_INVALID_ARG
    assert mask_ex(None, fake + 2, fake, sz.value) == H.HINM_ERR_ALIGNMENT
    assert mask_ex(fake, None, None, 0, per_tile=2) == H.HINM_ERR_INVALID_ARG
    # the fused epilogue: an unknown activation is refused; the flags are checked first
    assert lib.hinm_spmm_epilogue(ctypes.byref(L), fake, 16, fake, None, 4, 0, 0,
                                  None) == H.HINM_ERR_INVALID_ARG
    assert lib.hinm_spmm_epilogue(ctypes.byref(L), fake, 16, fake, None, 1, 1, 8,
                                  None) == H.HINM_ERR_INVALID_ARG
    assert lib.hinm_spmm_epilogue(ctypes.byref(L), fake, 16, fake, fake + 4, 1, 0, 0,
                                  None) == H.HINM_ERR_ALIGNMENT
    # Hard-Concrete: n a positive multiple of 4, tau positive and finite, pointers aligned
    assert lib.hinm_hard_concrete_forward(fake, fake, ctypes.c_longlong(6), ctypes.c_float(0.5),
                                          fake, None, None, None) == H.HINM_ERR_SHAPE
    assert lib.hinm_hard_concrete_forward(fake, fake, ctypes.c_longlong(8), ctypes.c_float(0.0),
                                          fake, None, None, None) == H.HINM_ERR_INVALID_ARG
    assert lib.hinm_hard_concrete_forward(fake, fake, ctypes.c_longlong(8),
                                          ctypes.c_float(float("inf")), fake, None, None,
                                          None) == H.HINM_ERR_INVALID_ARG
    assert lib.hinm_hard_concrete_forward(fake + 4, fake, ctypes.c_longlong(8), ctypes.c_float(0.5),
                                          fake, None, None, None) == H.HINM_ERR_ALIGNMENT
    # index translation: a NULL map is refused, and so is a layout of another version
    assert lib.hinm_translate_index(ctypes.byref(L), None, None) == H.HINM_ERR_INVALID_ARG
    Lbad = H.hinm_layout(H.HINM_LAYOUT_VERSION + 1, 256, 256, 64, 4, 1, 1, fake, fake, fake, fake,
                         fake, fake, fake, fake)
    assert lib.hinm_translate_index(ctypes.byref(Lbad), fake, None) == H.HINM_ERR_INVALID_ARG
    # hinm_spmm_ex: unknown flag bits are refused before anything else; the hint flag
    # passes the same argument checks as hinm_spmm
    assert lib.hinm_spmm_ex(ctypes.byref(L), fake, 16, fake, 2, None) == H.HINM_ERR_INVALID_ARG
    assert lib.hinm_spmm_ex(ctypes.byref(L), fake, 20, fake, H.HINM_SPMM_TILE_PAIRS,
                            None) == H.HINM_ERR_SHAPE
    assert lib.hinm_spmm_ex(ctypes.byref(L), fake + 8, 16, fake, H.HINM_SPMM_TILE_PAIRS,
                            None) == H.HINM_ERR_ALIGNMENT
    # compress size rejects inconsistent counts
    bad = (ctypes.c_int32 * 3)(10, 11, 235)
    out = H.hinm_layout_sizes()
    assert lib.hinm_compress_size(bad, 64, 256, 64, ctypes.byref(out)) == H.HINM_ERR_INVALID_ARG


def test_tile_pairs_hint_rule():
    """The host rule behind the SpMM's tile-pair hint: one shared single region (all 2:4 or
    all dense) in every tile and an ascending permutation; anything else gives no hint."""
    import numpy as np
    import pruning_hinm_spmm_b200 as H
    K = 256
    assert H.tile_pairs_hint([0, K, 0], None, K)                       # all 2:4
    assert H.tile_pairs_hint([[0, 0, K]] * 4, np.arange(K), K)         # all dense
    assert not H.tile_pairs_hint([64, 128, 64], None, K)               # HiNM regions
    assert not H.tile_pairs_hint([0, K, 0], np.arange(K)[::-1], K)     # permuted X rows
    assert not H.tile_pairs_hint([[0, K, 0], [0, 0, K]], None, K)      # tiles differ
    assert H.tile_pairs_hint(H.hinm_counts_from_vs(K, 0.5, 0.0), None, K)
    assert not H.tile_pairs_hint(H.hinm_counts_from_vs(K, 0.5, 0.25), None, K)


@pytest.mark.parametrize("T,K,n,G,k,seed", [(8, 64, 48, 4, 2, 1), (128, 1024, 512, 16, 2, 2),
                                            (32, 256, 128, 8, 1, 3), (64, 512, 256, 12, 3, 4),
                                            (16, 128, 96, 6, 4, 5)])
def test_gyro_input_round_host_matches_oracle(T, K, n, G, k, seed):
    """The native in-tile round (host code of the library) against the oracle, bit for bit:
    the refined band and both costs, over three chained rounds with fresh draws."""
    import pruning_hinm_spmm_b200 as H
    rng = np.random.default_rng(seed)
    I_tile = rng.exponential(1.0, (T, K)).astype(np.float32)
    band = rng.permutation(K)[:n].astype(np.int32)
    got, want = band.copy(), band.copy()
    for _ in range(3):
        groups = rng.choice(n // 4, G, replace=False).astype(np.int32)
        slots = np.stack([rng.choice(4, k, replace=False) for _ in range(G)]).astype(np.int32)
        got, gc = H.hinm_gyro_input_round_host(I_tile, got, groups, slots)
        want, wc = O.gyro_input_round(I_tile, want, groups, slots)
        np.testing.assert_array_equal(got, want)
        assert gc == wc
    assert H.hinm_gyro_band_cost_host(I_tile, got) == O.band_pruning_cost(I_tile, got)


@pytest.mark.parametrize("T,K,nt,G,k,seed", [(4, 16, 5, 3, 1, 1), (16, 64, 6, 4, 2, 2),
                                             (8, 256, 10, 5, 3, 3)])
def test_gyro_output_round_host_matches_oracle(T, K, nt, G, k, seed):
    """The native output-channel round against the oracle, bit for bit, over two rounds."""
    import pruning_hinm_spmm_b200 as H
    rng = np.random.default_rng(seed)
    I = rng.exponential(1.0, (nt * T, K)).astype(np.float32)
    n0 = rng.integers(0, K // 2, nt).astype(np.int32)
    order = rng.permutation(nt * T).astype(np.int32)
    got, want = order.copy(), order.copy()
    for _ in range(2):
        tiles = rng.choice(nt, G, replace=False).astype(np.int32)
        rows = np.stack([rng.choice(T, k, replace=False) for _ in range(G)]).astype(np.int32)
        got, gc = H.hinm_gyro_output_round_host(I, T, n0, got, tiles, rows)
        want, wc = O.gyro_output_round(I, T, n0, want, tiles, rows)
        np.testing.assert_array_equal(got, want)
        assert gc == wc


def test_gyro_host_validation():
    import pruning_hinm_spmm_b200 as H
    I_tile = np.ones((4, 16), dtype=np.float32)
    band = np.arange(8, dtype=np.int32)
    g1, s1 = np.array([0], dtype=np.int32), np.array([[1]], dtype=np.int32)
    with pytest.raises(H.HinmError):      # band length not a multiple of 4
        H.hinm_gyro_input_round_host(I_tile, band[:6], g1, s1)
    with pytest.raises(H.HinmError):      # repeated group
        H.hinm_gyro_input_round_host(I_tile, band, np.array([0, 0], dtype=np.int32),
                                     np.array([[1], [2]], dtype=np.int32))
    with pytest.raises(H.HinmError):      # slot outside [0, 4)
        H.hinm_gyro_input_round_host(I_tile, band, g1, np.array([[4]], dtype=np.int32))
    with pytest.raises(H.HinmError):      # repeated slot within a group
        H.hinm_gyro_input_round_host(I_tile, band, g1, np.array([[1, 1]], dtype=np.int32))
    bad = band.copy()
    bad[3] = 16
    with pytest.raises(H.HinmError):      # channel outside [0, K)
        H.hinm_gyro_input_round_host(I_tile, bad, g1, s1)
    bad[3] = 0
    with pytest.raises(H.HinmError):      # repeated channel
        H.hinm_gyro_input_round_host(I_tile, bad, g1, s1)
    inf = I_tile.copy()
    inf[2, 5] = np.inf                    # a non-finite importance the round reads
    with pytest.raises(H.HinmError):
        H.hinm_gyro_input_round_host(inf, band, g1, s1)
    nan = I_tile.copy()
    nan[1, 0] = np.nan
    with pytest.raises(H.HinmError):
        H.hinm_gyro_input_round_host(nan, band, g1, s1)
    I = np.ones((8, 16), dtype=np.float32)
    with pytest.raises(H.HinmError):      # row order not a permutation
        H.hinm_gyro_output_round_host(I, 4, [1, 1], [0, 1, 2, 3, 4, 5, 6, 6], [0], [[0]])
    with pytest.raises(H.HinmError):      # n0 > K
        H.hinm_gyro_output_round_host(I, 4, [1, 17], np.arange(8), [0], [[0]])
    I[5, 3] = np.nan
    with pytest.raises(H.HinmError):      # non-finite in a sampled tile
        H.hinm_gyro_output_round_host(I, 4, [1, 1], np.arange(8), [1], [[0]])


@pytest.mark.parametrize("shared", [True, False], ids=["shared_order", "per_tile_orders"])
def test_tile_orders_with_bands_matches_oracle(H, shared):
    """The binding's per-tile working orders after refined 2:4 bands equal the oracle's
    tile_perm_with_band tile by tile: each row stays a permutation, the positions of
    dense and pruned channels keep them, and the 2:4 positions hold the band in order."""
    rng = np.random.default_rng(41)
    nt, K = 5, 96
    region = rng.choice([O.REGION_PRUNED, O.REGION_24, O.REGION_DENSE], size=(nt, K),
                        p=[0.3, 0.5, 0.2]).astype(np.int8)
    perm = (rng.permutation(K).astype(np.int32) if shared else
            np.stack([rng.permutation(K) for _ in range(nt)]).astype(np.int32))
    bands = []
    for t in range(nt):
        pt = perm if shared else perm[t]
        members = [int(c) for c in pt if region[t][c] == O.REGION_24]
        bands.append(rng.permutation(np.array(members, dtype=np.int32)))
    got = H.tile_orders_with_bands(perm, region, bands)
    assert got.shape == (nt, K) and got.dtype == np.int32
    for t in range(nt):
        pt = perm if shared else perm[t]
        want = O.tile_perm_with_band(pt, region[t], bands[t])
        np.testing.assert_array_equal(got[t], want)
        assert sorted(got[t].tolist()) == list(range(K))
        keep = region[t][pt] != O.REGION_24
        np.testing.assert_array_equal(got[t][keep], pt[keep])
        np.testing.assert_array_equal(got[t][~keep], bands[t])


def test_empty_inputs_are_refused_before_launch(H):
    """Empty problems (no rows, no channels, no columns) are shape errors reported on the
    host: nothing is launched and no pointer is read."""
    lib = H.lib()
    fake = 0x10000
    for M, K, N in [(0, 64, 16), (64, 0, 16), (64, 64, 0)]:
        assert lib.hinm_importance(fake, fake, M, K, N, fake, fake, 1 << 20,
                                   None) == H.HINM_ERR_SHAPE, (M, K, N)
    for M, K in [(0, 64), (128, 0)]:
        assert lib.hinm_boundary_search(fake, None, M, K, 64, 0.5, 1 / 32, fake, fake, None,
                                        None, fake, 1 << 30, None) == H.HINM_ERR_SHAPE, (M, K)
        assert lib.hinm_mask(fake, None, fake, None, M, K, 64, fake, fake, fake, 1 << 30,
                             None) == H.HINM_ERR_SHAPE, (M, K)
    ws = ctypes.c_size_t(0)
    assert lib.hinm_search_workspace_size(0, 64, 64, 0.5, 1 / 32, ctypes.byref(ws)) == H.HINM_ERR_SHAPE
    L = H.hinm_layout(H.HINM_LAYOUT_VERSION, 256, 256, 64, 4, 1, 1, fake, fake, fake, fake, fake,
                      fake, fake, fake)
    assert lib.hinm_spmm(ctypes.byref(L), fake, 0, fake, None) == H.HINM_ERR_SHAPE
