"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle, element by element.

Integer / index / byte results (masks, regions, counts, ranks, layout bytes, the
importance bits) must match exactly.  The fp32 product must satisfy
|y - y_ref| <= 1e-3 * sum|w||x| + 1e-5 (bf16 inputs, fp32 accumulation); where every
partial sum is an exact integer it must match bitwise.
"""
import numpy as np
import pytest

import hinm_inputs as hi
from oracle import hinm_oracle as O

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

TOL_REL, TOL_ABS = 1e-3, 1e-5


@pytest.fixture(scope="module")
def H():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import pruning_hinm_spmm_b200 as H
    return H


def dev_bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def dev_i32(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).cuda()


def status_ok(H):
    assert H.hinm_device_status() == 0


def layout_equal(L_gpu, L_ref, tiles=None):
    info = L_gpu.tile_info.cpu().numpy()
    np.testing.assert_array_equal(info if tiles is None else info[tiles],
                                  L_ref.tile_info if tiles is None else L_ref.tile_info[tiles])
    vd = L_gpu.vals_dense.cpu().numpy().view(np.uint8).reshape(-1, 16384)
    vs = L_gpu.vals_sparse.cpu().numpy().view(np.uint8).reshape(-1, 16384)
    me = L_gpu.meta.cpu().numpy().view(np.uint32)
    idd = L_gpu.idx_dense.cpu().numpy()
    ids = L_gpu.idx_sparse.cpu().numpy()
    rd = L_gpu.run_dense.cpu().numpy()
    rs = L_gpu.run_sparse.cpu().numpy()
    for t in (range(info.shape[0]) if tiles is None else tiles):
        nd, ns, d0, s0 = info[t]
        nd_r, ns_r, d0_r, s0_r = L_ref.tile_info[t]
        assert (nd, ns) == (nd_r, ns_r)
        np.testing.assert_array_equal(vd[d0:d0 + nd], L_ref.vals_dense[d0_r:d0_r + nd])
        np.testing.assert_array_equal(vs[s0:s0 + ns], L_ref.vals_sparse[s0_r:s0_r + ns])
        np.testing.assert_array_equal(me[s0:s0 + ns], L_ref.meta[s0_r:s0_r + ns])
        np.testing.assert_array_equal(idd[d0:d0 + nd], L_ref.idx_dense[d0_r:d0_r + nd])
        np.testing.assert_array_equal(ids[s0:s0 + ns], L_ref.idx_sparse[s0_r:s0_r + ns])
        np.testing.assert_array_equal(rd[d0:d0 + nd], L_ref.run_dense[d0_r:d0_r + nd])
        np.testing.assert_array_equal(rs[s0:s0 + ns], L_ref.run_sparse[s0_r:s0_r + ns])


def check_y(y_gpu, y_ref, bound, rows=None):
    y = y_gpu if rows is None else y_gpu[rows]
    err = np.abs(y.astype(np.float64) - y_ref)
    lim = TOL_REL * bound + TOL_ABS
    bad = err > lim
    assert not bad.any(), f"{bad.sum()} outputs out of tolerance; worst {(err - lim).max():.3e}"


def run_path(H, w, v_s=None, N=None):
    """GPU path step by step; returns every intermediate as numpy."""
    M, K, T = w.M, w.K, w.T
    W, X = dev_bf16(w.W_bits), dev_bf16(w.X_bits)
    perm = dev_i32(w.perm)
    I = H.hinm_importance(W, X)
    nc = H.hinm_search_num_candidates(K, w.t_s, w.alpha)
    R = torch.empty((M // T, nc), dtype=torch.float64, device="cuda")
    counts, vs, rank = H.hinm_boundary_search(I, perm, T, w.t_s, w.alpha, retained_out=R)
    if v_s is not None:
        c = np.array(H.hinm_counts_from_vs(K, w.t_s, v_s), dtype=np.int32)
        counts_used = dev_i32(np.tile(c, (M // T, 1)))
        rank_used = None
    else:
        counts_used, rank_used = counts, rank
    bm, region = H.hinm_mask(I, perm, counts_used, T, rank_used)
    L = H.hinm_compress(W, bm, region, perm, counts_used, T)
    Y = H.hinm_spmm(L, X)
    torch.cuda.synchronize()
    status_ok(H)
    return dict(I=I.cpu().numpy(), counts=counts.cpu().numpy(), vs=vs.cpu().numpy(),
                R=R.cpu().numpy(),
                rank=rank.cpu().numpy(), counts_used=counts_used.cpu().numpy(),
                bitmask=bm.cpu().numpy().view(np.uint32), region=region.cpu().numpy(), layout=L,
                Y=Y.cpu().numpy())


CASES = [
    # name, workload factory, fixed v_s (None = searched)
    ("tiny_hinm_T64", lambda: hi.tiny_hinm(0), 0.2),
    ("tiny_searched", lambda: hi.tiny_hinm(0), None),
    ("ragged_K200_N24_perm", lambda: hi.custom(256, 200, 24, 128, seed=3, t_s=0.625, v_s=None,
                                              random_perm=True), 0.4),
    ("ragged_K196_N40_T64", lambda: hi.custom(192, 196, 40, 64, seed=4, t_s=0.5, v_s=None,
                                             random_perm=True), 0.25),
    ("pure24_small_outliers", lambda: hi.custom(256, 256, 136, 128, seed=5, t_s=0.5, v_s=None,
                                                outlier_frac=0.01), 0.0),
    ("column_pruning_only", lambda: hi.custom(128, 192, 16, 64, seed=6, t_s=0.5, v_s=None), 0.5),
    ("dense_ts0", lambda: hi.custom(128, 128, 32, 128, seed=7, t_s=0.0, v_s=None), 0.0),
    ("all_pruned_ts1", lambda: hi.custom(128, 128, 16, 64, seed=8, t_s=1.0, v_s=None), 1.0),
    ("multi_block_K640_N264", lambda: hi.custom(384, 640, 264, 128, seed=9, t_s=0.75, v_s=None,
                                               random_perm=True), 0.6),
]


@pytest.mark.parametrize("name,make,v_s", CASES, ids=[c[0] for c in CASES])
def test_path_matches_oracle(H, name, make, v_s):
    w = make()
    g = run_path(H, w, v_s)
    # a1 importance: bit-exact
    I_ref = O.importance(w.W_bits, w.X_bits)
    np.testing.assert_array_equal(g["I"].view(np.uint32), I_ref.view(np.uint32))
    # a2/a3 search: counts, v_s, rank bit-exact
    sr = O.boundary_search(I_ref, w.perm, w.T, w.t_s, w.alpha)
    np.testing.assert_array_equal(g["counts"], sr.counts)
    np.testing.assert_array_equal(g["vs"], sr.v_s)
    np.testing.assert_array_equal(g["rank"], sr.rank)
    np.testing.assert_array_equal(g["R"], np.array(sr.R))  # exact sums, rounded once
    counts = g["counts_used"]
    # a4 mask
    bm_ref, reg_ref = O.mask(I_ref, w.perm, w.T, counts)
    np.testing.assert_array_equal(g["region"], reg_ref)
    np.testing.assert_array_equal(g["bitmask"], bm_ref)
    # a5 layout bytes
    L_ref = O.compress(w.W_bits, bm_ref, reg_ref, w.perm, counts, w.T)
    layout_equal(g["layout"], L_ref)
    # a6 product
    y_ref, bound = O.spmm_reference(w.W_bits, bm_ref, w.X_bits)
    check_y(g["Y"], y_ref, bound)


def test_identity_x_reproduces_masked_weight(H):
    """X = I_K (N = K): Y must equal W ⊙ M exactly, which pins the value layout, the
    metadata placement and the gather to the tensor cores' reading of them."""
    w = hi.custom(256, 256, 256, 128, seed=11, t_s=0.625, v_s=None, random_perm=True)
    w.X_bits = hi.f32_to_bf16_bits(np.eye(256, dtype=np.float32))
    w.N = 256
    g = run_path(H, w, v_s=0.375)
    Wm = O.masked_weight(w.W_bits, g["bitmask"])
    np.testing.assert_array_equal(g["Y"], Wm.astype(np.float32))


@pytest.mark.parametrize("T,N,perm", [(64, 16, False), (128, 48, True), (128, 264, True)])
def test_integer_product_bitwise(H, T, N, perm):
    w = hi.integer_workload(2 * T, 384, N, T, seed=2, t_s=0.625, v_s=None, random_perm=perm)
    g = run_path(H, w, v_s=0.375)
    Wm = O.masked_weight(w.W_bits, g["bitmask"]).astype(np.int64)
    Xi = hi.bf16_bits_to_f32(w.X_bits).astype(np.int64)
    np.testing.assert_array_equal(g["Y"].astype(np.int64), Wm @ Xi)
    assert np.array_equal(g["Y"], np.round(g["Y"]))


@pytest.mark.parametrize("ntiles,N", [(7, 1032), (9, 1040), (6, 2048)])
def test_tile_pairs_mixed_modes_integer_bitwise(H, ntiles, N):
    """Wide N, T = 128: the SpMM's work units are tile pairs.  Per-tile counts make some
    pairs select the same X rows block by block (both all 2:4, or both all dense: one B
    stage feeds both tiles) and others not (HiNM counts with gathered blocks, or different
    counts: the tiles run in sequence), with an odd tile count (a lone last tile), N not a
    multiple of 240 (a ragged last column block) and N % 16 == 8 (column boxes of 16).
    Integer inputs: Y must equal the masked product exactly."""
    T, K = 128, 384
    w = hi.integer_workload(ntiles * T, K, N, T, seed=12, t_s=0.5, v_s=None)
    all24 = list(H.hinm_counts_from_vs(K, 0.5, 0.0))
    hinm = list(H.hinm_counts_from_vs(K, 0.5, 0.25))
    dense = [K, 0, 0]
    pattern = [all24, all24, dense, dense, hinm, hinm, all24, dense, all24]
    counts = np.array([pattern[t % len(pattern)] for t in range(ntiles)], dtype=np.int32)
    W, X, perm = dev_bf16(w.W_bits), dev_bf16(w.X_bits), dev_i32(w.perm)
    I = H.hinm_importance(W, X)
    _, _, rank = H.hinm_boundary_search(I, perm, T, w.t_s, w.alpha)
    c = dev_i32(counts)
    bm, region = H.hinm_mask(I, perm, c, T, rank)
    L = H.hinm_compress(W, bm, region, perm, c, T)
    Y = H.hinm_spmm(L, X, tile_pairs=True)   # pairs where they share, tile by tile elsewhere
    Y0 = H.hinm_spmm(L, X)                   # no hint: one tile per work unit
    torch.cuda.synchronize()
    status_ok(H)
    run_d, run_s = L.run_dense.cpu().numpy(), L.run_sparse.cpu().numpy()
    info = L.tile_info.cpu().numpy()
    assert (run_s[info[0, 3]:info[0, 3] + info[0, 1]] >= 0).all()  # pair 0 shares its B
    assert (run_d[info[4, 2]:info[4, 2] + info[4, 0]] < 0).any()   # pair 2 gathers
    Wm = O.masked_weight(w.W_bits, bm.cpu().numpy().view(np.uint32)).astype(np.int64)
    Xi = hi.bf16_bits_to_f32(w.X_bits).astype(np.int64)
    np.testing.assert_array_equal(Y.cpu().numpy().astype(np.int64), Wm @ Xi)
    np.testing.assert_array_equal(Y0.cpu().numpy().astype(np.int64), Wm @ Xi)


@pytest.mark.parametrize("T,N,pairs", [(128, 264, False), (64, 40, False), (128, 1040, True)])
def test_translate_index_layout_and_product(H, T, N, pairs):
    """Cross-layer index translation on the GPU: the translated layout equals the oracle's
    translation of the oracle's layout byte for byte, an identity map changes nothing, and
    the product with the reordered X is bitwise the original product (integer inputs, also
    equal to the exact masked product), with and without the tile-pair hint."""
    K = 384
    w = hi.integer_workload(3 * T, K, N, T, seed=21, t_s=0.625, v_s=None, random_perm=True)
    g = run_path(H, w, v_s=0.375)
    L = g["layout"]
    X = dev_bf16(w.X_bits)
    Y0 = H.hinm_spmm(L, X, tile_pairs=pairs).cpu().numpy()
    H.hinm_translate_index(L, dev_i32(np.arange(K)))
    torch.cuda.synchronize()
    status_ok(H)
    L_ref = O.compress(w.W_bits, g["bitmask"], g["region"], w.perm, g["counts_used"], T)
    layout_equal(L, L_ref)
    rng = np.random.default_rng(5)
    sigma = rng.permutation(K).astype(np.int32)      # delivered row r holds channel sigma[r]
    roc = np.argsort(sigma).astype(np.int32)
    H.hinm_translate_index(L, dev_i32(roc))
    X_del = dev_bf16(w.X_bits[sigma])
    Y1 = H.hinm_spmm(L, X_del, tile_pairs=pairs).cpu().numpy()
    torch.cuda.synchronize()
    status_ok(H)
    layout_equal(L, O.translate_index(L_ref, roc))
    np.testing.assert_array_equal(Y1.view(np.uint32), Y0.view(np.uint32))
    Wm = O.masked_weight(w.W_bits, g["bitmask"]).astype(np.int64)
    np.testing.assert_array_equal(Y1.astype(np.int64), Wm @ hi.bf16_bits_to_f32(w.X_bits).astype(np.int64))


def test_translate_index_bad_map_reported(H):
    """A map entry outside [0, K) is reported as HINM_ERR_INVALID_ARG (and mapped to row 0),
    not a fault; the context stays usable."""
    w = hi.custom(128, 128, 16, 128, seed=4, t_s=0.5, v_s=None)
    g = run_path(H, w, v_s=0.25)
    bad = np.arange(128, dtype=np.int32)
    bad[3] = 1 << 20
    H.hinm_translate_index(g["layout"], dev_i32(bad))
    torch.cuda.synchronize()
    assert H.hinm_device_status() == H.HINM_ERR_INVALID_ARG
    assert H.hinm_device_status() == 0


# one case per epilogue store site: the 256-column kernel (ragged N), the 16-column persistent
# path (more units than half the SMs), the split-K leader (decode shape), the pair kernel
EPI_CASES = [
    ("bn256_ragged", dict(M=384, K=384, N=264, T=128, v_s=None, perm=True, pairs=False)),
    ("bn16_persistent", dict(M=25600, K=128, N=16, T=128, v_s=None, perm=True, pairs=False)),
    ("splitk_leader", dict(M=256, K=1024, N=16, T=128, v_s=None, perm=True, pairs=False)),
    ("pair_kernel", dict(M=640, K=256, N=1040, T=128, v_s=0.0, perm=False, pairs=True)),
]


@pytest.mark.parametrize("name,cfg", EPI_CASES, ids=[c[0] for c in EPI_CASES])
def test_spmm_epilogue_matches_oracle(H, name, cfg):
    """The fused epilogue (per-row bias, ReLU / SiLU / GELU, fp32 or bf16 Y) at every store
    site.  Exact: no epilogue = hinm_spmm bit for bit, and the bf16 Y of the plain product is
    the round-to-nearest-even of the GPU's own fp32 Y.  Against the oracle: act(y + bias)
    within the product's bound times the activations' slope (<= 1.2), plus their fp32
    evaluation and, for bf16, half a bf16 ulp."""
    M, K, N, T = cfg["M"], cfg["K"], cfg["N"], cfg["T"]
    w = hi.custom(M, K, N, T, seed=31, t_s=0.5, v_s=cfg["v_s"], random_perm=cfg["perm"])
    W, X, perm = dev_bf16(w.W_bits), dev_bf16(w.X_bits), dev_i32(w.perm)
    hp = H.HotPath(M, K, N, T, 0.5, w.alpha)
    fixed = None
    if cfg["v_s"] is not None:
        fixed = dev_i32(np.tile(np.array(H.hinm_counts_from_vs(K, 0.5, cfg["v_s"]), dtype=np.int32),
                                (M // T, 1)))
    pairs = cfg["pairs"]
    Y = hp.run(W, X, perm, fixed_counts=fixed, tile_pairs=pairs).clone()
    L = hp.layout
    Y_plain = H.hinm_spmm_epilogue(L, X, tile_pairs=pairs)
    Y_b16 = H.hinm_spmm_epilogue(L, X, out_bf16=True, tile_pairs=pairs)
    torch.cuda.synchronize()
    status_ok(H)
    np.testing.assert_array_equal(Y_plain.cpu().numpy().view(np.uint32), Y.cpu().numpy().view(np.uint32))
    np.testing.assert_array_equal(Y_b16.view(torch.int16).cpu().numpy(),
                                  Y.to(torch.bfloat16).view(torch.int16).cpu().numpy())
    bm = hp.bitmask.cpu().numpy().view(np.uint32)
    y_ref, bound = O.spmm_reference(w.W_bits, bm, w.X_bits)
    rng = np.random.default_rng(3)
    bias = rng.normal(0.0, 0.05, M).astype(np.float32)
    bias_d = torch.from_numpy(bias).cuda()
    for act in (H.HINM_ACT_RELU, H.HINM_ACT_SILU, H.HINM_ACT_GELU):
        ref = O.spmm_epilogue_reference(y_ref, bias, act)
        base = 1.2 * (TOL_REL * bound + TOL_ABS) + 1e-6 * (np.abs(ref) + 1.0)
        for b16 in (False, True):
            got = H.hinm_spmm_epilogue(L, X, bias=bias_d, activation=act, out_bf16=b16,
                                       tile_pairs=pairs)
            torch.cuda.synchronize()
            g = got.float().cpu().numpy().astype(np.float64)
            tol = base + bf16_half_ulp(np.abs(ref) + base) if b16 else base
            err = np.abs(g - ref)
            assert (err <= tol).all(), f"act {act} bf16 {b16}: worst excess {(err - tol).max():.3e}"
    status_ok(H)


def bf16_half_ulp(v):
    """Half a bf16 ulp at magnitude v (>= 0): 2^(e - 8) for v in [2^e, 2^(e+1)), i.e. between
    2^-9 and 2^-8 of v; the round-to-nearest-even error of any value of magnitude <= v is at
    most this (ulps do not shrink as the magnitude grows)."""
    v = np.maximum(np.asarray(v, dtype=np.float64), 2.0 ** -133)
    return np.ldexp(1.0, np.floor(np.log2(v)).astype(np.int64) - 8)


def _hc_bound(la, eps, tau):
    """Per-element bound on |z_fp32 - z_fp64| from the fp32 operation order of the kernel:
    the noise logit as logf of eps / (1 - eps) (three roundings of the ratio: 3 half-ulps of
    relative error, so 3 * 2^-24 absolute after the log) with logf within 1 ulp, expf within
    2 ulp (CUDA's documented maxima), each fp32 add / multiply / reciprocal within half an
    ulp (the scale by 1/tau: the reciprocal's and the product's roundings), carried through
    the sigmoid's slope s(1 - s) and the stretch by 1.2; plus the fp32 stretch constants'
    offset from the fp64 ones."""
    d = 2.0 ** -24
    la = la.astype(np.float64)
    e = eps.astype(np.float64)
    l1, l2 = np.abs(np.log(e)), np.abs(np.log1p(-e))
    logit = np.log(e) - np.log1p(-e)
    err_logit = 4 * d + np.abs(logit) * 2 * d + (l1 + l2) * 2 * d
    x = (logit + la) / tau
    err_x = (err_logit + np.abs(logit + la) * d) / tau + np.abs(x) * 3 * d
    s = 1.0 / (1.0 + np.exp(-x))
    err_s = s * (1 - s) * err_x + 8 * d * s
    return 2.0 * (1.2 * err_s + 1.2 * s * 1e-7 + 4 * d + 4e-9)


@pytest.mark.parametrize("n,tau", [(4 * 10007, 2.0 / 3.0), (4 * 262147, 0.1), (1 << 22, 1.0)])
def test_hard_concrete_forward_matches_oracle(H, n, tau):
    """The Hard-Concrete forward on the GPU against the fp64 oracle: z within the fp32
    bound per element, the hardened bits exactly (z > 0.5) of the GPU's own z, and both
    regularisers within the summed bound; noise at the ends (eps = 0, 1) gives z = 0, 1."""
    rng = np.random.default_rng(n)
    la = rng.normal(0.0, 2.0, n).astype(np.float32)
    eps = rng.uniform(0.0, 1.0, n).astype(np.float32)
    eps[:4] = (0.0, 1.0, 0.5, 0.5)
    la[2:4] = (0.0, 40.0)
    z, hard, sums = H.hinm_hard_concrete_forward(torch.from_numpy(la).cuda(),
                                                 torch.from_numpy(eps).cuda(), tau)
    torch.cuda.synchronize()
    z, hard, sums = z.cpu().numpy(), hard.cpu().numpy(), sums.cpu().numpy()
    assert tuple(z[:4]) == (0.0, 1.0, z[2], 1.0) and abs(z[2] - 0.5) < 1e-6
    inner = slice(4, None)
    z_ref, _, _ = O.hard_concrete(la[inner], eps[inner], tau)
    bound = _hc_bound(la[inner], eps[inner], tau)
    err = np.abs(z[inner].astype(np.float64) - z_ref)
    assert (err <= bound).all(), f"worst excess {(err - bound).max():.3e}"
    np.testing.assert_array_equal(hard, (z > 0.5).astype(np.uint8))
    # the hardened bits against the oracle's own decision z_ref > 0.5, wherever z_ref is
    # farther from the threshold than the fp32 bound (there the two cannot disagree)
    _, hard_ref, _ = O.hard_concrete(la[inner], eps[inner], tau)
    sure = np.abs(z_ref - 0.5) > bound
    assert sure.mean() > 0.99
    np.testing.assert_array_equal(hard[inner][sure], hard_ref[sure])
    # the first group's reference from the GPU's own values (the ends of the noise range)
    s0 = float(z[:4].astype(np.float64).sum())
    want_z = s0 + float(z_ref.sum())
    want_h = abs(s0 - 2.0) + float(np.abs(z_ref.reshape(-1, 4).sum(axis=1) - 2.0).sum())
    tol = float(bound.sum()) * 4 + 1e-9 * n
    assert abs(sums[0] - want_z) <= tol and abs(sums[1] - want_h) <= tol


def test_hard_concrete_non_finite_inputs(H):
    """NaN and infinite inputs against the fp64 oracle: a NaN log alpha or noise, and the
    undefined sums -inf + inf of the logit (eps = 0 with log alpha = +inf, eps = 1 with
    log alpha = -inf) give z = NaN, hardened to 0, and NaN regulariser sums; log alpha =
    +-inf with interior noise gives z = 1 / 0."""
    nan, inf = np.float32(np.nan), np.float32(np.inf)
    la = np.array([nan, 0.0, inf, -inf, inf, -inf, 0.5, 1.0], dtype=np.float32)
    eps = np.array([0.3, nan, 0.0, 1.0, 0.4, 0.6, 0.5, 0.25], dtype=np.float32)
    z, hard, sums = H.hinm_hard_concrete_forward(torch.from_numpy(la).cuda(),
                                                 torch.from_numpy(eps).cuda(), 0.5)
    torch.cuda.synchronize()
    z, hard, sums = z.cpu().numpy(), hard.cpu().numpy(), sums.cpu().numpy()
    z_ref, hard_ref, sums_ref = O.hard_concrete(la, eps, 0.5)
    np.testing.assert_array_equal(np.isnan(z), np.isnan(z_ref))
    assert np.isnan(z[:4]).all()
    np.testing.assert_array_equal(z[4:6], z_ref[4:6].astype(np.float32))   # exactly 1, 0
    fin = slice(6, 8)  # finite inputs
    assert (np.abs(z[fin] - z_ref[fin]) <= _hc_bound(la[fin], eps[fin], 0.5)).all()
    np.testing.assert_array_equal(hard, hard_ref)
    assert np.isnan(sums).all() and np.isnan(sums_ref).all()


def test_hard_concrete_deterministic_mode(H):
    """eps = 1/2 removes the noise: z = clip(1.2 sigmoid(log alpha / tau) - 0.1) exactly as
    the oracle's deterministic mask, with the hardened mask at 0.5."""
    n, tau = 4096, 0.5
    la = np.linspace(-3.0, 3.0, n).astype(np.float32)
    eps = np.full(n, 0.5, dtype=np.float32)
    z, hard, _ = H.hinm_hard_concrete_forward(torch.from_numpy(la).cuda(),
                                              torch.from_numpy(eps).cuda(), tau)
    z = z.cpu().numpy()
    z_ref, _, _ = O.hard_concrete(la, eps, tau)
    assert (np.abs(z - z_ref) <= _hc_bound(la, eps, tau)).all()
    assert (z[la < -1.0] < 0.5).all() and (z[la > 1.0] > 0.5).all()


def test_channel_energy_rounding_fallback(H):
    """Channels whose fp64 sum sits on an fp32 rounding midpoint: the order matters there,
    so the GPU must reproduce the sequential sum (1 first: 1.0; 1 last: 1 + 2^-23)."""
    K, N, M = 64, 64, 8
    rng = np.random.default_rng(11)
    Xf = rng.normal(0.0, 1.0, (K, N)).astype(np.float32)
    Xf[0] = [1.0, 2.0 ** -12] + [2.0 ** -27] * (N - 2)
    Xf[1] = [2.0 ** -12] + [2.0 ** -27] * (N - 2) + [1.0]
    Xf[2] = 2.0 ** -27                       # all tiny: exact in any order
    Xf[3] = 0.0
    X = hi.f32_to_bf16_bits(Xf)
    W = hi.f32_to_bf16_bits(np.ones((M, K), dtype=np.float32))
    I = H.hinm_importance(dev_bf16(W), dev_bf16(X)).cpu().numpy()
    status_ok(H)
    I_ref = O.importance(W, X)
    assert I_ref[0, 0] == np.float32(1.0) and I_ref[0, 1] == np.float32(1.0 + 2.0 ** -23)
    np.testing.assert_array_equal(I.view(np.uint32), I_ref.view(np.uint32))


@pytest.mark.parametrize("name,make,v_s", CASES, ids=[c[0] for c in CASES])
def test_importance_stats_and_search_with_stats(H, name, make, v_s):
    """The importance step's fused tile statistics: I bit for bit as hinm_importance, V
    equal to the oracle's vector scores (by channel), the tile maxima equal to the largest
    exponent of the tile's importances, and the search given them returns exactly what the
    search computing them itself returns (counts, v_s, rank, every R(m))."""
    w = make()
    M, K, T = w.M, w.K, w.T
    nt = M // T
    W, X, perm = dev_bf16(w.W_bits), dev_bf16(w.X_bits), dev_i32(w.perm)
    I0 = H.hinm_importance(W, X)
    I1, stats = H.hinm_importance_stats(W, X, T)
    nc = H.hinm_search_num_candidates(K, w.t_s, w.alpha)
    R0 = torch.empty((nt, nc), dtype=torch.float64, device="cuda")
    R1 = torch.empty((nt, nc), dtype=torch.float64, device="cuda")
    c0, v0, r0 = H.hinm_boundary_search(I0, perm, T, w.t_s, w.alpha, retained_out=R0)
    c1, v1, r1 = H.hinm_boundary_search(I1, perm, T, w.t_s, w.alpha, retained_out=R1, stats=stats)
    torch.cuda.synchronize()
    status_ok(H)
    I_np = I0.cpu().numpy()
    np.testing.assert_array_equal(I1.cpu().numpy().view(np.uint32), I_np.view(np.uint32))
    V, pmax = H.tile_stats_views(stats, M, K, T)
    np.testing.assert_array_equal(V.cpu().numpy()[:, w.perm], O.vector_scores(I_np, w.perm, T))
    top = I_np.view(np.uint32).reshape(nt, T * K).max(axis=1).astype(np.int64)
    p_ref = np.where(top > 0, np.maximum(top >> 23, 1) - 1, 0)
    np.testing.assert_array_equal(pmax.cpu().numpy(), p_ref)
    for a, b in ((c0, c1), (v0, v1), (r0, r1), (R0, R1)):
        np.testing.assert_array_equal(a.cpu().numpy(), b.cpu().numpy())


@pytest.mark.parametrize("name,make,v_s", CASES, ids=[c[0] for c in CASES])
def test_search_decision_without_retained_matches_full_scan(H, name, make, v_s):
    """With no R requested the scan may stop evaluating candidates after a tile's decision;
    the counts and v_s must still equal the full scan's and the oracle's."""
    w = make()
    M, K, T = w.M, w.K, w.T
    I = H.hinm_importance(dev_bf16(w.W_bits), dev_bf16(w.X_bits))
    perm = dev_i32(w.perm)
    c_e, vs_e, _ = H.hinm_boundary_search(I, perm, T, w.t_s, w.alpha, want_rank=False)
    nc = H.hinm_search_num_candidates(K, w.t_s, w.alpha)
    R = torch.empty((M // T, nc), dtype=torch.float64, device="cuda")
    c_f, vs_f, _ = H.hinm_boundary_search(I, perm, T, w.t_s, w.alpha, want_rank=False,
                                          retained_out=R)
    torch.cuda.synchronize()
    status_ok(H)
    sr = O.boundary_search(I.cpu().numpy(), w.perm, T, w.t_s, w.alpha)
    np.testing.assert_array_equal(c_e.cpu().numpy(), sr.counts)
    np.testing.assert_array_equal(vs_e.cpu().numpy(), np.asarray(sr.v_s))
    np.testing.assert_array_equal(c_f.cpu().numpy(), sr.counts)
    np.testing.assert_array_equal(vs_f.cpu().numpy(), np.asarray(sr.v_s))


@pytest.mark.parametrize("M,K,N,perm", [(256, 512, 128, False), (384, 640, 264, True),
                                         (128, 4096, 16, True)])
def test_dense_ts0_matches_torch_matmul(H, M, K, N, perm):
    """t_s = 0 keeps every weight: the SpMM is a dense GEMM, so torch.matmul (fp32 of the bf16
    inputs) is an independent third opinion next to the oracle."""
    w = hi.custom(M, K, N, 128, seed=41, t_s=0.0, v_s=None, random_perm=perm)
    W, X = dev_bf16(w.W_bits), dev_bf16(w.X_bits)
    hp = H.HotPath(M, K, N, 128, 0.0, w.alpha)
    Y = hp.run(W, X, dev_i32(w.perm))
    torch.cuda.synchronize()
    status_ok(H)
    assert int(hp.counts[:, 2].min()) == K  # every vector dense
    Wf, Xf = W.float(), X.float()
    ref = (Wf.double() @ Xf.double()).cpu().numpy()
    bound = (Wf.abs().double() @ Xf.abs().double()).cpu().numpy()
    check_y(Y.cpu().numpy(), ref, bound)
    mm = torch.matmul(Wf, Xf).cpu().numpy()
    check_y(Y.cpu().numpy(), mm.astype(np.float64), bound)


@pytest.mark.parametrize("M,K,N,T,v_s,rperm", [
    (5120, 256, 2048, 128, 0.0, True),    # 20 tile pairs x 9 column blocks, gathered X rows
    (5120, 256, 2048, 128, 0.0, False),   # the same with every pair sharing its B stages
    (25600, 128, 16, 128, 0.25, True),    # 200 units of 16 columns, persistent (no split-K)
    (20480, 128, 264, 64, 0.25, True),    # T = 64, 320 tiles x 2 column blocks, ragged N
])
def test_spmm_units_shared_across_ctas(H, M, K, N, T, v_s, rperm):
    """More work units than SMs (several per persistent CTA, with a ragged last wave):
    Y against the fp64 masked product (the GPU's mask, checked elsewhere), and bitwise the
    same over two runs."""
    w = hi.custom(M, K, N, T, seed=51, t_s=0.5, v_s=v_s, random_perm=rperm)
    W, X, perm = dev_bf16(w.W_bits), dev_bf16(w.X_bits), dev_i32(w.perm)
    nt = M // T
    c = dev_i32(np.tile(np.array(H.hinm_counts_from_vs(K, 0.5, v_s), dtype=np.int32), (nt, 1)))
    hp = H.HotPath(M, K, N, T, 0.5, w.alpha)
    pairs = H.tile_pairs_hint(H.hinm_counts_from_vs(K, 0.5, v_s), w.perm, K)
    assert pairs == (v_s == 0.0 and not rperm)
    Y1 = hp.run(W, X, perm, fixed_counts=c, tile_pairs=pairs).clone()
    Y2 = hp.run(W, X, perm, fixed_counts=c, tile_pairs=pairs).clone()
    torch.cuda.synchronize()
    status_ok(H)
    np.testing.assert_array_equal(Y1.cpu().numpy().view(np.uint32), Y2.cpu().numpy().view(np.uint32))
    bm = hp.bitmask.cpu().numpy().view(np.uint32)
    y_ref, bound = O.spmm_reference(w.W_bits, bm, w.X_bits)
    check_y(Y1.cpu().numpy(), y_ref, bound)


def test_gpu_permutation_invariance(H):
    """Reordering input channels consistently leaves the GPU result unchanged (FlexHiNM-GP
    notes, 关键设计 2): run(W, X, pi) and run(W[:, pi], X[pi, :], identity) give the same
    counts, the same mask after remapping, the same value and metadata bytes, indices related
    by pi, and bitwise the same Y."""
    w = hi.custom(256, 640, 72, 128, seed=31, t_s=0.625, v_s=None, random_perm=True)
    M, K, N, T = w.M, w.K, w.N, w.T
    Wp = np.ascontiguousarray(w.W_bits[:, w.perm])
    Xp = np.ascontiguousarray(w.X_bits[w.perm, :])
    ident = np.arange(K, dtype=np.int32)
    out = []
    for Wb, Xb, pm in ((w.W_bits, w.X_bits, w.perm), (Wp, Xp, ident)):
        hp = H.HotPath(M, K, N, T, w.t_s, w.alpha)
        Y = hp.run(dev_bf16(Wb), dev_bf16(Xb), dev_i32(pm))
        torch.cuda.synchronize()
        status_ok(H)
        L = hp.layout
        out.append(dict(counts=hp.counts.cpu().numpy(), Y=Y.cpu().numpy(),
                        bits=O.unpack_bits(hp.bitmask.cpu().numpy().view(np.uint32), K),
                        vd=L.vals_dense.cpu().numpy(), vsp=L.vals_sparse.cpu().numpy(),
                        meta=L.meta.cpu().numpy(), info=L.tile_info.cpu().numpy(),
                        idd=L.idx_dense.cpu().numpy(), ids=L.idx_sparse.cpu().numpy()))
    a, b = out
    np.testing.assert_array_equal(a["counts"], b["counts"])
    np.testing.assert_array_equal(a["bits"][:, w.perm], b["bits"])
    np.testing.assert_array_equal(a["info"], b["info"])
    # the blocks each tile uses (buffers are allocated to capacity)
    dense = np.concatenate([np.arange(d0, d0 + nd) for nd, ns, d0, s0 in a["info"]])
    sparse = np.concatenate([np.arange(s0, s0 + ns) for nd, ns, d0, s0 in a["info"]])
    np.testing.assert_array_equal(a["vd"][dense], b["vd"][dense])
    np.testing.assert_array_equal(a["vsp"][sparse], b["vsp"][sparse])
    np.testing.assert_array_equal(a["meta"][sparse], b["meta"][sparse])
    for ia, ib in ((a["idd"][dense], b["idd"][dense]), (a["ids"][sparse], b["ids"][sparse])):
        real = ~((ia == 0) & (ib == 0))  # padding entries are 0 on both sides
        np.testing.assert_array_equal(ia[real], w.perm[ib[real]])
    np.testing.assert_array_equal(a["Y"].view(np.uint32), b["Y"].view(np.uint32))


def test_hand_built_first_drop(H):
    """The hand-built tile where regrouping makes R drop at m = 2: the GPU scan stops at m=1."""
    K, N, T = 64, 8, 64
    mags = np.array([8.0] * 28 + [3.0] * 2 + [2.875] * 2 + [1.25] * 2 + [1.0] * 2 + [0.5] * 28)
    signs = np.where(np.random.default_rng(0).random((T, K)) < 0.5, -1.0, 1.0)
    W = hi.f32_to_bf16_bits((signs * mags[None, :]).astype(np.float32))
    X = hi.f32_to_bf16_bits(np.ones((K, N), dtype=np.float32))
    I = H.hinm_importance(dev_bf16(W), dev_bf16(X))
    counts, vs, _ = H.hinm_boundary_search(I, None, T, 0.5, 1 / 32)
    assert tuple(counts.cpu().numpy()[0]) == (30, 4, 30)
    assert vs.cpu().numpy()[0] == 0.5 - 1 / 32


def test_bad_mask_is_reported_not_faulted(H):
    """A 2:4 group with 3 kept bits sets HINM_ERR_BAD_MASK in the device status word."""
    w = hi.custom(128, 128, 16, 128, seed=1, t_s=0.5, v_s=None)
    W, X = dev_bf16(w.W_bits), dev_bf16(w.X_bits)
    I = H.hinm_importance(W, X)
    c = dev_i32(np.array([H.hinm_counts_from_vs(128, 0.5, 0.0)], dtype=np.int32))
    bm, region = H.hinm_mask(I, None, c, 128)
    bm = bm.clone()
    bm[0, 0] = -1  # all 32 channels of row 0 kept: 8 groups with 4 kept bits
    H.hinm_compress(W, bm, region, None, c, 128)
    torch.cuda.synchronize()
    assert H.hinm_device_status() == H.HINM_ERR_BAD_MASK
    assert H.hinm_device_status() == 0  # cleared by the read


def test_extreme_dynamic_range_exact_sums(H):
    """Importances spanning more than 2^83 within a tile (weights near 1e-20 give fp32
    subnormal importances): the values below the tile's fixed-point window take the exact
    exponent-bucket path, and R(m), counts, rank and mask still match the oracle bit for bit."""
    rng = np.random.default_rng(5)
    M, K, N, T = 256, 256, 16, 128
    scale = np.where(rng.random(K) < 0.3, 1e-20, 1.0).astype(np.float32)
    Wf = (rng.standard_normal((M, K)).astype(np.float32) * scale[None, :])
    Wf[:, :8] *= np.float32(1e-19)  # a few columns entirely in the tiny range
    w = hi.Workload(name="extreme", M=M, K=K, N=N, T=T, W_bits=hi.f32_to_bf16_bits(Wf),
                    X_bits=hi.f32_to_bf16_bits(rng.standard_normal((K, N)).astype(np.float32)),
                    perm=rng.permutation(K).astype(np.int32), t_s=0.5, v_s=None)
    g = run_path(H, w, None)
    I_ref = O.importance(w.W_bits, w.X_bits)
    np.testing.assert_array_equal(g["I"].view(np.uint32), I_ref.view(np.uint32))
    nz = I_ref[I_ref > 0].astype(np.float64)
    assert np.log2(nz.max() / nz.min()) > 100   # really exercises the bucket path
    sr = O.boundary_search(I_ref, w.perm, T, w.t_s, w.alpha)
    np.testing.assert_array_equal(g["R"], np.array(sr.R))
    np.testing.assert_array_equal(g["counts"], sr.counts)
    np.testing.assert_array_equal(g["rank"], sr.rank)
    bm_ref, reg_ref = O.mask(I_ref, w.perm, T, sr.counts)
    np.testing.assert_array_equal(g["bitmask"], bm_ref)


def test_invalid_permutation_reported(H):
    """A permutation with a repeated or an out-of-range channel is reported on the device
    status word (every access stays clamped inside the matrices)."""
    w = hi.custom(128, 256, 16, 64, seed=5, t_s=0.5, v_s=0.25)
    W, X = dev_bf16(w.W_bits), dev_bf16(w.X_bits)
    I = H.hinm_importance(W, X)
    c = dev_i32(np.array([H.hinm_counts_from_vs(w.K, w.t_s, w.v_s)] * (w.M // w.T), dtype=np.int32))
    good = np.arange(w.K, dtype=np.int32)
    H.hinm_mask(I, dev_i32(good), c, w.T)
    torch.cuda.synchronize()
    assert H.hinm_device_status() == 0
    dup = good.copy()
    dup[7] = dup[3]
    oob = good.copy()
    oob[11] = w.K + 5
    for bad in (dup, oob):
        H.hinm_mask(I, dev_i32(bad), c, w.T)
        torch.cuda.synchronize()
        assert H.hinm_device_status() == H.HINM_ERR_INVALID_ARG
        assert H.hinm_device_status() == 0  # cleared by the read


def test_bounded_wait_times_out_and_context_survives(H):
    """A wait that nothing completes gives up after its limit with HINM_ERR_DEVICE_TIMEOUT
    (the same bounded wait every pipelined kernel uses); the abort flag releases the other
    waiter, and the context keeps working afterwards."""
    import time
    torch.cuda.synchronize()
    assert H.hinm_device_status() == 0
    t0 = time.perf_counter()
    H.hinm_selftest_wait_timeout(20_000_000)  # 20 ms
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    assert H.hinm_device_status() == H.HINM_ERR_DEVICE_TIMEOUT
    assert 0.015 < elapsed < 1.0  # gave up after about the limit, not the 2 s default
    assert H.hinm_device_status() == 0
    w = hi.tiny_hinm()
    g = run_path(H, w, None)  # the context is still usable
    assert H.hinm_device_status() == 0
    assert g["counts"].shape[0] == w.M // w.T


SWEEP_LINEARS = ["q", "k", "v", "o", "gate", "up", "down"]
SWEEP_TS = [0.5, 0.625, 0.75]


@pytest.mark.parametrize("layer", list(range(1, 32)))
def test_llama_sweep_other_layers_sampled(H, layer):
    """Layers 1..31 of the sweep (one linear and one t_s per layer, rotating; N = 16): the
    search's counts, v_s and ranking, the mask, region and layout bytes of one sampled tile
    bit for bit, and that tile's Y within tolerance."""
    linear = SWEEP_LINEARS[layer % 7]
    t_s = SWEEP_TS[layer % 3]
    N = 16
    w = hi.llama_sweep_layer(layer, linear, N, t_s)
    M, K, T = w.M, w.K, w.T
    nt = M // T
    W, X, perm = dev_bf16(w.W_bits), dev_bf16(w.X_bits), dev_i32(w.perm)
    hp = H.HotPath(M, K, N, T, w.t_s, w.alpha)
    Y = hp.run(W, X, perm)  # counts from the search
    torch.cuda.synchronize()
    status_ok(H)
    tiles = [layer % nt]
    rows = np.concatenate([np.arange(t * T, (t + 1) * T) for t in tiles])
    I_rows = O.importance_rows(w.W_bits, w.X_bits, rows)
    np.testing.assert_array_equal(hp.I[rows].cpu().numpy().view(np.uint32), I_rows.view(np.uint32))
    I_full_rows = np.zeros((M, K), dtype=np.float32)
    I_full_rows[rows] = I_rows
    sr = O.boundary_search(I_full_rows, w.perm, T, t_s, w.alpha, tiles=tiles)
    counts = hp.counts.cpu().numpy()
    np.testing.assert_array_equal(counts[tiles], sr.counts[tiles])
    np.testing.assert_array_equal(hp.vs.cpu().numpy()[tiles], np.asarray(sr.v_s)[tiles])
    np.testing.assert_array_equal(hp.rank.cpu().numpy()[tiles], sr.rank[tiles])
    bm_ref, reg_ref = O.mask(I_full_rows, w.perm, T, counts, tiles=tiles)
    bm = hp.bitmask.cpu().numpy().view(np.uint32)
    np.testing.assert_array_equal(bm[rows], bm_ref[rows])
    np.testing.assert_array_equal(hp.region.cpu().numpy()[tiles], reg_ref[tiles])
    L_ref = O.compress(w.W_bits, bm_ref, reg_ref, w.perm, counts, T, tiles=tiles)
    layout_equal(hp.layout, L_ref, tiles=tiles)
    y_ref, bound = O.spmm_reference(w.W_bits, bm_ref, w.X_bits, rows=rows)
    check_y(Y.cpu().numpy(), y_ref, bound, rows=rows)
