"""Pins of the CPU oracle to facts fixed outside the oracle itself.

Each test checks an oracle function against something the pages or the mathematics fix:
a printed example (tests/golden), a closed form, exact rational arithmetic, brute force
on tiny inputs, an invariant, or a special case that reduces to a textbook rule.  The
cases are chosen so that a dropped term, a wrong sign or index, a transposed operand or
a wrong tie rule fails at least one of them.
"""
import itertools
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest

import hinm_inputs as hi
from oracle import hinm_oracle as O


def bf(a):
    return hi.f32_to_bf16_bits(np.asarray(a, dtype=np.float32))


def f32(bits):
    return hi.bf16_bits_to_f32(bits)


# ----------------------------------------------------------------------------- importance
def test_energy_closed_form_ones():
    # X = 1 everywhere: s_c = N exactly, I = w^2 * N.
    K, N = 7, 13
    X = bf(np.ones((K, N)))
    assert np.array_equal(O.channel_energy(X), np.full(K, N, dtype=np.float32))
    W = bf([[0.5, -2.0, 3.0, 0.25, 1.0, -1.5, 0.125]])
    I = O.importance(W, X)
    np.testing.assert_array_equal(I[0], np.array([0.25, 4.0, 9.0, 0.0625, 1.0, 2.25, 0.015625],
                                                 dtype=np.float32) * N)


def test_energy_is_the_sequential_fp64_sum():
    # The reading fixes the order (n ascending, fp64).  Row [1, 2^-12, 62 x 2^-27]: the
    # squares are 1, 2^-24 and 2^-54.  In order, 1 + 2^-24 is exact and each 2^-54 is a
    # quarter of an fp64 ulp at 1, so it is lost: the sum is 1 + 2^-24, the midpoint between
    # fp32 1 and 1 + 2^-23, which rounds to even (1).  The same squares with the 1 last add
    # up exactly first (2^-24 + 62 * 2^-54), then 1 + 2^-24 + 31 * 2^-53 rounds to
    # 1 + 2^-24 + 2^-48 in fp64, above the midpoint: 1 + 2^-23.  The exact sum rounds up too.
    N = 64
    a = [1.0, 2.0 ** -12] + [2.0 ** -27] * (N - 2)
    b = [2.0 ** -12] + [2.0 ** -27] * (N - 2) + [1.0]
    X = bf([a, b])
    s = O.channel_energy(X)
    assert s[0] == np.float32(1.0)
    assert s[1] == np.float32(1.0 + 2.0 ** -23)
    exact = sum(Fraction(v) ** 2 for v in a)
    assert exact > 1 + Fraction(1, 2 ** 24)          # so fl32(exact sum) would be 1 + 2^-23


def test_importance_hand_example_not_transposed():
    # W = [[1, 2], [3, 0.5]], X = [[1, 1, 1], [2, 0, 0]]  ->  s = [3, 4]
    # I = [[1*3, 4*4], [9*3, 0.25*4]] = [[3, 16], [27, 1]]
    W = bf([[1.0, 2.0], [3.0, 0.5]])
    X = bf([[1.0, 1.0, 1.0], [2.0, 0.0, 0.0]])
    np.testing.assert_array_equal(O.channel_energy(X), np.array([3.0, 4.0], dtype=np.float32))
    np.testing.assert_array_equal(O.importance(W, X), np.array([[3, 16], [27, 1]], dtype=np.float32))


def test_importance_rows_hand_example():
    # the hand example above: row 1 alone is [27, 1], row 0 alone [3, 16]; the energies are
    # still taken over all of X
    W = bf([[1.0, 2.0], [3.0, 0.5]])
    X = bf([[1.0, 1.0, 1.0], [2.0, 0.0, 0.0]])
    np.testing.assert_array_equal(O.importance_rows(W, X, np.array([1])),
                                  np.array([[27, 1]], dtype=np.float32))
    np.testing.assert_array_equal(O.importance_rows(W, X, np.array([1, 0])),
                                  np.array([[27, 1], [3, 16]], dtype=np.float32))


def test_vector_scores_accumulate_in_fp64():
    """R3: a vector's score is the fp64 sum of its importances.  Column a holds 1 and then
    63 values of 2^-25 (exact sum 1 + 63 * 2^-25, exact in fp64; an fp32 running sum would
    stay at 1), column b holds 1 + 2^-23 and zeros: a outranks b only with the fp64 sum."""
    T = 64
    I = np.zeros((T, 4), dtype=np.float32)
    I[0, 0] = 1.0
    I[1:, 0] = np.float32(2.0 ** -25)
    I[0, 1] = np.float32(1.0 + 2.0 ** -23)
    I[:, 2] = np.float32(2.0 ** -30)
    V = O.vector_scores(I, np.arange(4, dtype=np.int32), T)
    assert Fraction(float(V[0, 0])) == 1 + 63 * Fraction(1, 2 ** 25)
    assert float(V[0, 1]) == 1.0 + 2.0 ** -23
    np.testing.assert_array_equal(O.vector_order(V[0]), [0, 1, 2, 3])


def test_importance_exact_rational():
    rng = np.random.default_rng(3)
    M, K, N = 5, 6, 9
    W = bf(rng.normal(0, 0.3, (M, K)))
    X = bf(rng.normal(0, 1.0, (K, N)))
    I = O.importance(W, X)
    for c in range(K):
        exact = sum(Fraction(float(x)) ** 2 for x in f32(X[c]))
        s32 = np.float32(float(exact))          # tiny sums are exact in fp64
        for i in range(M):
            w = Fraction(float(f32(W[i, c])))
            want = np.float32(float(w * w * Fraction(float(s32))))
            assert I[i, c] == want


# ----------------------------------------------------------------------------- counts
def test_closed_form_triples(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "closed_form_boundaries.json")))
    for tr in g["triples"]:
        assert O.partial_sparsity(tr["t_s"], tr["v_s"]) == pytest.approx(tr["p_s"], abs=1e-12)
        # and the forward form t_s = v_s + (1 - v_s) p_s / 2
        assert tr["v_s"] + (1 - tr["v_s"]) * tr["p_s"] * 0.5 == pytest.approx(tr["t_s"], abs=1e-12)
    assert len(O.LEGAL_NIBBLES) == g["patterns_per_group_of_4"] == math.comb(4, 2)


@pytest.mark.parametrize("K,t_s,v_s,want", [
    (256, 0.5, 0.2, (52, 152, 52)),
    (4096, 0.5, 0.0, (0, 4096, 0)),
    (4096, 0.75, 0.6, (2458, 1228, 410)),
    (11008, 0.625, 0.4, (4404, 4952, 1652)),
    (4096, 0.5, 0.5, (2048, 0, 2048)),      # p_s = 0: pure column pruning
    (4096, 0.0, 0.0, (0, 0, 4096)),         # dense
    (4096, 1.0, 1.0, (4096, 0, 0)),         # everything pruned
    # the rounding of the group count (R5): 2 (t_s - v_s) K / 4 = 24.5 groups, exactly
    # representable, rounds up to 25 (a truncation would give 24)
    (196, 0.5, 0.25, (48, 100, 48)),
    # t_s - v_s = 0.625 - 0.4 is 0.22499999999999998 in binary64, so the count is just
    # below 22.5 groups and rounds to 22 (R5: evaluated in double, left to right)
    (200, 0.625, 0.4, (81, 88, 31)),
])
def test_counts_table(K, t_s, v_s, want):
    assert O.counts_from_vs(K, t_s, v_s) == want


def test_counts_invariants():
    for K in (64, 100, 256, 1000, 4096, 11008):
        for t_s in (0.5, 0.625, 0.75, 0.875):
            if t_s * K != int(t_s * K):
                continue
            for m in range(0, 40):
                v_s = t_s - m / 32.0
                if v_s < max(0.0, 2 * t_s - 1):
                    break
                try:
                    n0, n24, n4 = O.counts_from_vs(K, t_s, v_s)
                except ValueError:
                    continue
                assert n0 + n24 + n4 == K
                assert n24 % 4 == 0
                # overall sparsity is exactly t_s: kept = n4 + n24/2 = (1 - t_s) K
                assert n4 * 2 + n24 == 2 * K - 2 * int(t_s * K)
                if v_s < 1:
                    p_s = O.partial_sparsity(t_s, v_s)
                    assert abs(n24 - p_s * (K - n0)) <= 4


def test_counts_rejects():
    with pytest.raises(ValueError):
        O.counts_from_vs(100, 0.333, 0.1)       # t_s K not whole
    with pytest.raises(ValueError):
        O.counts_from_vs(256, 0.75, 0.3)        # v_s < 2 t_s - 1 -> n_4 < 0


def test_search_candidates_span():
    c = O.search_candidates(4096, 0.75, 1 / 32)
    assert len(c) == 9 and c[0] == (3072, 0, 1024) and c[-1] == (2048, 2048, 0)
    c = O.search_candidates(4096, 0.5, 1 / 32)
    assert len(c) == 17 and c[-1] == (0, 4096, 0)
    c = O.search_candidates(11008, 0.625, 1 / 32)
    assert len(c) == 13


# ----------------------------------------------------------------------------- 2:4 selection
def brute_pair(v):
    """Max-sum pair over all C(4,2) pairs, exact sums, ties -> lexicographically smallest."""
    best = None
    for a, b in itertools.combinations(range(4), 2):
        s = Fraction(float(v[a])) + Fraction(float(v[b]))
        if best is None or s > best[0]:
            best = (s, (a, b))
    return best[1]


def test_top2_matches_brute_force_all_ties():
    for v in itertools.product([0.0, 1.0, 2.0], repeat=4):
        keep = O.top2_keep(np.array(v, dtype=np.float32))
        assert keep.sum() == 2
        assert tuple(np.nonzero(keep)[0]) == brute_pair(v)


def test_top2_matches_brute_force_random():
    rng = np.random.default_rng(11)
    vals = rng.random((5000, 4)).astype(np.float32) ** 3
    keep = O.top2_keep(vals)
    assert (keep.sum(axis=1) == 2).all()
    for r in range(vals.shape[0]):
        assert tuple(np.nonzero(keep[r])[0]) == brute_pair(vals[r])


def test_magnitude_24_special_case():
    """X = 1: I = w^2 N, and with v_s = 0 (all vectors 2:4) and the identity order the
    mask is plain magnitude 2:4 along the input dimension (rkmt.cn, section 二)."""
    rng = np.random.default_rng(5)
    M, K, N, T = 8, 32, 4, 8
    W = bf(rng.normal(0, 1, (M, K)))
    Wf = f32(W)
    # distinct magnitudes in every group, so no tie rule is involved
    for i in range(M):
        for g in range(K // 4):
            assert len(set(np.abs(Wf[i, 4 * g:4 * g + 4]).tolist())) == 4
    X = bf(np.ones((K, N)))
    I = O.importance(W, X)
    counts = np.tile(np.array(O.counts_from_vs(K, 0.5, 0.0)), (M // T, 1))
    bm, region = O.mask(I, np.arange(K, dtype=np.int32), T, counts)
    keep = O.unpack_bits(bm, K)
    want = np.zeros((M, K), dtype=bool)
    for i in range(M):
        for g in range(K // 4):
            top = np.argsort(-np.abs(Wf[i, 4 * g:4 * g + 4]))[:2]
            want[i, 4 * g + top] = True
    assert np.array_equal(keep, want)
    assert (region == O.REGION_24).all()


def test_column_pruning_special_case():
    """v_s = t_s (p_s = 0): HiNM reduces to whole-column pruning of the lowest vectors."""
    rng = np.random.default_rng(8)
    M, K, N, T = 16, 24, 5, 8
    W = bf(rng.normal(0, 1, (M, K)))
    X = bf(rng.normal(0, 1, (K, N)))
    perm = rng.permutation(K).astype(np.int32)
    I = O.importance(W, X)
    counts = np.tile(np.array(O.counts_from_vs(K, 0.5, 0.5)), (M // T, 1))
    bm, region = O.mask(I, perm, T, counts)
    keep = O.unpack_bits(bm, K)
    Id = I.astype(np.float64)
    for t in range(M // T):
        # independent: sum each channel's importance over the tile, keep the top half
        score = {c: sum(float(Id[t * T + i, c]) for i in range(T)) for c in range(K)}
        pos = {int(c): j for j, c in enumerate(perm)}
        kept = sorted(range(K), key=lambda c: (-score[c], pos[c]))[:K // 2]
        want = np.zeros(K, dtype=bool)
        want[kept] = True
        for i in range(T):
            assert np.array_equal(keep[t * T + i], want)
        assert set(np.nonzero(region[t] == O.REGION_DENSE)[0]) == set(kept)


def test_structured_pruning_golden(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "structured_pruning_3x3.json")))
    W = bf(g["W"])
    # column pruning: the mask drops column 1 entirely
    keep = np.ones((3, 3), dtype=bool)
    keep[:, g["pruned_column"]] = False
    got = O.masked_weight(W, O.pack_bits(keep))
    np.testing.assert_allclose(got, f32(bf(g["W_pruned_col"])), rtol=0, atol=0)
    # row pruning
    keep = np.ones((3, 3), dtype=bool)
    keep[g["pruned_row"], :] = False
    np.testing.assert_allclose(O.masked_weight(W, O.pack_bits(keep)), f32(bf(g["W_pruned_row"])),
                               rtol=0, atol=0)
    # unstructured magnitude pruning at the printed threshold
    keep = np.abs(f32(W)) > g["threshold"]
    np.testing.assert_allclose(O.masked_weight(W, O.pack_bits(keep)),
                               f32(bf(g["W_pruned_threshold"])), rtol=0, atol=0)


# ----------------------------------------------------------------------------- search
def exact_R(I_tile_w, keep):
    return sum((Fraction(float(v)) for v in I_tile_w[keep].astype(np.float64)), Fraction(0))


def test_fsum_is_exactly_rounded():
    rng = np.random.default_rng(1)
    for _ in range(200):
        vals = (rng.random(50) * 2.0 ** rng.integers(-40, 40, 50)).astype(np.float32).astype(np.float64)
        ex = sum((Fraction(v) for v in vals), Fraction(0))
        assert math.fsum(vals.tolist()) == float(ex)
    vals = [2.0 ** 60] + [1.0] * 1000
    assert math.fsum(vals) == float(sum(Fraction(v) for v in vals))


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_search_brute_force(seed):
    rng = np.random.default_rng(seed)
    M, K, N, T = 16, 64, 6, 8
    W = bf(rng.normal(0, 1, (M, K)) * rng.random(K) ** 4)      # uneven column magnitudes
    X = bf(rng.normal(0, 1, (K, N)))
    perm = rng.permutation(K).astype(np.int32)
    I = O.importance(W, X)
    sr = O.boundary_search(I, perm, T, 0.5, 1 / 32)
    cands = O.search_candidates(K, 0.5, 1 / 32)
    for t in range(M // T):
        I_tile_w = I[t * T:(t + 1) * T][:, perm]
        # independent ranking of working positions by exact tile sums
        sums = [sum(Fraction(float(I_tile_w[i, j])) for i in range(T)) for j in range(K)]
        order = sorted(range(K), key=lambda j: (-sums[j], j))
        R = []
        for (n0, n24, n4) in cands:
            keep = np.zeros((T, K), dtype=bool)
            dense = order[:n4]
            mid = sorted(order[n4:n4 + n24])
            keep[:, dense] = True
            for gi in range(0, len(mid), 4):
                grp = mid[gi:gi + 4]
                for i in range(T):
                    a, b = brute_pair([I_tile_w[i, j] for j in grp])
                    keep[i, grp[a]] = keep[i, grp[b]] = True
            R.append(exact_R(I_tile_w, keep))
        assert [float(r) for r in R] == sr.R[t]
        first_drop = next((m for m in range(len(R) - 1) if float(R[m + 1]) < float(R[m])),
                          len(R) - 1)
        assert sr.m[t] == first_drop
        assert tuple(sr.counts[t]) == cands[first_drop]
        assert sr.v_s[t] == 0.5 - first_drop / 32
        total = sum(Fraction(float(v)) for v in I_tile_w.ravel())
        assert all(r <= total for r in R)


def test_search_first_drop_hand_built():
    """Hand-built tile (K = 64, t_s = 0.5, alpha = 1/32, X = 1, |w| constant per column).

    Column magnitudes by working position: 0..27 -> 8, 28..29 -> 3, 30..31 -> 2.875,
    32..33 -> 1.25, 34..35 -> 1, 36..63 -> 0.5 (so rank == position).
      m=0: dense 0..31                       R0 = 28*64 + 2*9 + 2*8.265625
      m=1: dense 0..29, 2:4 {30..33}         keeps 30,31 -> R1 == R0 (no strict drop)
      m=2: dense 0..27, 2:4 {28..31},{32..35} keeps 28,29 and 32,33 -> R2 < R1
    so the scan stops at m = 1 (v_s = 0.5 - 1/32).  Moving from m=0 to m=1 can never lose
    importance (the band's per-row top-2 includes the two vectors that left the dense
    region); only regrouping at m >= 1 can."""
    K, N, T = 64, 4, 8
    mags = np.array([8.0] * 28 + [3.0] * 2 + [2.875] * 2 + [1.25] * 2 + [1.0] * 2 + [0.5] * 28)
    signs = np.where(np.random.default_rng(0).random((T, K)) < 0.5, -1.0, 1.0)
    W = bf(signs * mags[None, :])
    X = bf(np.ones((K, N)))
    I = O.importance(W, X)
    sr = O.boundary_search(I, np.arange(K, dtype=np.int32), T, 0.5, 1 / 32)
    R = sr.R[0]
    unit = T * N
    assert R[0] == unit * (28 * 64 + 2 * 9 + 2 * 8.265625)
    assert R[1] == R[0]
    assert R[2] == unit * (28 * 64 + 2 * 9 + 2 * 1.5625)
    assert sr.m[0] == 1 and sr.v_s[0] == 0.5 - 1 / 32
    assert tuple(sr.counts[0]) == (30, 4, 30)


def test_search_runs_to_end_gaussian():
    """Gaussian weights: 2:4 keeps more importance than column pruning, R rises all the
    way and the scan ends at v_s = max(0, 2 t_s - 1)."""
    w = hi.custom(256, 256, 16, 64, seed=0, t_s=0.5, v_s=None)
    I = O.importance(w.W_bits, w.X_bits)
    sr = O.boundary_search(I, w.perm, 64, 0.5, 1 / 32)
    assert (sr.m == 16).all() and (sr.v_s == 0.0).all()
    for R in sr.R:
        assert all(R[m + 1] >= R[m] for m in range(len(R) - 1))


# ----------------------------------------------------------------------------- mask
@pytest.mark.parametrize("T", [64, 128])
def test_mask_counts_invariants(T):
    w = hi.custom(2 * T, 200, 8, T, seed=9, t_s=0.625, v_s=0.4, random_perm=True)
    I = O.importance(w.W_bits, w.X_bits)
    counts = np.tile(np.array(O.counts_from_vs(200, 0.625, 0.4)), (2, 1))
    bm, region = O.mask(I, w.perm, T, counts)
    keep = O.unpack_bits(bm, 200)
    n0, n24, n4 = counts[0]
    assert keep.sum() == (1 - 0.625) * 2 * T * 200
    assert (bm[:, -1] >> np.uint32(200 % 32) == 0).all()      # bits past K are zero
    for t in range(2):
        reg_w = region[t][w.perm]
        assert (reg_w == O.REGION_DENSE).sum() == n4 and (reg_w == O.REGION_24).sum() == n24
        kt = keep[t * T:(t + 1) * T][:, w.perm]
        assert kt[:, reg_w == O.REGION_DENSE].all()
        assert not kt[:, reg_w == O.REGION_PRUNED].any()
        g = O.groups_24(reg_w)
        assert (kt[:, g].sum(axis=-1) == 2).all()


def test_permutation_invariance():
    """Reordering input channels consistently does not change the computation
    (FlexHiNM-GP notes, 关键设计 2): run(W, X, pi) == run(W[:, pi], X[pi, :], id)."""
    w = hi.custom(128, 192, 24, 64, seed=12, t_s=0.625, v_s=None, random_perm=True)
    a = O.hot_path(w.W_bits, w.X_bits, w.perm, 64, 0.625)
    Wp = np.ascontiguousarray(w.W_bits[:, w.perm])
    Xp = np.ascontiguousarray(w.X_bits[w.perm, :])
    b = O.hot_path(Wp, Xp, np.arange(192, dtype=np.int32), 64, 0.625)
    assert np.array_equal(a["counts"], b["counts"])
    ka = O.unpack_bits(a["bitmask"], 192)
    kb = O.unpack_bits(b["bitmask"], 192)
    assert np.array_equal(ka[:, w.perm], kb)
    La, Lb = a["layout"], b["layout"]
    assert np.array_equal(La.vals_dense, Lb.vals_dense)
    assert np.array_equal(La.vals_sparse, Lb.vals_sparse)
    assert np.array_equal(La.meta, Lb.meta)
    assert np.array_equal(La.tile_info, Lb.tile_info)
    # idx_a = pi[idx_b] on real entries (padding is 0 on both sides)
    for ia, ib in ((La.idx_dense, Lb.idx_dense), (La.idx_sparse, Lb.idx_sparse)):
        real = ~((ia == 0) & (ib == 0))
        assert np.array_equal(ia[real], w.perm[ib[real]])
    assert np.array_equal(a["y"], b["y"])


def test_tile_permutation_permutes_rows():
    w = hi.custom(192, 128, 8, 64, seed=21, t_s=0.5, v_s=0.25)
    a = O.hot_path(w.W_bits, w.X_bits, w.perm, 64, 0.5, v_s=0.25)
    order = [2, 0, 1]
    rows = np.concatenate([np.arange(t * 64, (t + 1) * 64) for t in order])
    b = O.hot_path(np.ascontiguousarray(w.W_bits[rows]), w.X_bits, w.perm, 64, 0.5, v_s=0.25)
    assert np.array_equal(a["y"][rows], b["y"])
    assert np.array_equal(a["bitmask"][rows], b["bitmask"])


# ----------------------------------------------------------------------------- layout
def test_swizzle_and_meta_bijections():
    offs = {O.swizzled_offset(r, k) for r in range(128) for k in range(64)}
    assert offs == set(range(0, 16384, 2))
    slots = {O.meta_word_index(m, g) for m in range(128) for g in range(32)}
    assert slots == {(w, 4 * n) for w in range(512) for n in range(8)}


def test_layout_worked_examples():
    """Positions worked by hand from the layout's definitions (a bijection test alone would
    pass a consistent mistake in both the writer and the reader).

    Values: rows are 128 bytes apart, and the 16-byte chunk of column k of row r sits at
    chunk (k // 8) XOR (r mod 8), the 128-byte swizzle.  Metadata: word w of lane L, bits
    [16 s + 4 q, +4), holds group 8 w + 4 ((L // 8) mod 2) + q of row
    16 (L // 16) + 8 s + (L mod 8)."""
    # (r, k) -> byte offset
    for (r, k), off in {(0, 0): 0, (0, 9): 16 + 2, (1, 0): 128 + 16, (1, 8): 128 + 0,
                        (3, 17): 3 * 128 + (2 ^ 3) * 16 + 2,
                        (7, 63): 7 * 128 + 0 + 7 * 2}.items():
        assert O.swizzled_offset(r, k) == off, (r, k)
    # (row m, group g) -> (lane * 4 + word, bit shift)
    for (m, g), slot in {(0, 0): (0, 0),            # lane 0, word 0, s = 0, q = 0
                         (0, 1): (0, 4),            # q = 1
                         (1, 4): (9 * 4, 0),        # group 4 is in lane half h = 1: lane 8 + 1
                         (8, 0): (0, 16),           # row 8 is s = 1 of lane 0
                         (9, 13): (9 * 4 + 1, 20),  # word 1, h = 1, q = 1; s = 1, lane 9
                         (16, 0): (16 * 4, 0),      # rows 16.. are lanes 16..
                         (5, 9): (5 * 4 + 1, 4),    # word 1, h = 0, q = 1
                         (127, 31): (127 * 4 + 3, 28)}.items():
        assert O.meta_word_index(m, g) == slot, (m, g)


@pytest.mark.parametrize("perm", [False, True], ids=["identity", "permuted"])
def test_all_equal_importances_follow_the_tie_rules(perm):
    """Every importance equal (W = X = 1): every vector score ties, so the ranking is the
    working order (R4: the lower working position ranks higher) -- the first n_4 working
    positions dense, the next n_24 in 2:4, the rest pruned -- and in every 2:4 group every
    row keeps its first two members (R7: equal values, the lower position wins)."""
    T, K, N = 64, 64, 8
    W = bf(np.ones((2 * T, K)))
    X = bf(np.ones((K, N)))
    p = np.random.default_rng(4).permutation(K).astype(np.int32) if perm else np.arange(K, dtype=np.int32)
    n0, n24, n4 = O.counts_from_vs(K, 0.5, 0.25)
    I = O.importance(W, X)
    sr = O.boundary_search(I, p, T, 0.5, 1 / 32)
    for t in range(2):
        np.testing.assert_array_equal(sr.rank[t], np.arange(K))
    counts = np.tile(np.array([n0, n24, n4], dtype=np.int32), (2, 1))
    bm, reg = O.mask(I, p, T, counts)
    keep = O.unpack_bits(bm, K)
    for t in range(2):
        want_reg = np.empty(K, dtype=np.int8)
        want_keep = np.zeros(K, dtype=bool)
        for j in range(K):
            c = p[j]
            if j < n4:
                want_reg[c], want_keep[c] = O.REGION_DENSE, True
            elif j < n4 + n24:
                want_reg[c], want_keep[c] = O.REGION_24, (j - n4) % 4 < 2
            else:
                want_reg[c] = O.REGION_PRUNED
        np.testing.assert_array_equal(reg[t], want_reg)
        for r in range(t * T, (t + 1) * T):
            np.testing.assert_array_equal(keep[r], want_keep)


@pytest.mark.parametrize("T,K,t_s,v_s,perm", [
    (64, 256, 0.5, 0.2, False), (128, 200, 0.625, 0.4, True), (64, 96, 0.75, 0.5, True)])
def test_compress_round_trip(T, K, t_s, v_s, perm):
    w = hi.custom(2 * T, K, 8, T, seed=3, t_s=t_s, v_s=v_s, random_perm=perm)
    I = O.importance(w.W_bits, w.X_bits)
    counts = np.tile(np.array(O.counts_from_vs(K, t_s, v_s)), (2, 1))
    bm, region = O.mask(I, w.perm, T, counts)
    L = O.compress(w.W_bits, bm, region, w.perm, counts, T)
    np.testing.assert_array_equal(L.tile_info[:, 0], -(-counts[:, 2] // 64))
    np.testing.assert_array_equal(L.tile_info[:, 1], -(-counts[:, 1] // 128))
    Wm = O.masked_weight(w.W_bits, bm).astype(np.float32)
    np.testing.assert_array_equal(O.decompress(L), Wm)
    nib = (L.meta[:, :, None] >> (4 * np.arange(8, dtype=np.uint32))) & np.uint32(0xF)
    assert set(np.unique(nib).tolist()) <= set(O.LEGAL_NIBBLES)
    n0, n24, n4 = counts[0]
    # padded index entries are 0; real entries are distinct channels of the right region
    for t in range(2):
        nd, ns, d0, s0 = L.tile_info[t]
        dense_idx = L.idx_dense[d0:d0 + nd].ravel()[:n4]
        assert set(dense_idx.tolist()) == set(np.nonzero(region[t] == O.REGION_DENSE)[0].tolist())
        assert (L.idx_dense[d0:d0 + nd].ravel()[n4:] == 0).all()
        sp_idx = L.idx_sparse[s0:s0 + ns].ravel()[:n24]
        assert set(sp_idx.tolist()) == set(np.nonzero(region[t] == O.REGION_24)[0].tolist())
    # contiguous-run flags: a block is flagged iff its indices are one ascending run
    for idx, run in ((L.idx_dense, L.run_dense), (L.idx_sparse, L.run_sparse)):
        for b in range(idx.shape[0]):
            is_run = all(int(idx[b, v]) == int(idx[b, 0]) + v for v in range(idx.shape[1]))
            assert run[b] == (idx[b, 0] if is_run else -1)


def test_contiguous_runs_identity_pure24():
    """Pure 2:4 with the identity order: every 2:4 block is one run of 128 channels."""
    w = hi.custom(128, 256, 8, 128, seed=1, t_s=0.5, v_s=None)
    I = O.importance(w.W_bits, w.X_bits)
    counts = np.array([O.counts_from_vs(256, 0.5, 0.0)])
    bm, region = O.mask(I, w.perm, 128, counts)
    L = O.compress(w.W_bits, bm, region, w.perm, counts, 128)
    np.testing.assert_array_equal(L.run_sparse, [0, 128])


# ----------------------------------------------------------------------------- index translation
def _layout_fields_equal(A, B):
    for f in ("tile_info", "vals_dense", "vals_sparse", "meta", "idx_dense", "idx_sparse",
              "run_dense", "run_sparse"):
        np.testing.assert_array_equal(getattr(A, f), getattr(B, f), err_msg=f)


@pytest.mark.parametrize("v_s,perm", [(0.25, True), (0.0, False), (0.5, False)])
def test_translate_index_pins(v_s, perm):
    """The cross-layer index translation ([P1] 关键设计 2): (i) the identity row map leaves
    the layout unchanged (its run flags included: the recomputation is compress's rule);
    (ii) translations compose, translate(translate(L, a), b) == translate(L, b[a]); (iii)
    the translated layout times X with its rows reordered equals the original product
    exactly (integer data, so the fp64 sums are exact), through decompress, itself pinned
    by the round trip above."""
    T, K = 64, 256
    w = hi.integer_workload(2 * T, K, 8, T, seed=7, t_s=0.5, v_s=v_s, random_perm=perm)
    I = O.importance(w.W_bits, w.X_bits)
    counts = np.tile(np.array(O.counts_from_vs(K, 0.5, v_s)), (2, 1))
    bm, region = O.mask(I, w.perm, T, counts)
    L = O.compress(w.W_bits, bm, region, w.perm, counts, T)
    _layout_fields_equal(O.translate_index(L, np.arange(K)), L)
    rng = np.random.default_rng(11)
    a, b = rng.permutation(K), rng.permutation(K)
    _layout_fields_equal(O.translate_index(O.translate_index(L, a), b), O.translate_index(L, b[a]))
    sigma = rng.permutation(K)                 # delivered row r holds channel sigma[r]
    row_of_channel = np.argsort(sigma)         # sigma^-1
    Lt = O.translate_index(L, row_of_channel)
    X = f32(w.X_bits).astype(np.float64)
    X_del = X[sigma]
    y = O.decompress(L).astype(np.float64) @ X
    y_t = O.decompress(Lt).astype(np.float64) @ X_del
    np.testing.assert_array_equal(y_t, y)
    # a reordered X generally breaks the runs: only blocks that stay ascending keep a flag
    for idx, run in ((Lt.idx_dense, Lt.run_dense), (Lt.idx_sparse, Lt.run_sparse)):
        for k in range(idx.shape[0]):
            ok = all(int(idx[k, v]) == int(idx[k, 0]) + v for v in range(idx.shape[1]))
            assert run[k] == (idx[k, 0] if ok else -1)


# ----------------------------------------------------------------------------- spmm reference
def test_spmm_identity_x_gives_masked_weight():
    w = hi.custom(128, 64, 64, 64, seed=2, t_s=0.5, v_s=0.25)
    I = O.importance(w.W_bits, w.X_bits)
    counts = np.tile(np.array(O.counts_from_vs(64, 0.5, 0.25)), (2, 1))
    bm, _ = O.mask(I, w.perm, 64, counts)
    eye = bf(np.eye(64))
    y, bound = O.spmm_reference(w.W_bits, bm, eye)
    np.testing.assert_array_equal(y, O.masked_weight(w.W_bits, bm))
    np.testing.assert_array_equal(bound, np.abs(O.masked_weight(w.W_bits, bm)))


def test_spmm_dense_case_triple_loop():
    """t_s = 0 keeps everything: y = W X, checked against a plain triple loop."""
    w = hi.custom(64, 16, 3, 64, seed=6, t_s=0.0, v_s=0.0)
    r = O.hot_path(w.W_bits, w.X_bits, w.perm, 64, 0.0, v_s=0.0)
    Wf, Xf = f32(w.W_bits).astype(np.float64), f32(w.X_bits).astype(np.float64)
    for i in range(64):
        for n in range(3):
            acc = Fraction(0)
            for c in range(16):
                acc += Fraction(float(Wf[i, c])) * Fraction(float(Xf[c, n]))
            assert abs(r["y"][i, n] - float(acc)) <= 1e-12 * max(1.0, abs(float(acc)))
    assert O.unpack_bits(r["bitmask"], 16).all()


def test_spmm_integer_exact():
    w = hi.integer_workload(128, 128, 16, 64, seed=1, t_s=0.5, v_s=0.25, random_perm=True)
    r = O.hot_path(w.W_bits, w.X_bits, w.perm, 64, 0.5, v_s=0.25)
    assert np.array_equal(r["y"], np.round(r["y"]))
    Wm = O.masked_weight(w.W_bits, r["bitmask"]).astype(np.int64)
    Xi = f32(w.X_bits).astype(np.int64)
    assert np.array_equal(r["y"].astype(np.int64), Wm @ Xi)


# ----------------------------------------------------------------------------- Hard-Concrete
def test_hard_concrete_closed_forms():
    """eps = 1/2 and log alpha = 0 give s = 1/2, z = 1/2; s = 1/12 and s = 11/12 sit exactly on
    the clip edges (z = 0, z = 1); large |log alpha| saturates to 0 / 1; the regularisers of
    a binary mask with two ones per group are (n/2, 0)."""
    tau = 2.0 / 3.0
    logit = lambda p: math.log(p / (1.0 - p))
    la = np.array([0.0, tau * logit(1 / 12), tau * logit(11 / 12), 60.0], dtype=np.float64)
    z, hard, sums = O.hard_concrete(la, np.full(4, 0.5), tau)
    # z[0] is 1/2 up to the fp64 rounding of the stretch (1.1 - (-0.1) is not exact), so its
    # hardening is a tie and is not asserted
    assert abs(z[0] - 0.5) < 1e-15
    assert abs(z[1]) < 1e-15 and abs(z[2] - 1.0) < 1e-15 and z[3] == 1.0
    np.testing.assert_array_equal(hard[1:], [0, 1, 1])
    z2, _, s2 = O.hard_concrete(np.array([50.0, -50.0, 50.0, -50.0] * 3), np.full(12, 0.5), tau)
    np.testing.assert_array_equal(z2, [1.0, 0.0] * 6)
    np.testing.assert_array_equal(s2, [6.0, 0.0])


def test_hard_concrete_noise_enters_as_log_eps_minus_log_one_minus_eps():
    """A worked value at an asymmetric noise draw: eps = 3/4, log alpha = 0, tau = 1 give
    the logit log 3, s = 3/4 and z = 1.2 * 3/4 - 0.1 = 0.8; eps = 1/4 gives s = 1/4 and
    z = 0.2.  (The mirror identity and the clip masses are symmetric in eps <-> 1 - eps,
    so they alone would not tell the two apart.)"""
    z, hard, _ = O.hard_concrete(np.zeros(4), np.array([0.75, 0.25, 0.75, 0.25]), 1.0)
    np.testing.assert_allclose(z, [0.8, 0.2, 0.8, 0.2], rtol=0, atol=1e-15)
    np.testing.assert_array_equal(hard, [1, 0, 1, 0])


def test_hard_concrete_mirror_and_regularisers():
    """Flipping both the noise and the logit mirrors the mask: z(eps, a) + z(1 - eps, -a) = 1
    (the logit changes sign, the stretch and the clip are symmetric about 1/2); the
    regularisers equal their loops written out."""
    rng = np.random.default_rng(3)
    la = rng.normal(0, 2, 4096)
    eps = rng.uniform(1e-6, 1 - 1e-6, 4096)
    z, hard, sums = O.hard_concrete(la, eps, 0.5)
    zm, _, _ = O.hard_concrete(-la, 1.0 - eps, 0.5)
    assert np.abs(z + zm - 1.0).max() < 1e-12
    want0 = math.fsum(z.tolist())
    want1 = math.fsum(abs(math.fsum(z[4 * g:4 * g + 4].tolist()) - 2.0) for g in range(1024))
    assert abs(sums[0] - want0) <= 1e-9 and abs(sums[1] - want1) <= 1e-9
    np.testing.assert_array_equal(hard, (z > 0.5).astype(np.uint8))


def test_hard_concrete_clip_mass_matches_the_logistic_law():
    """With eps uniform, log(eps) - log(1 - eps) is logistic (CDF sigmoid), so
    P(z = 0) = sigmoid(tau logit(1/12) - log alpha) and P(z = 1) = sigmoid(-tau logit(11/12)
    + log alpha).  On 2^20 seeded draws the empirical masses match within 5 standard
    deviations: this pins the sign of the noise and of log alpha and the stretch interval."""
    n, tau, la0 = 1 << 20, 2.0 / 3.0, 0.7
    rng = np.random.default_rng(9)
    eps = rng.uniform(0.0, 1.0, n)
    eps = np.clip(eps, 1e-12, 1 - 1e-12)
    z, _, _ = O.hard_concrete(np.full(n, la0), eps, tau)
    logit = lambda p: math.log(p / (1.0 - p))
    sig = lambda x: 1.0 / (1.0 + math.exp(-x))
    p0 = sig(tau * logit(1 / 12) - la0)
    p1 = sig(-tau * logit(11 / 12) + la0)
    for got, p in (((z == 0.0).mean(), p0), ((z == 1.0).mean(), p1)):
        assert abs(got - p) < 5 * math.sqrt(p * (1 - p) / n), (got, p)


# ----------------------------------------------------------------------------- SpMM epilogue
def test_activation_closed_forms_and_identities():
    """ReLU, SiLU, GELU: values at 0 and at known points, SiLU(x) - SiLU(-x) = x and
    GELU(x) - GELU(-x) = x (sigmoid(x) + sigmoid(-x) = 1, Phi(x) + Phi(-x) = 1), GELU(1) =
    Phi(1) = 0.8413447460685429..., SiLU(1) = 1 / (1 + e^-1)."""
    x = np.linspace(-6.0, 6.0, 241)
    np.testing.assert_array_equal(O.activation(x, O.ACT_NONE), x)
    np.testing.assert_array_equal(O.activation(x, O.ACT_RELU), np.where(x > 0, x, 0.0))
    for act in (O.ACT_SILU, O.ACT_GELU):
        d = O.activation(x, act) - O.activation(-x, act)
        assert np.abs(d - x).max() < 1e-14
        assert O.activation(np.array([0.0]), act)[0] == 0.0
    assert abs(O.activation(np.array([1.0]), O.ACT_GELU)[0] - 0.8413447460685429) < 1e-15
    assert abs(O.activation(np.array([1.0]), O.ACT_SILU)[0] - 1.0 / (1.0 + math.exp(-1.0))) < 1e-15


def test_epilogue_reference_bias_per_row():
    """The bias is added per output row (output channel) before the activation."""
    y = np.arange(12, dtype=np.float64).reshape(3, 4) - 5.0
    b = np.array([1.0, -2.0, 0.5])
    got = O.spmm_epilogue_reference(y, b, O.ACT_RELU)
    np.testing.assert_array_equal(got, np.maximum(y + b[:, None], 0.0))
    np.testing.assert_array_equal(O.spmm_epilogue_reference(y, None, O.ACT_NONE), y)


# ----------------------------------------------------------------------------- gyro-permutation
def test_group_cost_and_retained_hand_example():
    """Two rows whose top-2 differ: row 0 (9, 8, 7, 1) keeps 9 + 8 and prunes 7 + 1; row 1
    (1, 2, 9, 8) keeps 9 + 8 and prunes 1 + 2.  Retained 17 + 17 = 34, pruned 8 + 3 = 11,
    and together they are the group's whole importance (45)."""
    I_tile = np.array([[9, 8, 7, 1], [1, 2, 9, 8]], dtype=np.float32)
    assert O.group_retained(I_tile, [0, 1, 2, 3]) == 34.0
    assert O.group_pruning_cost(I_tile, [0, 1, 2, 3]) == 11.0
    # member order does not matter; a different grouping of the same channels changes both
    assert O.group_pruning_cost(I_tile, [3, 1, 0, 2]) == 11.0
    I2 = np.array([[9, 8, 7, 1, 6, 5, 4, 3], [1, 2, 9, 8, 3, 4, 5, 6]], dtype=np.float32)
    assert O.group_pruning_cost(I2, [4, 5, 6, 7]) == 7.0 + 7.0   # (4 + 3), (3 + 4)
    assert O.band_pruning_cost(I2, np.arange(8)) == 11.0 + 14.0


def _brute_balanced_partitions(S, k):
    """Every partition of range(S) into S/k unordered blocks of size k."""
    def rec(rest):
        if not rest:
            yield []
            return
        first = rest[0]
        import itertools
        for comb in itertools.combinations(rest[1:], k - 1):
            block = [first, *comb]
            left = [x for x in rest if x not in block]
            for tail in rec(left):
                yield [block, *tail]
    yield from rec(list(range(S)))


def test_balanced_kmeans_regroups_planted_pairs():
    """Points 0, 0.1 | 10, 5 | 5.1, 10.1 seeded as those three pairs: the seeds' centroids
    are 0.05, 7.5 and 7.6; the best balanced assignment to them (worked out by hand:
    {5, 5.1} -> 7.5 and {10, 10.1} -> 7.6 cost 24.02 against 25 for the seeds) regroups the
    planted pairs {5, 5.1} and {10, 10.1}, which is then a fixed point; every cluster keeps
    exactly k = 2 points."""
    F = np.array([[0.0], [0.1], [10.0], [5.0], [5.1], [10.1]])
    cl = O.balanced_kmeans(F, 2, 10)
    assert cl == [[0, 1], [3, 4], [2, 5]]
    assert O.balanced_kmeans(F, 2, 0) == [[0, 1], [2, 3], [4, 5]]   # no iteration: the seeds


def test_balanced_kmeans_fixed_point_brute_force():
    """The result is a fixed point of the balanced iteration: with the result's centroids,
    no balanced partition (all 15 of 6 points into pairs, enumerated) has a smaller total
    squared distance; and the within-cluster sum of squares does not rise from the seed
    partition to the result."""
    rng = np.random.default_rng(4)
    for trial in range(20):
        F = rng.normal(size=(6, 3))
        cl = O.balanced_kmeans(F, 2, 20)
        C = [F[c].mean(axis=0) for c in cl]

        def assign_cost(part):
            # best matching of the blocks to the centroids (3! ways), squared distances
            import itertools
            best = None
            for p in itertools.permutations(range(3)):
                v = sum(((F[b] - C[p[i]]) ** 2).sum() for i, blk in enumerate(part) for b in blk)
                best = v if best is None else min(best, v)
            return best
        mine = sum(((F[b] - C[i]) ** 2).sum() for i, c in enumerate(cl) for b in c)
        assert mine <= min(assign_cost(p) for p in _brute_balanced_partitions(6, 2)) + 1e-12
        seed = [[0, 1], [2, 3], [4, 5]]
        sse = lambda part: sum(((F[c] - F[c].mean(axis=0)) ** 2).sum() for c in part)
        assert sse(cl) <= sse(seed) + 1e-12


def test_gyro_input_round_k1_hand_example():
    """k = 1 (every cluster one vector): tile row [9 8 7 1 | 6 5 4 3], sampling the 7 (group 0,
    slot 2) and the 3 (group 1, slot 3): swapping them prunes 3 + 1 and 6 + 5 ... the
    cheaper of the two assignments: cost 8 + 7 = 15 before, 4 + 9 = 13 after."""
    I_tile = np.array([[9, 8, 7, 1, 6, 5, 4, 3]], dtype=np.float32)
    out, (before, after) = O.gyro_input_round(I_tile, np.arange(8), [0, 1], [[2], [3]])
    assert (before, after) == (15.0, 13.0)
    np.testing.assert_array_equal(out, [0, 1, 7, 3, 4, 5, 6, 2])


def test_gyro_input_round_brute_force_and_invariants():
    """k = 2, G = 3: the chosen placement of the clusters costs the least of all 3! (costs
    recomputed here from sorted rows); the band stays a permutation of its channels, the
    unsampled groups keep their members, and over rounds the band's pruning cost never rises."""
    import itertools
    rng = np.random.default_rng(21)
    T, K = 12, 48
    I_tile = rng.exponential(1.0, (T, K)).astype(np.float32)
    band = rng.permutation(K)[:40]                      # 10 groups
    groups, slots = [2, 5, 8], [[0, 3], [1, 2], [0, 1]]
    out, (before, after) = O.gyro_input_round(I_tile, band, groups, slots)
    vecs = [int(band[4 * g + s]) for g, ss in zip(groups, slots) for s in ss]
    F = I_tile[:, vecs].T.astype(np.float64)
    clusters = O.balanced_kmeans(F, 2, 8)

    def cost(members):  # the two smallest per row, rows ascending
        acc = 0.0
        for r in range(T):
            v = np.sort(I_tile[r, members].astype(np.float64))
            acc += v[1] + v[0]
        return acc

    def members_with(i, cl):
        m = [int(x) for x in band[4 * groups[i]:4 * groups[i] + 4]]
        for s, p in zip(sorted(slots[i]), cl):
            m[s] = vecs[p]
        return m
    best = min(sum(cost(members_with(i, clusters[p[i]])) for i in range(3))
               for p in itertools.permutations(range(3)))
    assert abs(min(after, before) - min(best, before)) <= 1e-9 * before
    assert sorted(out.tolist()) == sorted(band.tolist())
    for g in set(range(10)) - set(groups):
        np.testing.assert_array_equal(out[4 * g:4 * g + 4], band[4 * g:4 * g + 4])
    b = band.copy()
    costs = [O.band_pruning_cost(I_tile, b)]
    for it in range(4):
        gs = rng.choice(10, 4, replace=False)
        ss = [sorted(rng.choice(4, 2, replace=False)) for _ in gs]
        b, _ = O.gyro_input_round(I_tile, b, gs, ss)
        costs.append(O.band_pruning_cost(I_tile, b))
    assert all(c1 <= c0 + 1e-9 * c0 for c0, c1 in zip(costs, costs[1:]))


def test_tile_perm_with_band():
    perm_t = np.array([5, 0, 3, 1, 4, 2])
    region_t = np.array([1, 2, 0, 1, 1, 1], dtype=np.int8)   # by channel
    # 2:4 channels in working order: 5, 0, 3, 4 at positions 0, 1, 2, 4 (1 dense, 2 pruned)
    out = O.tile_perm_with_band(perm_t, region_t, [4, 3, 0, 5])
    np.testing.assert_array_equal(out, [4, 3, 0, 1, 5, 2])


def test_column_pruning_cost_hand_example():
    """Rows [1 5 2 9], [2 1 2 0]: scores 3 6 4 9; the two smallest (3 + 4) = 7."""
    I_rows = np.array([[1, 5, 2, 9], [2, 1, 2, 0]], dtype=np.float32)
    assert O.column_pruning_cost(I_rows, 2) == 7.0
    assert O.column_pruning_cost(I_rows, 0) == 0.0


def test_gyro_output_round_brute_force_and_invariants():
    """G = 3 tiles, k = 1 row each: the chosen placement costs the least of all 3!; the row
    order stays a permutation; unsampled tiles keep their rows; rounds never raise the cost."""
    import itertools
    rng = np.random.default_rng(8)
    T, K, nt = 4, 16, 5
    I = rng.exponential(1.0, (nt * T, K)).astype(np.float32)
    n0 = np.array([5, 6, 4, 7, 5])
    order = rng.permutation(nt * T)
    tiles, rows = [0, 2, 4], [[1], [3], [0]]
    out, (before, after) = O.gyro_output_round(I, T, n0, order, tiles, rows)
    chans = [int(order[t * T + r[0]]) for t, r in zip(tiles, rows)]

    def cpc(rows_, n):  # independent: sort the column sums
        V = np.sort(I[rows_].astype(np.float64).sum(axis=0))
        return float(V[:n].sum())

    def tile_with(i, ch):
        t = tiles[i]
        cur = [int(x) for x in order[t * T:(t + 1) * T]]
        cur[rows[i][0]] = ch
        return cur
    best = min(sum(cpc(tile_with(i, chans[p[i]]), n0[tiles[i]]) for i in range(3))
               for p in itertools.permutations(range(3)))
    assert abs(min(after, before) - min(best, before)) <= 1e-9 * before
    assert sorted(out.tolist()) == list(range(nt * T))
    for t in (1, 3):
        np.testing.assert_array_equal(out[t * T:(t + 1) * T], order[t * T:(t + 1) * T])
