"""Plausible mistakes planted in the CPU oracle, one at a time.

tests/test_oracle_mutations.py applies one mutant in a child process and runs the oracle's
pins (tests/test_oracle_pins.py) against it: every mutant must make at least one pin fail.
Each mutant replaces one oracle function (or an encoder and its decoder together, where a
consistent mistake would otherwise pass a round trip) with a copy that carries a single
change: a dropped term, a wrong sign, index or tie rule, a transposed operand, an
off-by-one.  Nothing here is imported by the oracle or the product.
"""
import math

import numpy as np

from oracle import hinm_oracle as O

_orig = {name: getattr(O, name) for name in dir(O) if callable(getattr(O, name))}


# ------------------------------------------------------------------------- importance
def _energy_drops_square(X_bits):
    X = O._bf16_to_f64(X_bits)
    acc = np.zeros(X.shape[0])
    for n in range(X.shape[1]):
        acc += X[:, n]
    return acc.astype(np.float32)


def _energy_over_wrong_axis(X_bits):
    X = O._bf16_to_f64(X_bits).T
    acc = np.zeros(X.shape[0])
    for n in range(X.shape[1]):
        acc += X[:, n] * X[:, n]
    return acc.astype(np.float32)


def _importance_w_not_squared(W_bits, X_bits, rows):
    W = O._bf16_to_f32(W_bits if rows is None else np.asarray(W_bits)[rows])
    s = O.channel_energy(X_bits)
    return (W * s[None, :]).astype(np.float32)


def _importance_rows_ignored(W_bits, X_bits, rows):
    return _orig["importance_rows"](W_bits, X_bits, None)


# ------------------------------------------------------------------ vector scores / rank
def _scores_skip_last_row(I, perm, T):
    M, K = I.shape
    nt = M // T
    if np.asarray(perm).ndim == 1:
        Iw = I[:, perm].reshape(nt, T, K)
    else:
        Iw = np.stack([I[t * T:(t + 1) * T][:, O.tile_perm(perm, t)] for t in range(nt)])
    V = np.zeros((nt, K))
    for i in range(T - 1):
        V += Iw[:, i, :].astype(np.float64)
    return V


def _order_ascending(V_t):
    return np.lexsort((np.arange(V_t.shape[0]), V_t))


def _order_ties_high_first(V_t):
    return np.lexsort((-np.arange(V_t.shape[0]), -V_t))


# --------------------------------------------------------------------------- counts
def _counts_truncates(K, t_s, v_s):
    x = 2.0 * (t_s - v_s) * K / 4.0
    n24 = 4 * int(math.floor(x))
    tk = t_s * K
    if tk != math.floor(tk):
        raise ValueError("t_s*K not whole")
    n0 = int(tk) - n24 // 2
    n4 = K - n0 - n24
    if n24 < 0 or n0 < 0 or n4 < 0:
        raise ValueError("negative count")
    return n0, n24, n4


def _counts_n0_full(K, t_s, v_s):
    x = 2.0 * (t_s - v_s) * K / 4.0
    n24 = 4 * int(math.floor(x + 0.5))
    tk = t_s * K
    if tk != math.floor(tk):
        raise ValueError("t_s*K not whole")
    n0 = int(tk) - n24
    n4 = K - n0 - n24
    if n24 < 0 or n0 < 0 or n4 < 0:
        raise ValueError("negative count")
    return n0, n24, n4


def _candidates_drop_last(K, t_s, alpha):
    return _orig["search_candidates"](K, t_s, alpha)[:-1] or _orig["search_candidates"](K, t_s, alpha)


# ------------------------------------------------------------------ regions and 2:4
def _regions_swapped(rank_t, counts):
    n0, n24, n4 = counts
    reg = np.full(rank_t.shape, O.REGION_PRUNED, dtype=np.int8)
    reg[rank_t < n4 + n24] = O.REGION_DENSE
    reg[rank_t < n4] = O.REGION_24
    return reg


def _groups_descending(region_w):
    pos = np.nonzero(region_w == O.REGION_24)[0][::-1]
    if pos.size % 4:
        raise ValueError("multiple of 4")
    return pos.reshape(-1, 4)


def _top2_ties_high(vals):
    v = vals[..., :, None]
    w = vals[..., None, :]
    kidx = np.arange(4)
    higher = kidx[None, :] > kidx[:, None]
    beats = (w > v) | ((w == v) & higher)
    return beats.sum(axis=-1) < 2


def _top2_keeps_smallest(vals):
    v = vals[..., :, None]
    w = vals[..., None, :]
    kidx = np.arange(4)
    lower = kidx[None, :] < kidx[:, None]
    beats = (w < v) | ((w == v) & lower)
    return beats.sum(axis=-1) < 2


def _retained_ignores_keep(I_tile_w, keep):
    return math.fsum(I_tile_w.astype(np.float64).ravel().tolist())


# ---------------------------------------------------------------------- search rule
def _search_with(rule):
    def search(I, perm, T, t_s, alpha, tiles=None):
        M, K = I.shape
        nt = M // T
        cands = O.search_candidates(K, t_s, alpha)
        counts = np.zeros((nt, 3), dtype=np.int32)
        vs = np.zeros(nt)
        ms = np.zeros(nt, dtype=np.int32)
        rank = np.zeros((nt, K), dtype=np.int32)
        Rs = [[] for _ in range(nt)]
        for t in (range(nt) if tiles is None else tiles):
            I_tile_w = I[t * T:(t + 1) * T][:, O.tile_perm(perm, t)]
            V_t = O.vector_scores(I[t * T:(t + 1) * T], O.tile_perm(perm, t), T)[0]
            order = O.vector_order(V_t)
            rank[t, order] = np.arange(K, dtype=np.int32)
            R = [O.retained_importance(I_tile_w, O.tile_mask_working(I_tile_w, O.regions_from_rank(rank[t], c)))
                 for c in cands]
            m_star = rule(R)
            counts[t] = cands[m_star]
            vs[t] = t_s - m_star * alpha
            ms[t] = m_star
            Rs[t] = R
        return O.SearchResult(counts=counts, v_s=vs, m=ms, R=Rs, rank=rank)
    return search


def _rule_nonstrict(R):
    for m in range(len(R) - 1):
        if R[m + 1] <= R[m]:
            return m
    return len(R) - 1


def _rule_one_past(R):
    for m in range(len(R) - 1):
        if R[m + 1] < R[m]:
            return m + 1
    return len(R) - 1


# ------------------------------------------------------------------------- layout
def _pack_msb_first(keep):
    """Bit b of word w holds column 32 w + 31 - b (the reader below agrees)."""
    return _orig["pack_bits"](_reverse_in_words(keep))


def _reverse_in_words(keep):
    R, K = keep.shape
    words = (K + 31) // 32
    padded = np.zeros((R, words * 32), dtype=bool)
    padded[:, :K] = keep
    return padded.reshape(R, words, 32)[:, :, ::-1].reshape(R, words * 32)


def _unpack_msb_first(bitmask, K):
    R, words = bitmask.shape
    full = _orig["unpack_bits"](bitmask, words * 32)
    return full.reshape(R, words, 32)[:, :, ::-1].reshape(R, words * 32)[:, :K]


def _swizzle_without_xor(r, k):
    return r * 128 + ((k >> 3) << 4) + (k & 7) * 2


def _meta_halves_swapped(m, g):
    w, rem = divmod(g, 8)
    h, q = divmod(rem, 4)
    s = (m >> 3) & 1
    L = (m & 7) + 8 * s + 16 * (m >> 4)
    return L * 4 + w, 16 * h + 4 * q


def _swap_fields(meta):
    out = np.zeros_like(meta)
    for n in range(8):
        nib = (meta >> np.uint32(4 * n)) & np.uint32(0xF)
        a, b = nib & np.uint32(3), nib >> np.uint32(2)
        out |= ((b | (a << np.uint32(2))) << np.uint32(4 * n)).astype(np.uint32)
    return out


def _compress_fields_swapped(*args, **kw):
    L = _orig["compress"](*args, **kw)
    L.meta = _swap_fields(L.meta)
    return L


def _decompress_fields_swapped(L):
    import copy
    L2 = copy.copy(L)
    L2.meta = _swap_fields(L.meta)
    return _orig["decompress"](L2)


def _translate_forward(L, row_of_channel):
    return _orig["translate_index"](L, np.argsort(np.asarray(row_of_channel)))


# --------------------------------------------------------------------------- product
def _spmm_ignores_mask(W_bits, bitmask, X_bits, rows=None):
    W = O._bf16_to_f64(W_bits if rows is None else W_bits[rows])
    X = O._bf16_to_f64(X_bits)
    return W @ X, np.abs(W) @ np.abs(X)


def _masked_weight_inverted(W_bits, bitmask):
    K = W_bits.shape[1]
    return np.where(~O.unpack_bits(bitmask, K), O._bf16_to_f64(W_bits), 0.0)


# ------------------------------------------------------------ epilogue, Hard-Concrete
def _gelu_tanh(x, act):
    if act == O.ACT_GELU:
        x = np.asarray(x, dtype=np.float64)
        return 0.5 * x * (1.0 + np.tanh(math.sqrt(2.0 / math.pi) * (x + 0.044715 * x ** 3)))
    return _orig["activation"](x, act)


def _bias_per_column(y, bias, act):
    z = np.asarray(y, dtype=np.float64)
    if bias is not None:
        z = z + np.asarray(bias, dtype=np.float64)[None, : z.shape[1]]
    return O.activation(z, act)


def _hc_no_stretch(log_alpha, eps, tau):
    la = np.asarray(log_alpha, dtype=np.float64)
    e = np.asarray(eps, dtype=np.float64)
    s = 1.0 / (1.0 + np.exp(-(np.log(e) - np.log1p(-e) + la) / tau))
    z = np.minimum(1.0, np.maximum(0.0, s))
    hard = (z > 0.5).astype(np.uint8)
    sums = np.array([z.sum(), np.abs(z.reshape(-1, 4).sum(axis=1) - 2.0).sum()])
    return z, hard, sums


# ------------------------------------------------------------------------------ gyro
def _group_cost_largest(I_tile, members):
    acc = 0.0
    for r in range(I_tile.shape[0]):
        v = sorted((float(I_tile[r, c]) for c in members), reverse=True)
        acc += v[0] + v[1]
    return acc


def _column_cost_largest(I_rows, n0):
    V = np.zeros(I_rows.shape[1])
    for r in range(I_rows.shape[0]):
        V = V + np.asarray(I_rows[r], dtype=np.float64)
    order = np.lexsort((np.arange(V.size), -V))
    return float(sum(V[j] for j in order[:n0]))


def _kmeans_unbalanced(F, k, iters):
    S, d = F.shape
    G = S // k
    clusters = [list(range(i * k, (i + 1) * k)) for i in range(G)]
    for _ in range(iters):
        C = np.array([F[cl].mean(axis=0) if cl else np.zeros(d) for cl in clusters])
        near = [int(np.argmin(((F[p] - C) ** 2).sum(axis=1))) for p in range(S)]
        new = [sorted(p for p in range(S) if near[p] == c) for c in range(G)]
        if new == clusters:
            break
        clusters = new
    return clusters


# ------------------------------------------------------------ readings of the grouping
def _mask_groups_in_rank_order(I_tile_w, region_w):
    """2:4 groups formed from the 2:4 vectors in rank order (score descending) instead of
    ascending working position."""
    T, K = I_tile_w.shape
    V = np.zeros(K)
    for i in range(T):
        V += I_tile_w[i].astype(np.float64)
    order = np.lexsort((np.arange(K), -V))
    pos = np.array([j for j in order if region_w[j] == O.REGION_24], dtype=np.int64)
    keep = np.zeros((T, K), dtype=bool)
    keep[:, region_w == O.REGION_DENSE] = True
    if pos.size:
        g = pos.reshape(-1, 4)
        keep_g = O.top2_keep(I_tile_w[:, g])
        for k in range(4):
            keep[:, g[:, k]] = keep_g[:, :, k]
    return keep


def _compress_index_not_permuted(W_bits, bitmask, region, perm, counts, T, tiles=None):
    """The index holds working positions instead of input channels (the permutation is not
    folded in)."""
    L = _orig["compress"](W_bits, bitmask, region, perm, counts, T, tiles)
    p = np.asarray(perm)
    if p.ndim == 1:
        inv = np.argsort(p)
        L.idx_dense = inv[L.idx_dense].astype(np.int32)
        L.idx_sparse = inv[L.idx_sparse].astype(np.int32)
        L.run_dense = O.contiguous_runs(L.idx_dense)
        L.run_sparse = O.contiguous_runs(L.idx_sparse)
    return L


def _retained_fp32(I_tile_w, keep):
    acc = np.float32(0.0)
    for v in I_tile_w[keep].ravel():
        acc = np.float32(acc + np.float32(v))
    return float(acc)


def _gyro_round_keeps_worse(I_tile, band, groups, slots, kmeans_iters=8):
    """The round's arrangement is taken even when the sampled groups' cost rises."""
    from scipy.optimize import linear_sum_assignment
    band = np.array(band, dtype=np.int64).copy()
    groups = [int(g) for g in np.asarray(groups).ravel()]
    slots = np.asarray(slots, dtype=np.int64)
    G, k = slots.shape
    vecs = [int(band[4 * g + int(x)]) for g, ss in zip(groups, slots) for x in ss]
    F = np.asarray(I_tile, dtype=np.float64)[:, vecs].T.copy()
    clusters = O.balanced_kmeans(F, k, kmeans_iters)
    cost = O.gyro_input_cost_matrix(I_tile, band, groups, slots, clusters)
    rows, cols = linear_sum_assignment(-cost)   # and the assignment maximises the cost
    assign = {int(i): int(c) for c, i in zip(rows, cols)}
    before = sum(O.group_pruning_cost(I_tile, [int(x) for x in band[4 * g:4 * g + 4]])
                 for g in groups)
    new = band.copy()
    after = 0.0
    for i in range(G):
        g = groups[i]
        m = [int(x) for x in band[4 * g:4 * g + 4]]
        for sl, pt in zip(sorted(int(x) for x in slots[i]), clusters[assign[i]]):
            m[sl] = vecs[pt]
        new[4 * g:4 * g + 4] = m
        after += cost[assign[i], i]
    return new, (before, after)


# ------------------------------------------------------------------ orders and signs
def _energy_descending(X_bits):
    X = O._bf16_to_f64(X_bits)
    acc = np.zeros(X.shape[0])
    for n in reversed(range(X.shape[1])):
        acc += X[:, n] * X[:, n]
    return acc.astype(np.float32)


def _scores_fp32(I, perm, T):
    M, K = I.shape
    nt = M // T
    Iw = (I[:, perm].reshape(nt, T, K) if np.asarray(perm).ndim == 1 else
          np.stack([I[t * T:(t + 1) * T][:, O.tile_perm(perm, t)] for t in range(nt)]))
    V = np.zeros((nt, K), dtype=np.float32)
    for i in range(T):
        V = (V + Iw[:, i, :].astype(np.float32)).astype(np.float32)
    return V.astype(np.float64)


def _scan_from_the_other_end(R):
    """The scan starts at the last candidate (v_s lowest) and walks up."""
    for m in range(len(R) - 1, 0, -1):
        if R[m - 1] < R[m]:
            return m
    return 0


def _spmm_bound_signed(W_bits, bitmask, X_bits, rows=None):
    y, _ = _orig["spmm_reference"](W_bits, bitmask, X_bits, rows)
    Wm = O.masked_weight(W_bits if rows is None else W_bits[rows],
                         bitmask if rows is None else bitmask[rows])
    return y, Wm @ O._bf16_to_f64(X_bits)


def _hc_logit_sign(log_alpha, eps, tau):
    e = np.asarray(eps, dtype=np.float64)
    return _orig["hard_concrete"](log_alpha, 1.0 - e, tau)


def _silu_wrong_sign(x, act):
    if act == O.ACT_SILU:
        x = np.asarray(x, dtype=np.float64)
        return x / (1.0 + np.exp(x))
    return _orig["activation"](x, act)


# ------------------------------------------------------------------ layout bookkeeping
def _tile_blocks_floor(counts):
    nt = counts.shape[0]
    info = np.zeros((nt, 4), dtype=np.int32)
    d0 = s0 = 0
    for t in range(nt):
        n0, n24, n4 = (int(x) for x in counts[t])
        nd, ns = n4 // O.DENSE_BK, n24 // O.SPARSE_BK
        info[t] = (nd, ns, d0, s0)
        d0 += nd
        s0 += ns
    return info


def _runs_any_ascending(idx):
    out = np.full(idx.shape[0], -1, dtype=np.int32)
    if idx.shape[0]:
        run = (np.diff(idx, axis=1) > 0).all(axis=1)
        out[run] = idx[run, 0]
    return out


MUTANTS = {
    "energy_drops_square": {"channel_energy": _energy_drops_square},
    "energy_over_wrong_axis": {"channel_energy": _energy_over_wrong_axis},
    "importance_w_not_squared": {"importance_rows": _importance_w_not_squared},
    "importance_rows_ignored": {"importance_rows": _importance_rows_ignored},
    "scores_skip_last_row": {"vector_scores": _scores_skip_last_row},
    "order_ascending": {"vector_order": _order_ascending},
    "order_ties_high_first": {"vector_order": _order_ties_high_first},
    "counts_truncate": {"counts_from_vs": _counts_truncates},
    "counts_n0_full_n24": {"counts_from_vs": _counts_n0_full},
    "candidates_drop_last": {"search_candidates": _candidates_drop_last},
    "regions_dense_24_swapped": {"regions_from_rank": _regions_swapped},
    "groups_descending": {"groups_24": _groups_descending},
    "top2_ties_to_higher": {"top2_keep": _top2_ties_high},
    "top2_keeps_smallest": {"top2_keep": _top2_keeps_smallest},
    "retained_ignores_keep": {"retained_importance": _retained_ignores_keep},
    "search_nonstrict_drop": {"boundary_search": _search_with(_rule_nonstrict)},
    "search_one_past_drop": {"boundary_search": _search_with(_rule_one_past)},
    "bit_order_reversed": {"pack_bits": _pack_msb_first, "unpack_bits": _unpack_msb_first},
    "swizzle_without_xor": {"swizzled_offset": _swizzle_without_xor},
    "meta_halves_swapped": {"meta_word_index": _meta_halves_swapped},
    "meta_fields_swapped": {"compress": _compress_fields_swapped,
                            "decompress": _decompress_fields_swapped},
    "translate_forward_map": {"translate_index": _translate_forward},
    "spmm_ignores_mask": {"spmm_reference": _spmm_ignores_mask},
    "masked_weight_inverted": {"masked_weight": _masked_weight_inverted},
    "gelu_tanh_form": {"activation": _gelu_tanh},
    "bias_per_column": {"spmm_epilogue_reference": _bias_per_column},
    "hard_concrete_no_stretch": {"hard_concrete": _hc_no_stretch},
    "group_cost_largest_two": {"group_pruning_cost": _group_cost_largest},
    "column_cost_largest": {"column_pruning_cost": _column_cost_largest},
    "kmeans_unbalanced": {"balanced_kmeans": _kmeans_unbalanced},
    "groups_in_rank_order": {"tile_mask_working": _mask_groups_in_rank_order},
    "index_without_permutation": {"compress": _compress_index_not_permuted},
    "retained_in_fp32": {"retained_importance": _retained_fp32},
    "gyro_keeps_worse_rounds": {"gyro_input_round": _gyro_round_keeps_worse},
    "energy_sums_descending": {"channel_energy": _energy_descending},
    "scores_in_fp32": {"vector_scores": _scores_fp32},
    "scan_from_the_other_end": {"boundary_search": _search_with(_scan_from_the_other_end)},
    "bound_signed": {"spmm_reference": _spmm_bound_signed},
    "hard_concrete_logit_sign": {"hard_concrete": _hc_logit_sign},
    "silu_wrong_sign": {"activation": _silu_wrong_sign},
    "tile_blocks_round_down": {"tile_blocks": _tile_blocks_floor},
    "runs_accept_any_ascending_indices": {"contiguous_runs": _runs_any_ascending},
}


def apply(name):
    for attr, fn in MUTANTS[name].items():
        setattr(O, attr, fn)
