"""CPU oracle for the HiNM (hierarchical N:M) hot path -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` / ``--impl
reference`` legs of ``bench.py`` may import this module.  The product path
(``pruning_hinm_spmm_b200``) never imports it, and this module imports nothing from
the product path: the two share only the seeded input generator ``hinm_inputs``.

It is a plain, slow, step-by-step restatement of what the pages define, in fp64 where
the pages leave the precision open.  Sources (page title, section):

* [P1] "FlexHiNM-GP: Flexible Hierarchical Pruning via Region Allocation and Channel
  Permutation" (papernotes.org notes): 整体框架 (tiles of output rows, each runs the
  boundary search), 关键设计 1 (three regions, closed form t_s = v_s + (1-v_s) p_s/2,
  retained second-order importance R_total = R_dense + R_24, scan from v_s = t_s
  downward by alpha, stop at the first drop), 关键设计 2 (importance matrix D; the
  permutation reorders channels without changing the result and is folded into the
  HiNM index), 关键设计 4 (dense part + 2:4 part gathered by the precomputed index,
  summed into one output), 亮点与洞察 (high importance -> dense, middle -> 2:4,
  low -> pruned).
* [P2] "面向Transformer的块稀疏剪枝：N:M稀疏模式在硬件加速上的优势" (rkmt.cn),
  section 二: groups of 4 consecutive elements along the input dimension, keep 2.
* [P3] "结构化稀疏与剪枝:2:4 稀疏模式为何能让 GPU 矩阵吞吐翻倍" (geek-doc.cn),
  section 三: 2 stored values per group of 4 plus 2-bit position indices (6 patterns);
  section 五: the mask M has W's shape and the layer computes with W ⊙ M.
* [P4] PermLLM notes (lowest.today), "Интеграция с существующими методами обрезки":
  the mask is chosen on the permuted importance S·P, i.e. in working order.
* [P5] "非结构化剪枝与结构化剪枝" (apxml.com), 结构化剪枝: removing a whole column.

Readings where the pages are silent are marked [reading] at the step that takes them.

Parity pins: every function here is pinned by ``tests/test_oracle_pins.py`` against
closed forms, brute force on tiny inputs, exact rational arithmetic, invariants and the
pages' printed examples (``tests/golden/``).  No function is "parity unpinned".
"""
from __future__ import annotations

import math
from dataclasses import dataclass
from typing import Dict, List, Optional, Tuple

import numpy as np

REGION_PRUNED = 0   # 0:4 -- the whole column vector is removed
REGION_24 = 1       # 2:4 -- two of every four consecutive 2:4 vectors kept per row
REGION_DENSE = 2    # 4:4 -- the whole column vector is kept

# Compressed-layout geometry (a builder's choice; the pages fix none of it).
BLOCK_ROWS = 128        # rows per compressed block (tile rows, zero-padded when T = 64)
DENSE_BK = 64           # dense vectors per dense block (64 bf16 = 128 bytes per row)
SPARSE_BK = 128         # 2:4 vectors per sparse block (64 kept values = 128 bytes per row)
META_WORDS = 512        # 32-bit metadata words per sparse block (128 lanes x 4 words)
PAD_NIBBLE = 0x4        # metadata of a padded group: positions (0, 1), both values 0
LEGAL_NIBBLES = (0x4, 0x8, 0xC, 0x9, 0xD, 0xE)  # a | b << 2 with a < b: the C(4,2) = 6 patterns


def _bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(
        np.float32).astype(np.float64)


def _bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


# ---------------------------------------------------------------------------------------
# a1. importance
# ---------------------------------------------------------------------------------------
def channel_energy(X_bits: np.ndarray) -> np.ndarray:
    """s_c = sum_n x_cn^2 for every input channel c, returned as fp32.

    [P1] 关键设计 1/2 name a second-order importance D without giving its formula; the
    diagonal proxy w^2 * ||x_c||^2 is the plainest reading.  [reading] The sum runs in
    fp64 with n ascending (each x^2 of a bf16 x is exact in fp64) and is rounded once to
    fp32 (round-to-nearest-even).
    """
    X = _bf16_to_f64(X_bits)
    K, N = X.shape
    acc = np.zeros(K, dtype=np.float64)
    for n in range(N):                      # fixed order: n = 0, 1, ..., N-1
        acc += X[:, n] * X[:, n]
    return acc.astype(np.float32)


def importance(W_bits: np.ndarray, X_bits: np.ndarray) -> np.ndarray:
    """I[i, c] = fl32( fl32(w_ic^2) * s_c ), an M x K fp32 matrix indexed by original channel.

    [P1] 关键设计 1 (second-order importance of the weights), 关键设计 2 (importance matrix D).
    w^2 of a bf16 w is exact in fp32 (barring underflow); the product with s_c is one
    fp32 rounding.
    """
    return importance_rows(W_bits, X_bits, None)


def importance_rows(W_bits: np.ndarray, X_bits: np.ndarray,
                    rows: Optional[np.ndarray]) -> np.ndarray:
    """The rows ``rows`` of ``importance(W, X)`` (every row when rows is None), with the
    channel energies s_c still taken over all of X: I[i, c] = fl32(fl32(w_ic^2) * s_c)."""
    W = _bf16_to_f32(W_bits if rows is None else np.asarray(W_bits)[rows])
    s = channel_energy(X_bits)
    w2 = (W * W).astype(np.float32)
    return (w2 * s[None, :]).astype(np.float32)


# ---------------------------------------------------------------------------------------
# a2. vector scores
# ---------------------------------------------------------------------------------------
def tile_perm(perm: np.ndarray, t: int) -> np.ndarray:
    """Working order of tile t: ``perm`` is one order [K] for every tile or one per tile
    [M/T, K] ([P1] 关键设计 2: the input-channel permutation is found inside each tile)."""
    perm = np.asarray(perm)
    return perm if perm.ndim == 1 else perm[t]


def vector_scores(I: np.ndarray, perm: np.ndarray, T: int) -> np.ndarray:
    """V[t, j] = sum over the tile's rows (ascending) of I[row, perm_t[j]], in fp64.

    [P1] 整体框架 (W is cut into tiles of output rows), 研究背景 (vectors are ranked by
    importance), 亮点与洞察 (vector-level regions).  [reading] A vector is one input
    channel restricted to the tile's T rows; its score is the sum of its elements'
    importance, accumulated sequentially over ascending rows in fp64.
    """
    M, K = I.shape
    nt = M // T
    if np.asarray(perm).ndim == 1:
        Iw = I[:, perm].reshape(nt, T, K)
    else:
        Iw = np.stack([I[t * T:(t + 1) * T][:, tile_perm(perm, t)] for t in range(nt)])
    V = np.zeros((nt, K), dtype=np.float64)
    for i in range(T):                      # fixed order: rows ascending
        V += Iw[:, i, :].astype(np.float64)
    return V


def vector_order(V_t: np.ndarray) -> np.ndarray:
    """Working positions sorted by (score descending, position ascending).

    [P1] 亮点与洞察: high-importance vectors are kept dense, middle ones go to 2:4, low
    ones are pruned.  [reading] Equal scores rank the lower working position first.
    """
    K = V_t.shape[0]
    return np.lexsort((np.arange(K), -V_t))


def vector_rank(V: np.ndarray) -> np.ndarray:
    """rank[t, j] = position of working position j in ``vector_order(V[t])``."""
    nt, K = V.shape
    rank = np.empty((nt, K), dtype=np.int32)
    for t in range(nt):
        order = vector_order(V[t])
        rank[t, order] = np.arange(K, dtype=np.int32)
    return rank


# ---------------------------------------------------------------------------------------
# closed-form boundary -> region counts
# ---------------------------------------------------------------------------------------
def partial_sparsity(t_s: float, v_s: float) -> float:
    """p_s = 2 (t_s - v_s) / (1 - v_s), the closed form of [P1] 关键设计 1."""
    return 2.0 * (t_s - v_s) / (1.0 - v_s)


def counts_from_vs(K: int, t_s: float, v_s: float) -> Tuple[int, int, int]:
    """(n_0, n_24, n_4) vectors per tile for the boundary (t_s, v_s).

    [P1] 关键设计 1: t_s = v_s + (1 - v_s) p_s / 2, so the 2:4 region holds a fraction
    (1 - v_s) p_s = 2 (t_s - v_s) of the K vectors.  [reading] The pages never round:
    n_24 = 4 * floor(2 (t_s - v_s) K / 4 + 1/2) (a whole number of groups of 4),
    n_0 = t_s K - n_24 / 2 (keeps the overall sparsity exactly t_s), n_4 = K - n_0 - n_24.
    t_s K must be a whole number and every count non-negative.
    """
    x = 2.0 * (t_s - v_s) * K / 4.0
    n24 = 4 * int(math.floor(x + 0.5))
    tk = t_s * K
    if tk != math.floor(tk):
        raise ValueError(f"t_s*K = {tk!r} is not a whole number of vectors")
    n0 = int(tk) - n24 // 2
    n4 = K - n0 - n24
    if n24 < 0 or n0 < 0 or n4 < 0:
        raise ValueError(f"negative region count for t_s={t_s}, v_s={v_s}, K={K}")
    return n0, n24, n4


def search_candidates(K: int, t_s: float, alpha: float) -> List[Tuple[int, int, int]]:
    """Counts for v_s = t_s - m*alpha, m = 0, 1, ..., m_max.

    [P1] 关键设计 1: the scan starts at v_s = t_s (p_s = 0) and steps v_s down by alpha.
    [reading] p_s <= 1 bounds v_s >= max(0, 2 t_s - 1), so
    m_max = floor((t_s - max(0, 2 t_s - 1)) / alpha); a trailing candidate whose counts
    round to a negative region is dropped.  The adaptive terms beta, gamma of the step
    are undefined on the pages and taken as 0.
    """
    m_max = int(math.floor((t_s - max(0.0, 2.0 * t_s - 1.0)) / alpha))
    out = []
    for m in range(m_max + 1):
        v_s = t_s - m * alpha
        try:
            out.append(counts_from_vs(K, t_s, v_s))
        except ValueError:
            if m == 0:
                raise
            break
    return out


# ---------------------------------------------------------------------------------------
# regions and 2:4 selection
# ---------------------------------------------------------------------------------------
def regions_from_rank(rank_t: np.ndarray, counts: Tuple[int, int, int]) -> np.ndarray:
    """Region of every working position: rank < n_4 dense, next n_24 are 2:4, rest pruned.

    [P1] 亮点与洞察 and 关键设计 1 (vector pruning 0:4 of the lowest vectors).
    """
    n0, n24, n4 = counts
    reg = np.full(rank_t.shape, REGION_PRUNED, dtype=np.int8)
    reg[rank_t < n4 + n24] = REGION_24
    reg[rank_t < n4] = REGION_DENSE
    return reg


def groups_24(region_w: np.ndarray) -> np.ndarray:
    """The 2:4-region working positions in ascending order, as rows of 4 (one group each).

    [P2] 二: groups are 4 consecutive elements along the input dimension.  [reading]
    "Consecutive" is in working (permuted) order, which is what the input-channel
    gyro-permutation arranges ([P1] 关键设计 2, [P4] mask on S·P).
    """
    pos = np.nonzero(region_w == REGION_24)[0]
    if pos.size % 4:
        raise ValueError("the 2:4 region must hold a multiple of 4 vectors")
    return pos.reshape(-1, 4)


def top2_keep(vals: np.ndarray) -> np.ndarray:
    """Keep flags for the last axis of size 4: the 2 largest values, lower index on ties.

    [P2] 二 (keep 2 of every 4), [P3] 三 (exactly 2 of 4).  Element k is kept iff fewer
    than 2 members beat it, where k' beats k if v_k' > v_k, or v_k' == v_k and k' < k.
    """
    v = vals[..., :, None]           # v_k
    w = vals[..., None, :]           # v_k'
    kidx = np.arange(4)
    lower = kidx[None, :] < kidx[:, None]          # [k, k']: k' < k
    beats = (w > v) | ((w == v) & lower)
    return beats.sum(axis=-1) < 2


def tile_mask_working(I_tile_w: np.ndarray, region_w: np.ndarray) -> np.ndarray:
    """Boolean keep-mask of one tile in working order (T x K).

    Dense vectors keep every element, pruned vectors none, and each 2:4 group keeps the
    top-2 of its 4 members in every row ([P1] 关键设计 1, [P2] 二).
    """
    T, K = I_tile_w.shape
    keep = np.zeros((T, K), dtype=bool)
    keep[:, region_w == REGION_DENSE] = True
    g = groups_24(region_w)
    if g.size:
        vals = I_tile_w[:, g]                     # T x G x 4
        keep_g = top2_keep(vals)
        for k in range(4):
            keep[:, g[:, k]] = keep_g[:, :, k]
    return keep


def retained_importance(I_tile_w: np.ndarray, keep: np.ndarray) -> float:
    """R = sum of the importance of every kept element of a tile.

    [P1] 关键设计 1: R_total = R_dense + R_24, the second-order importance summed over the
    retained weights.  [reading] The
    sum is taken exactly and rounded once to fp64 (math.fsum is exactly rounded), so the
    comparison between candidates does not depend on a summation order.
    """
    return math.fsum(I_tile_w[keep].astype(np.float64).tolist())


# ---------------------------------------------------------------------------------------
# a3. boundary search
# ---------------------------------------------------------------------------------------
@dataclass
class SearchResult:
    counts: np.ndarray          # int32 [nt, 3] = (n_0, n_24, n_4)
    v_s: np.ndarray             # fp64 [nt]
    m: np.ndarray               # int32 [nt], chosen step index
    R: List[List[float]]        # per tile, R(m) for every candidate
    rank: np.ndarray            # int32 [nt, K]


def boundary_search(I: np.ndarray, perm: np.ndarray, T: int, t_s: float, alpha: float,
                    tiles: Optional[List[int]] = None) -> SearchResult:
    """Per tile, scan v_s = t_s, t_s - alpha, ... and stop at the first drop of R.

    [P1] 整体框架 (each tile runs the boundary search) and 关键设计 1 (start at v_s = t_s,
    step down by alpha, stop as soon as the objective decreases).  Returns the first m
    with R(m+1) < R(m), else the last candidate.  ``tiles`` restricts the work to a
    sample of tiles (other rows of the result are left zero).
    """
    M, K = I.shape
    nt = M // T
    cands = search_candidates(K, t_s, alpha)
    V = vector_scores(I, perm, T) if tiles is None else None
    counts = np.zeros((nt, 3), dtype=np.int32)
    vs = np.zeros(nt, dtype=np.float64)
    ms = np.zeros(nt, dtype=np.int32)
    rank = np.zeros((nt, K), dtype=np.int32)
    Rs: List[List[float]] = [[] for _ in range(nt)]
    for t in (range(nt) if tiles is None else tiles):
        I_tile_w = I[t * T:(t + 1) * T][:, tile_perm(perm, t)]
        V_t = V[t] if V is not None else vector_scores(I[t * T:(t + 1) * T], tile_perm(perm, t),
                                                       T)[0]
        order = vector_order(V_t)
        rank[t, order] = np.arange(K, dtype=np.int32)
        R = []
        for c in cands:
            keep = tile_mask_working(I_tile_w, regions_from_rank(rank[t], c))
            R.append(retained_importance(I_tile_w, keep))
        m_star = len(cands) - 1
        for m in range(len(cands) - 1):
            if R[m + 1] < R[m]:
                m_star = m
                break
        counts[t] = cands[m_star]
        vs[t] = t_s - m_star * alpha
        ms[t] = m_star
        Rs[t] = R
    return SearchResult(counts=counts, v_s=vs, m=ms, R=Rs, rank=rank)


# ---------------------------------------------------------------------------------------
# a4. mask
# ---------------------------------------------------------------------------------------
def mask(I: np.ndarray, perm: np.ndarray, T: int, counts: np.ndarray,
         tiles: Optional[List[int]] = None) -> Tuple[np.ndarray, np.ndarray]:
    """Bit-packed keep-mask (M x ceil(K/32) uint32) and region (M/T x K int8, by channel).

    [P3] 五: the mask has W's shape and the layer computes with W ⊙ M.  Bit b of word w
    of row i covers original channel c = 32 w + b; bits past K are 0.  Regions and 2:4
    groups are chosen in working order and mapped back through perm ([P4]).
    """
    M, K = I.shape
    nt = M // T
    words = (K + 31) // 32
    bitmask = np.zeros((M, words), dtype=np.uint32)
    region = np.zeros((nt, K), dtype=np.int8)
    for t in (range(nt) if tiles is None else tiles):
        pt = tile_perm(perm, t)
        I_tile_w = I[t * T:(t + 1) * T][:, pt]
        V_t = vector_scores(I[t * T:(t + 1) * T], pt, T)[0]
        order = vector_order(V_t)
        rank_t = np.empty(K, dtype=np.int32)
        rank_t[order] = np.arange(K, dtype=np.int32)
        reg_w = regions_from_rank(rank_t, tuple(int(x) for x in counts[t]))
        keep_w = tile_mask_working(I_tile_w, reg_w)
        keep_c = np.zeros((T, K), dtype=bool)
        keep_c[:, pt] = keep_w
        region[t, pt] = reg_w
        bitmask[t * T:(t + 1) * T] = pack_bits(keep_c)
    return bitmask, region


def pack_bits(keep: np.ndarray) -> np.ndarray:
    """Pack a boolean (rows x K) array into uint32 words, bit b of word w = column 32w+b."""
    R, K = keep.shape
    words = (K + 31) // 32
    padded = np.zeros((R, words * 32), dtype=np.uint64)
    padded[:, :K] = keep
    weights = (np.uint64(1) << np.arange(32, dtype=np.uint64))
    return (padded.reshape(R, words, 32) * weights).sum(axis=-1).astype(np.uint32)


def unpack_bits(bitmask: np.ndarray, K: int) -> np.ndarray:
    R, words = bitmask.shape
    bits = (bitmask[:, :, None].astype(np.uint64) >> np.arange(32, dtype=np.uint64)) & np.uint64(1)
    return bits.reshape(R, words * 32)[:, :K].astype(bool)


# ---------------------------------------------------------------------------------------
# a5. compress -- the HiNM layout (byte for byte as include/hinm.h documents it)
# ---------------------------------------------------------------------------------------
def swizzled_offset(r: int, k: int) -> int:
    """Byte offset of bf16 element (row r, column k) in a 128-row x 64-column block.

    Rows are 128 bytes apart; within a row the 16-byte chunk k//8 is stored at chunk
    position (k//8) XOR (r mod 8) -- the 128-byte swizzle of the tensor cores' K-major
    shared-memory operand, so a block is copied to shared memory unchanged.
    """
    return r * 128 + (((k >> 3) ^ (r & 7)) << 4) + (k & 7) * 2


def meta_word_index(m: int, g: int) -> Tuple[int, int]:
    """(word index, bit shift) of the 4-bit metadata of (row m, group g) in a sparse block.

    The 2 KB metadata block is 128 lanes x 4 words (lane-major).  Word w of lane L
    describes logical columns [32 w, 32 w + 32) of the block: its bits [16 s + 4 q,
    16 s + 4 q + 4) hold the group 8 w + 4 h + q of row 16 (L // 16) + 8 s + (L mod 8),
    where h = (L // 8) mod 2.  This is the tensor-memory placement of sparse-MMA
    metadata for a 128-row, 16-bit A operand.
    """
    w, rem = divmod(g, 8)
    h, q = divmod(rem, 4)
    s = (m >> 3) & 1
    L = (m & 7) + 8 * h + 16 * (m >> 4)
    return L * 4 + w, 16 * s + 4 * q


@dataclass
class Layout:
    M: int
    K: int
    T: int
    tile_info: np.ndarray       # int32 [nt, 4] = (dense blocks, sparse blocks, first dense, first sparse)
    vals_dense: np.ndarray      # uint8 [nd_total, 16384]
    vals_sparse: np.ndarray     # uint8 [ns_total, 16384]
    meta: np.ndarray            # uint32 [ns_total, 512]
    idx_dense: np.ndarray       # int32 [nd_total, 64]
    idx_sparse: np.ndarray      # int32 [ns_total, 128]
    run_dense: np.ndarray       # int32 [nd_total]: idx[0] if idx[v] == idx[0] + v for all v, else -1
    run_sparse: np.ndarray      # int32 [ns_total]


def tile_blocks(counts: np.ndarray) -> np.ndarray:
    """tile_info: dense blocks ceil(n_4/64), sparse blocks ceil(n_24/128), prefix offsets."""
    nt = counts.shape[0]
    info = np.zeros((nt, 4), dtype=np.int32)
    d0 = s0 = 0
    for t in range(nt):
        n0, n24, n4 = (int(x) for x in counts[t])
        nd = -(-n4 // DENSE_BK)
        ns = -(-n24 // SPARSE_BK)
        info[t] = (nd, ns, d0, s0)
        d0 += nd
        s0 += ns
    return info


def compress(W_bits: np.ndarray, bitmask: np.ndarray, region: np.ndarray, perm: np.ndarray,
             counts: np.ndarray, T: int, tiles: Optional[List[int]] = None) -> Layout:
    """Pack W ⊙ M into the HiNM layout: dense values, 2:4 values + 2-bit metadata, index.

    [P1] 关键设计 2/4: the dense tile and the 2:4 values are stored separately; the 2:4
    part is gathered against X by a precomputed index into which the input permutation is
    folded (idx = perm[j]).  [P3] 三: per group of 4, 2 values and two 2-bit positions
    (a | b << 2, a < b).  Dense vectors and 2:4 vectors are each laid out in ascending
    working position.  Padding: value 0, nibble 0x4, index 0; rows >= T (T = 64) are padding.
    """
    M, K = W_bits.shape
    nt = M // T
    keep_c = unpack_bits(bitmask, K)
    info = tile_blocks(counts)
    nd_tot = int(info[:, 0].sum())
    ns_tot = int(info[:, 1].sum())
    vals_dense = np.zeros((nd_tot, 16384), dtype=np.uint8)
    vals_sparse = np.zeros((ns_tot, 16384), dtype=np.uint8)
    meta = np.zeros((ns_tot, META_WORDS), dtype=np.uint32)
    idx_dense = np.zeros((nd_tot, DENSE_BK), dtype=np.int32)
    idx_sparse = np.zeros((ns_tot, SPARSE_BK), dtype=np.int32)
    Wb = np.asarray(W_bits, dtype=np.uint16)
    for t in (range(nt) if tiles is None else tiles):
        nd, ns, d0, s0 = (int(x) for x in info[t])
        pt = tile_perm(perm, t)
        reg_w = region[t][pt]
        dense_j = np.nonzero(reg_w == REGION_DENSE)[0]
        sp_j = np.nonzero(reg_w == REGION_24)[0]
        rows = range(t * T, (t + 1) * T)
        # dense blocks
        for b in range(nd):
            blk = np.zeros(16384, dtype=np.uint8)
            for k in range(DENSE_BK):
                p = b * DENSE_BK + k
                if p >= dense_j.size:
                    continue
                c = int(pt[dense_j[p]])
                idx_dense[d0 + b, k] = c
                for r, i in enumerate(rows):
                    v = int(Wb[i, c]) if keep_c[i, c] else 0
                    off = swizzled_offset(r, k)
                    blk[off] = v & 0xFF
                    blk[off + 1] = v >> 8
            vals_dense[d0 + b] = blk
        # sparse blocks
        for b in range(ns):
            blk = np.zeros(16384, dtype=np.uint8)
            mw = np.zeros(META_WORDS, dtype=np.uint64)
            for g in range(SPARSE_BK // 4):
                base = b * SPARSE_BK + 4 * g
                members = [int(pt[sp_j[base + k]]) if base + k < sp_j.size else None
                           for k in range(4)]
                for k in range(4):
                    if members[k] is not None:
                        idx_sparse[s0 + b, 4 * g + k] = members[k]
                for r in range(BLOCK_ROWS):
                    if r < T and members[0] is not None:
                        i = t * T + r
                        kept = [k for k in range(4) if keep_c[i, members[k]]]
                        if len(kept) != 2:
                            raise ValueError(f"row {i} group {g}: {len(kept)} kept positions, want 2")
                        a, bb = kept
                        va, vb = int(Wb[i, members[a]]), int(Wb[i, members[bb]])
                    else:
                        a, bb, va, vb = 0, 1, 0, 0
                    for slot, v in ((0, va), (1, vb)):
                        off = swizzled_offset(r, 2 * g + slot)
                        blk[off] = v & 0xFF
                        blk[off + 1] = v >> 8
                    wi, sh = meta_word_index(r, g)
                    mw[wi] |= np.uint64((a | (bb << 2)) << sh)
            vals_sparse[s0 + b] = blk
            meta[s0 + b] = mw.astype(np.uint32)
    return Layout(M=M, K=K, T=T, tile_info=info, vals_dense=vals_dense,
                  vals_sparse=vals_sparse, meta=meta, idx_dense=idx_dense, idx_sparse=idx_sparse,
                  run_dense=contiguous_runs(idx_dense), run_sparse=contiguous_runs(idx_sparse))


def contiguous_runs(idx: np.ndarray) -> np.ndarray:
    """Per block: the first index if the block's indices are one ascending run
    (idx[v] = idx[0] + v), else -1.  Lets the product load such blocks of X as one tile."""
    out = np.full(idx.shape[0], -1, dtype=np.int32)
    if idx.shape[0]:
        steps = idx - idx[:, :1]
        run = (steps == np.arange(idx.shape[1], dtype=np.int32)[None, :]).all(axis=1)
        out[run] = idx[run, 0]
    return out


def translate_index(L: Layout, row_of_channel: np.ndarray) -> Layout:
    """Cross-layer index translation: the layout for an X whose rows arrive reordered.

    [P1] 关键设计 2: reordering channels leaves the result unchanged, and the translation
    between layers is folded into the HiNM index, done while the data is moved, with no
    extra runtime step.  [reading] When X arrives with row r holding input channel
    sigma[r] (the previous layer's output in its permuted row order), every index entry
    c becomes row_of_channel[c] = sigma^-1[c], and each block's run flag is recomputed by
    the same rule as ``compress`` (``contiguous_runs``).  Values, metadata and tile_info
    are unchanged, so the product with the reordered X equals the original product.
    """
    roc = np.asarray(row_of_channel, dtype=np.int64)
    idx_d = roc[L.idx_dense].astype(np.int32) if L.idx_dense.size else L.idx_dense.copy()
    idx_s = roc[L.idx_sparse].astype(np.int32) if L.idx_sparse.size else L.idx_sparse.copy()
    return Layout(M=L.M, K=L.K, T=L.T, tile_info=L.tile_info.copy(),
                  vals_dense=L.vals_dense.copy(), vals_sparse=L.vals_sparse.copy(),
                  meta=L.meta.copy(), idx_dense=idx_d, idx_sparse=idx_s,
                  run_dense=contiguous_runs(idx_d), run_sparse=contiguous_runs(idx_s))


def decompress(L: Layout) -> np.ndarray:
    """Rebuild W ⊙ M (fp32, M x K) from a layout; the inverse of ``compress``."""
    out = np.zeros((L.M, L.K), dtype=np.float32)
    nt = L.M // L.T

    def val(blk: np.ndarray, r: int, k: int) -> float:
        off = swizzled_offset(r, k)
        bits = np.uint16(int(blk[off]) | (int(blk[off + 1]) << 8))
        return float(_bf16_to_f32(np.array([bits]))[0])

    for t in range(nt):
        nd, ns, d0, s0 = (int(x) for x in L.tile_info[t])
        for b in range(nd):
            for k in range(DENSE_BK):
                c = int(L.idx_dense[d0 + b, k])
                for r in range(L.T):
                    v = val(L.vals_dense[d0 + b], r, k)
                    if v != 0.0:
                        out[t * L.T + r, c] += v
        for b in range(ns):
            for g in range(SPARSE_BK // 4):
                for r in range(L.T):
                    wi, sh = meta_word_index(r, g)
                    nib = (int(L.meta[s0 + b, wi]) >> sh) & 0xF
                    a, bb = nib & 3, nib >> 2
                    for slot, pos in ((0, a), (1, bb)):
                        v = val(L.vals_sparse[s0 + b], r, 2 * g + slot)
                        if v != 0.0:
                            out[t * L.T + r, int(L.idx_sparse[s0 + b, 4 * g + pos])] += v
    return out


# ---------------------------------------------------------------------------------------
# a6. SpMM reference
# ---------------------------------------------------------------------------------------
def masked_weight(W_bits: np.ndarray, bitmask: np.ndarray) -> np.ndarray:
    """W ⊙ M in fp64 ([P3] 五)."""
    K = W_bits.shape[1]
    return np.where(unpack_bits(bitmask, K), _bf16_to_f64(W_bits), 0.0)


def spmm_reference(W_bits: np.ndarray, bitmask: np.ndarray, X_bits: np.ndarray,
                   rows: Optional[np.ndarray] = None) -> Tuple[np.ndarray, np.ndarray]:
    """y_ref = (W ⊙ M) X in fp64 and the error scale bound = |W ⊙ M| |X|.

    [P1] 关键设计 4: the output is the dense part plus the 2:4 part; their sum is exactly
    the masked product.  ``rows`` restricts the product to a sample of output rows.
    """
    Wm = masked_weight(W_bits if rows is None else W_bits[rows],
                       bitmask if rows is None else bitmask[rows])
    X = _bf16_to_f64(X_bits)
    return Wm @ X, np.abs(Wm) @ np.abs(X)


def hot_path(W_bits: np.ndarray, X_bits: np.ndarray, perm: np.ndarray, T: int, t_s: float,
             alpha: float = 1.0 / 32.0, v_s: Optional[float] = None) -> Dict[str, object]:
    """The whole path: importance -> boundary search (or fixed v_s) -> mask -> compress -> y."""
    I = importance(W_bits, X_bits)
    K = W_bits.shape[1]
    nt = W_bits.shape[0] // T
    if v_s is None:
        sr = boundary_search(I, perm, T, t_s, alpha)
        counts = sr.counts
    else:
        sr = None
        counts = np.tile(np.array(counts_from_vs(K, t_s, v_s), dtype=np.int32), (nt, 1))
    bitmask, region = mask(I, perm, T, counts)
    lay = compress(W_bits, bitmask, region, perm, counts, T)
    y, bound = spmm_reference(W_bits, bitmask, X_bits)
    return dict(I=I, search=sr, counts=counts, bitmask=bitmask, region=region,
                layout=lay, y=y, bound=bound)


# ---------------------------------------------------------------------------------------
# Hard-Concrete soft 2:4 mask, forward
# ---------------------------------------------------------------------------------------
HC_LOW, HC_HIGH = -0.1, 1.1   # the stretch interval (-0.1, 1.1) of [P1] 关键设计 3


def hard_concrete(log_alpha: np.ndarray, eps: np.ndarray, tau: float):
    """Hard-Concrete forward over groups of 4 consecutive elements, in fp64.

    [P1] 关键设计 3: with noise eps ~ U(0, 1) (an input here), the soft mask is
    s = sigmoid((log eps - log(1 - eps) + log alpha) / tau), stretched to (-0.1, 1.1) and
    clipped to [0, 1]: z = min(1, max(0, s * (1.1 - (-0.1)) + (-0.1))).  The two
    regularisers are mean(z) (overall sparsity) and the mean over groups of |sum of the
    group's 4 z - 2| (exactly two kept per group); the hardened mask thresholds z at 0.5.
    [reading] "at 0.5" keeps z > 0.5; the regularisers are returned as sums (before their
    means and weights): (sum z, sum over groups |sum z - 2|).
    """
    la = np.asarray(log_alpha, dtype=np.float64).ravel()
    e = np.asarray(eps, dtype=np.float64).ravel()
    if la.size % 4:
        raise ValueError("elements come in groups of 4")
    x = (np.log(e) - np.log1p(-e) + la) / float(tau)
    s = 1.0 / (1.0 + np.exp(-x))
    z = np.minimum(1.0, np.maximum(0.0, s * (HC_HIGH - HC_LOW) + HC_LOW))
    hard = (z > 0.5).astype(np.uint8)
    sums = np.array([z.sum(), np.abs(z.reshape(-1, 4).sum(axis=1) - 2.0).sum()])
    return z, hard, sums


# ---------------------------------------------------------------------------------------
# SpMM epilogue: bias, activation, bf16 output
# ---------------------------------------------------------------------------------------
ACT_NONE, ACT_RELU, ACT_SILU, ACT_GELU = 0, 1, 2, 3


def activation(x: np.ndarray, act: int) -> np.ndarray:
    """The epilogue's activations in fp64.  [reading] The pages name none; these are the
    common ones of the linears the method prunes: ReLU max(x, 0), SiLU x sigmoid(x), GELU
    x Phi(x) = x (1 + erf(x / sqrt 2)) / 2 (the erf form)."""
    x = np.asarray(x, dtype=np.float64)
    if act == ACT_NONE:
        return x.copy()
    if act == ACT_RELU:
        return np.maximum(x, 0.0)
    if act == ACT_SILU:
        return x / (1.0 + np.exp(-x))
    if act == ACT_GELU:
        erf = np.vectorize(math.erf)
        return 0.5 * x * (1.0 + erf(x / math.sqrt(2.0)))
    raise ValueError(f"activation {act}")


def spmm_epilogue_reference(y: np.ndarray, bias: Optional[np.ndarray], act: int) -> np.ndarray:
    """act(y + bias[row]) in fp64 on the SpMM's fp64 reference product ([P1] 关键设计 4:
    the one output of the dense and 2:4 parts; [reading] the bias is per output row of Y,
    i.e. per output channel of the layer)."""
    z = np.asarray(y, dtype=np.float64)
    if bias is not None:
        z = z + np.asarray(bias, dtype=np.float64)[:, None]
    return activation(z, act)


# ---------------------------------------------------------------------------------------
# Gyro-permutation (offline; produces the per-tile working order and the row order)
# ---------------------------------------------------------------------------------------
def group_retained(I_tile: np.ndarray, members: List[int]) -> float:
    """Retained 2:4 importance of one group: over the tile's rows (ascending, fp64 sum),
    the two largest of the group's four values, each added as fp64 ([P1] 关键设计 1: the
    retained second-order importance of a 2:4 group)."""
    acc = 0.0
    for r in range(I_tile.shape[0]):
        v = sorted((float(I_tile[r, c]) for c in members), reverse=True)
        acc += v[0] + v[1]
    return acc


def group_pruning_cost(I_tile: np.ndarray, members: List[int]) -> float:
    """Pruning cost of one 2:4 group: over the tile's rows (ascending, fp64 sum), the two
    smallest of the group's four values -- the importance the 2:4 selection removes
    ([P1] 关键设计 2: the assignment minimises the pruning cost).  Per row the larger of the
    two is added first: acc += (double)third + (double)fourth."""
    acc = 0.0
    for r in range(I_tile.shape[0]):
        v = sorted((float(I_tile[r, c]) for c in members), reverse=True)
        acc += v[2] + v[3]
    return acc


def balanced_kmeans(F: np.ndarray, k: int, iters: int) -> List[List[int]]:
    """Balanced K-means of S = G k points (rows of F, fp64) into G clusters of exactly k.

    [P1] 关键设计 2 names a balanced K-means over the sampled vectors.  [reading] Lloyd
    iterations from the initial partition "points G_i k .. G_i k + k - 1 form cluster i" (the
    vectors sampled from the same group); each iteration takes every cluster's centroid (the
    mean of its members, summed in ascending point order, divided by k) and reassigns the
    points by the min-cost assignment of the S points to the G k seats (cluster c's k seats)
    under the squared Euclidean distance (summed over ascending coordinates) -- which keeps
    every cluster at exactly k -- until the partition repeats or after ``iters`` iterations.
    The assignment step is a library routine (scipy's linear_sum_assignment).  Returns the
    clusters as ascending lists of point indices, cluster i's seed being group i.
    """
    from scipy.optimize import linear_sum_assignment

    S, d = F.shape
    G = S // k
    clusters = [list(range(i * k, (i + 1) * k)) for i in range(G)]
    for _ in range(iters):
        C = np.zeros((G, d))
        for c in range(G):
            acc = np.zeros(d)
            for p in clusters[c]:
                acc = acc + F[p]
            C[c] = acc / k
        cost = np.zeros((S, S))
        for p in range(S):
            for c in range(G):
                diff = F[p] - C[c]
                dist = 0.0
                for x in diff:                      # ascending coordinates
                    dist += x * x
                cost[p, c * k:(c + 1) * k] = dist
        rows, cols = linear_sum_assignment(cost)
        new = [sorted(int(p) for p, seat in zip(rows, cols) if seat // k == c) for c in range(G)]
        if new == clusters:
            break
        clusters = new
    return clusters


def gyro_input_round(I_tile: np.ndarray, band: np.ndarray, groups: np.ndarray,
                     slots: np.ndarray, kmeans_iters: int = 8):
    """One round of the in-tile input-channel gyro-permutation on a tile's 2:4 band.

    [P1] 关键设计 2: per tile, sample vectors, cluster them with a balanced K-means, then
    assign the clusters by the Hungarian algorithm on the pruning-cost matrix (smaller is
    better); the permutation leaves the product unchanged and is folded into the index.
    [reading] ``band`` is the tile's 2:4-region channels in working order (groups of 4
    consecutive entries).  The caller's random draws choose G distinct groups and, in each,
    k slots (``groups`` [G], ``slots`` [G, k]); the S = G k vectors in those slots leave them
    (sample order: group by group, slots as given).  Their features are their importance
    columns over the tile's rows; the balanced K-means groups them into G clusters of k,
    seeded by their source groups; cost[c][i] is the pruning cost of group groups[i] with its
    sampled slots, in ascending slot order, holding cluster c's vectors in ascending sample
    order.  The minimum-cost assignment (scipy's linear_sum_assignment) places the clusters;
    the new arrangement is kept only if the sampled groups' total pruning cost (fp64, in the
    order of ``groups``) does not rise ("iterated to refine": a round never makes it worse).
    Returns (band, (cost before, cost after)).
    """
    from scipy.optimize import linear_sum_assignment

    band = np.array(band, dtype=np.int64).copy()
    groups = [int(g) for g in np.asarray(groups).ravel()]
    slots = np.asarray(slots, dtype=np.int64)
    G, k = slots.shape
    vecs = [int(band[4 * g + int(s)]) for g, ss in zip(groups, slots) for s in ss]
    F = np.asarray(I_tile, dtype=np.float64)[:, vecs].T.copy()      # S x T
    clusters = balanced_kmeans(F, k, kmeans_iters)

    def members_with(i, cl):
        g = groups[i]
        m = [int(x) for x in band[4 * g:4 * g + 4]]
        for s, p in zip(sorted(int(x) for x in slots[i]), cl):
            m[s] = vecs[p]
        return m

    cost = gyro_input_cost_matrix(I_tile, band, groups, slots, clusters)
    rows, cols = linear_sum_assignment(cost)
    before = 0.0
    for i in range(G):
        g = groups[i]
        before += group_pruning_cost(I_tile, [int(x) for x in band[4 * g:4 * g + 4]])
    assign = {int(i): int(c) for c, i in zip(rows, cols)}
    after = 0.0
    for i in range(G):
        after += cost[assign[i], i]
    if after <= before:
        new = band.copy()
        for i in range(G):
            m = members_with(i, clusters[assign[i]])
            new[4 * groups[i]:4 * groups[i] + 4] = m
        return new, (before, after)
    return band, (before, before)


def gyro_input_cost_matrix(I_tile: np.ndarray, band: np.ndarray, groups, slots,
                           clusters: List[List[int]]) -> np.ndarray:
    """cost[c][i] of ``gyro_input_round``: the pruning cost of group groups[i] with its sampled
    slots (ascending) holding the vectors of cluster c (ascending sample order; a sample's
    vector is band[4 groups[g] + slots[g][j]] for sample g k + j)."""
    band = np.asarray(band, dtype=np.int64)
    groups = [int(g) for g in np.asarray(groups).ravel()]
    slots = np.asarray(slots, dtype=np.int64)
    G, k = slots.shape
    vecs = [int(band[4 * g + int(s)]) for g, ss in zip(groups, slots) for s in ss]
    cost = np.zeros((len(clusters), G))
    for c, cl in enumerate(clusters):
        for i in range(G):
            g = groups[i]
            m = [int(x) for x in band[4 * g:4 * g + 4]]
            for s, p in zip(sorted(int(x) for x in slots[i]), cl):
                m[s] = vecs[p]
            cost[c, i] = group_pruning_cost(I_tile, m)
    return cost


def band_pruning_cost(I_tile: np.ndarray, band: np.ndarray) -> float:
    """Pruning cost of a whole band: fp64 sum over its groups (ascending) of their costs."""
    acc = 0.0
    for g in range(len(band) // 4):
        acc += group_pruning_cost(I_tile, [int(x) for x in band[4 * g:4 * g + 4]])
    return acc


def tile_perm_with_band(perm_t: np.ndarray, region_t: np.ndarray, band: np.ndarray) -> np.ndarray:
    """A tile's working order with its 2:4 band rearranged: the working positions that hold
    2:4-region channels (region by channel, ascending position) take the band's channels in
    order; every other position keeps its channel.  Running the path with this order and the
    same counts groups the band as given (regions depend on the channels' scores, not on
    their positions, except for the position tie-break of equal scores)."""
    perm_t = np.asarray(perm_t, dtype=np.int64)
    pos = [j for j in range(perm_t.size) if region_t[perm_t[j]] == REGION_24]
    out = perm_t.copy()
    out[pos] = np.asarray(band, dtype=np.int64)
    return out.astype(np.int32)


def column_pruning_cost(I_rows: np.ndarray, n0: int) -> float:
    """The importance that column-vector pruning removes from a tile with these rows: the
    sum of its n0 smallest vector scores (a vector's score = its column sum over the rows,
    fp64 in ascending row order), the n0 smallest summed in ascending order of score
    (equal scores: lower channel first).  [P1] 关键设计 2 runs output-channel permutation
    before the column-vector pruning; this is that step's cost."""
    V = np.zeros(I_rows.shape[1])
    for r in range(I_rows.shape[0]):
        V = V + np.asarray(I_rows[r], dtype=np.float64)
    order = np.lexsort((np.arange(V.size), V))
    acc = 0.0
    for j in order[:n0]:
        acc += float(V[j])
    return acc


def gyro_output_round(I: np.ndarray, T: int, n0: np.ndarray, row_order: np.ndarray,
                      tiles: np.ndarray, rows: np.ndarray, kmeans_iters: int = 8):
    """One round of the output-channel gyro-permutation over a layer's tiles.

    [P1] 关键设计 2: output channels are permuted before the column-vector pruning, by the
    same sample / balanced K-means / Hungarian round.  [reading] ``row_order`` [M] lists the
    output channels in their current order (tile t holds row_order[tT .. tT+T-1]); the
    caller's draws pick G distinct tiles and k positions in each (``tiles`` [G],
    ``rows`` [G, k]); those S = G k output channels leave their positions; their features
    are their importance rows (fp64); the balanced K-means groups them into G clusters of k;
    cost[c][i] is the column-pruning cost (``column_pruning_cost`` with the tile's n0) of
    tile tiles[i] with its sampled positions, ascending, holding cluster c's channels in
    ascending sample order.  The minimum-cost assignment places the clusters; kept only if
    the sampled tiles' total cost does not rise.  Returns (row_order, (before, after)).
    The layer then computes W[row_order] and produces Y[row_order]; the next layer's index
    is translated by the inverse order (hinm_translate_index)."""
    from scipy.optimize import linear_sum_assignment

    order = np.array(row_order, dtype=np.int64).copy()
    tiles = [int(t) for t in np.asarray(tiles).ravel()]
    rows = np.asarray(rows, dtype=np.int64)
    G, k = rows.shape
    chans = [int(order[t * T + int(r)]) for t, rr in zip(tiles, rows) for r in rr]
    F = np.asarray(I, dtype=np.float64)[chans]                       # S x K
    clusters = balanced_kmeans(F, k, kmeans_iters)

    def tile_rows_with(i, cl):
        t = tiles[i]
        ch = [int(x) for x in order[t * T:(t + 1) * T]]
        for r, p in zip(sorted(int(x) for x in rows[i]), cl):
            ch[r] = chans[p]
        return ch

    cost = np.zeros((G, G))
    for c in range(G):
        for i in range(G):
            cost[c, i] = column_pruning_cost(I[tile_rows_with(i, clusters[c])], int(n0[tiles[i]]))
    ra, ca = linear_sum_assignment(cost)
    before = 0.0
    for i in range(G):
        t = tiles[i]
        before += column_pruning_cost(I[order[t * T:(t + 1) * T]], int(n0[t]))
    assign = {int(i): int(c) for c, i in zip(ra, ca)}
    after = 0.0
    for i in range(G):
        after += cost[assign[i], i]
    if after <= before:
        new = order.copy()
        for i in range(G):
            t = tiles[i]
            new[t * T:(t + 1) * T] = tile_rows_with(i, clusters[assign[i]])
        return new, (before, after)
    return order, (before, before)
