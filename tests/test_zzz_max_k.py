"""The whole path at the widest inputs the ABI accepts: K = 16384, its largest, and
K = 13824, the intermediate width of LLaMA-2-13B-shaped layers; and K = 8448 with tiles of
64 rows, the per-block packing of long rows with half-filled blocks.

Above K = 12288 the kernels take the configurations that narrower shapes never reach:
- the search stages one row of importances per CTA (`band_sum_kernel<1>`);
- the mask from a materialized I stages one row (`bitmask_kernel<1>`), the mask from W two
  (`bitmask_w_kernel<2>`);
- the ranking sorts up to 16 chunks per tile in 160 KB of shared memory;
- packing gathers one block per CTA (`pack_kernel`).
At K = 8448 with T = 64, `pack_kernel` (every K above 8192) fills only the first 64 of each
block's 128 rows, a combination no other case reaches.

Each width runs with and without the materialized importance, with a seeded random
permutation and a fixed v_s (mixed dense, 2:4 and pruned regions); the search runs and is
compared in full. Counts, v_s, rank and every R(m), the regions, the bitmask and every layout
byte must be the oracle's bit for bit, and Y must be within the product tolerance
(FlexHiNM-GP notes, 关键设计 1, 2 and 4).

The file sorts last so that, under `-x`, every other test has run before these.
"""
import numpy as np
import pytest

import hinm_inputs as hi
from oracle import hinm_oracle as O

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

from test_gpu_parity import check_y, layout_equal, run_path  # noqa: E402
from test_gpu_imp_from_w import _w_path  # noqa: E402

# (M, K, N, T)
SHAPES = [(256, 13824, 24, 128), (256, 16384, 24, 128), (128, 8448, 40, 64)]
IDS = [f"K{k}_T{t}" for _, k, _, t in SHAPES]
V_S = 0.4
_ORACLE = {}


@pytest.fixture(scope="module")
def H():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import pruning_hinm_spmm_b200 as H
    return H


def _workload(shape):
    M, K, N, T = shape
    return hi.custom(M, K, N, T, seed=17, t_s=0.625, v_s=None, random_perm=True)


def _oracle(w):
    """The oracle's run on workload w (search, then the mask, layout and product with the
    fixed-v_s counts), computed once per shape."""
    key = (w.M, w.K, w.N, w.T)
    if key not in _ORACLE:
        I_ref = O.importance(w.W_bits, w.X_bits)
        sr = O.boundary_search(I_ref, w.perm, w.T, w.t_s, w.alpha)
        nt = w.M // w.T
        counts = np.tile(np.array(O.counts_from_vs(w.K, w.t_s, V_S), dtype=np.int32), (nt, 1))
        bm, reg = O.mask(I_ref, w.perm, w.T, counts)
        L = O.compress(w.W_bits, bm, reg, w.perm, counts, w.T)
        y, bound = O.spmm_reference(w.W_bits, bm, w.X_bits)
        _ORACLE[key] = dict(I=I_ref, sr=sr, counts=counts, bitmask=bm, region=reg, layout=L,
                            y=y, bound=bound)
    return _ORACLE[key]


def _compare(g, ref, counts_used):
    sr = ref["sr"]
    np.testing.assert_array_equal(g["counts"], sr.counts)
    np.testing.assert_array_equal(np.asarray(g["vs"]), np.asarray(sr.v_s))
    np.testing.assert_array_equal(g["rank"], sr.rank)
    np.testing.assert_array_equal(g["R"], np.array(sr.R))
    np.testing.assert_array_equal(counts_used, ref["counts"])
    np.testing.assert_array_equal(g["region"], ref["region"])
    np.testing.assert_array_equal(g["bitmask"], ref["bitmask"])
    check_y(g["Y"], ref["y"], ref["bound"])


@pytest.mark.parametrize("shape", SHAPES, ids=IDS)
def test_widest_inputs_with_materialized_importance(H, shape):
    w = _workload(shape)
    ref = _oracle(w)
    g = run_path(H, w, V_S)
    np.testing.assert_array_equal(g["I"].view(np.uint32), ref["I"].view(np.uint32))
    _compare(g, ref, g["counts_used"])
    layout_equal(g["layout"], ref["layout"])


@pytest.mark.parametrize("shape", SHAPES, ids=IDS)
def test_widest_inputs_from_w(H, shape):
    w = _workload(shape)
    ref = _oracle(w)
    g = _w_path(H, w, w.perm, V_S)
    _compare(g, ref, g["used"])
    layout_equal(g["L"], ref["layout"])
