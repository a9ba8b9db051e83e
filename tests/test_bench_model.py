"""The algorithmic FLOP / byte model and the roofline arithmetic bench.py reports (CPU only)."""
import os
import sys

import numpy as np
import pytest

import hinm_inputs as hi
from oracle import hinm_oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402

PEAKS = {"hbm_gbs": 6542.1, "bf16_tflops": 1663.1}


def test_pure24_model_and_tensor_roofline():
    M, K, N, T = 4096, 4096, 2048, 128
    counts = np.tile(np.array(O.counts_from_vs(K, 0.5, 0.0), dtype=np.int64), (M // T, 1))
    m = bench.workload_model(M, K, N, T, counts)
    assert m["kept"] == M * K // 2                       # overall sparsity exactly t_s
    assert m["flops_eff"] == 2.0 * M * K * N
    assert m["flops_dense"] == 0.0 and m["flops_sparse_eq"] == m["flops_eff"]
    assert m["flops_actual"] == m["flops_eff"] / 2
    # X once, Y once, kept values, 2 bits per kept value, one index per vector
    want = 2.0 * M * K / 2 + M * K / 8.0 + 4.0 * (M // T) * K + 2.0 * K * N + 4.0 * M * N
    assert m["bytes"]["spmm"] == pytest.approx(want)
    t_roof = m["flops_eff"] / (2 * PEAKS["bf16_tflops"] * 1e12)    # 2:4 at twice dense
    bound, ach, peak, unit, frac = bench.roofline_for("spmm", 2 * t_roof, m, PEAKS, "measured")
    assert bound == "tensor" and unit == "TFLOP/s"
    assert peak == pytest.approx(2 * PEAKS["bf16_tflops"])
    assert frac == pytest.approx(0.5)
    assert ach == pytest.approx(m["flops_eff"] / (2 * t_roof) / 1e12)


def test_mixed_peak_and_hbm_bound_decode():
    # up-proj counts: the tensor peak is the FLOP-weighted mix of dense and 2:4
    M, K, N, T = 11008, 4096, 4096, 128
    counts = np.tile(np.array(O.counts_from_vs(K, 0.75, 0.6)), (M // T, 1))
    m = bench.workload_model(M, K, N, T, counts)
    t_t = m["flops_dense"] / 1663.1e12 + m["flops_sparse_eq"] / (2 * 1663.1e12)
    bound, ach, peak, unit, frac = bench.roofline_for("spmm", t_t, m, PEAKS, "measured")
    assert bound == "tensor" and frac == pytest.approx(1.0)
    assert 1663.1 < peak < 2 * 1663.1
    # decode: 16 tokens make the same weights HBM-bound
    M, K, N = 4096, 11008, 16
    counts = np.tile(np.array(O.counts_from_vs(K, 0.625, 0.4)), (M // T, 1))
    m = bench.workload_model(M, K, N, T, counts)
    t_h = m["bytes"]["spmm"] / (PEAKS["hbm_gbs"] * 1e9)
    bound, ach, peak, unit, frac = bench.roofline_for("spmm", 2 * t_h, m, PEAKS, "measured")
    assert bound == "hbm" and unit == "GB/s" and frac == pytest.approx(0.5)


def test_model_kept_matches_the_oracle_mask():
    w = hi.custom(256, 512, 16, 64, seed=21, t_s=0.625, v_s=0.25, random_perm=True)
    I = O.importance(w.W_bits, w.X_bits)
    counts = np.tile(np.array(O.counts_from_vs(w.K, w.t_s, w.v_s)), (w.M // w.T, 1))
    bm, _ = O.mask(I, w.perm, w.T, counts)
    kept_bits = int(sum(bin(int(x)).count("1") for x in bm.view(np.uint32).ravel()))
    assert bench.workload_model(w.M, w.K, w.N, w.T, counts)["kept"] == kept_bits
