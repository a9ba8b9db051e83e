"""Seeded synthetic inputs for the HiNM hot path.

This module only draws random numbers and rounds them to bf16; it holds none of
the pruning or matmul arithmetic.  Both the CPU oracle (``oracle/``) and the CUDA
path (``pruning_hinm_spmm_b200``) consume the exact bytes produced here.

The pages' workloads are LLaMA-2-7B / DeiT / BERT linears on public suites
(FlexHiNM-GP notes, "主实验表格" table); none of those weights or datasets are used.
The synthetic stand-ins are LLaMA-2-7B-*shaped* linears:

* W ~ N(0, 0.02) per element, optionally with a Bernoulli(p) outlier mask that
  multiplies the drawn value by 10 before rounding;
* X ~ N(0, 1);
* pi = a seeded random permutation of the K input channels (or the identity).

Draw order from ``numpy.random.Generator(PCG64(seed))``: W (fp32 normal), then X,
then pi, then the outlier mask.  Rounding to bf16 is round-to-nearest-even on the
fp32 bit pattern.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Optional

import numpy as np


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (round-to-nearest-even), returning uint16 bit patterns."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    # finite values stay below 0xFF800000, so the 32-bit sum cannot wrap
    r = (u + (np.uint32(0x7FFF) + lsb)) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns (uint16) to fp32 values (exact)."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


@dataclass
class Workload:
    """One synthetic problem: W (M x K), X (K x N), tile height T, permutation, sparsity."""
    name: str
    M: int
    K: int
    N: int
    T: int
    W_bits: np.ndarray          # uint16 [M, K], bf16 bit patterns, row-major
    X_bits: np.ndarray          # uint16 [K, N], bf16 bit patterns, row-major
    perm: np.ndarray            # int32 [K]; working position j holds input channel perm[j]
    t_s: float                  # target overall sparsity
    v_s: Optional[float]        # fixed vector-sparsity boundary, or None = searched
    alpha: float = 1.0 / 32.0   # boundary-search step
    meta: dict = field(default_factory=dict)


def make_workload(name: str, M: int, K: int, N: int, T: int, *, seed: int,
                  t_s: float, v_s: Optional[float], w_std: float = 0.02,
                  outlier_frac: float = 0.0, outlier_scale: float = 10.0,
                  random_perm: bool = False, alpha: float = 1.0 / 32.0) -> Workload:
    rng = np.random.Generator(np.random.PCG64(seed))
    W = rng.standard_normal((M, K), dtype=np.float32) * np.float32(w_std)
    X = rng.standard_normal((K, N), dtype=np.float32)
    if random_perm:
        perm = rng.permutation(K).astype(np.int32)
    else:
        perm = np.arange(K, dtype=np.int32)
    if outlier_frac > 0.0:
        out = rng.random((M, K), dtype=np.float32) < np.float32(outlier_frac)
        W = np.where(out, W * np.float32(outlier_scale), W).astype(np.float32)
    return Workload(name=name, M=M, K=K, N=N, T=T,
                    W_bits=f32_to_bf16_bits(W), X_bits=f32_to_bf16_bits(X),
                    perm=perm, t_s=t_s, v_s=v_s, alpha=alpha,
                    meta=dict(seed=seed, w_std=w_std, outlier_frac=outlier_frac,
                              random_perm=random_perm))


# The five workloads the hot path is specified on (LLaMA-2-7B-shaped linears).
def tiny_hinm(seed: int = 0) -> Workload:
    """W 256x256, X 256x16, tile 64 rows, t_s=0.5, v_s=0.2 (p_s=0.75)."""
    return make_workload("tiny_hinm_256x256x16_T64", 256, 256, 16, 64, seed=seed,
                         t_s=0.5, v_s=0.2)


def pure24(seed: int = 0, M: int = 4096, K: int = 4096, N: int = 2048) -> Workload:
    """W 4096x4096 with 1% x10 outliers, X 4096x2048, tile 128, t_s=0.5, v_s=0 (pure 2:4)."""
    return make_workload(f"pure24_{M}x{K}x{N}_T128", M, K, N, 128, seed=seed,
                         t_s=0.5, v_s=0.0, outlier_frac=0.01)


def hinm_up_proj(seed: int = 0, M: int = 11008, K: int = 4096, N: int = 4096) -> Workload:
    """W 11008x4096, X 4096x4096, tile 128, t_s=0.75, v_s=0.6, seeded input permutation."""
    return make_workload(f"hinm_up_{M}x{K}x{N}_T128", M, K, N, 128, seed=seed,
                         t_s=0.75, v_s=0.6, random_perm=True)


def decode_down_proj(seed: int = 0, M: int = 4096, K: int = 11008, N: int = 16) -> Workload:
    """W 4096x11008, X 11008x16, tile 128, t_s=0.625, v_s=0.4 (HBM-bound decode)."""
    return make_workload(f"decode_down_{M}x{K}x{N}_T128", M, K, N, 128, seed=seed,
                         t_s=0.625, v_s=0.4)


LLAMA7B_LINEARS = {  # name: (M = out_features, K = in_features), seed offset
    "q": (4096, 4096, 0), "k": (4096, 4096, 1), "v": (4096, 4096, 2), "o": (4096, 4096, 3),
    "gate": (11008, 4096, 4), "up": (11008, 4096, 5), "down": (4096, 11008, 6),
}


def llama_sweep_layer(layer: int, linear: str, N: int, t_s: float) -> Workload:
    """One linear of the 32-layer LLaMA-2-7B-shaped sweep; v_s comes from the search."""
    M, K, off = LLAMA7B_LINEARS[linear]
    return make_workload(f"llama7b_L{layer}_{linear}_{M}x{K}x{N}_ts{t_s}", M, K, N, 128,
                         seed=1000 * layer + off, t_s=t_s, v_s=None)


def custom(M: int, K: int, N: int, T: int, *, seed: int, t_s: float,
           v_s: Optional[float], random_perm: bool = False, outlier_frac: float = 0.0,
           alpha: float = 1.0 / 32.0) -> Workload:
    """Small seeded case for parity tests (several tiles, ragged K/N tails)."""
    return make_workload(f"custom_{M}x{K}x{N}_T{T}_s{seed}", M, K, N, T, seed=seed,
                         t_s=t_s, v_s=v_s, random_perm=random_perm,
                         outlier_frac=outlier_frac, alpha=alpha)


def integer_workload(M: int, K: int, N: int, T: int, *, seed: int, t_s: float,
                     v_s: Optional[float], random_perm: bool = False) -> Workload:
    """W, X drawn from {-2,...,2} (exact in bf16): every partial sum is an exact integer."""
    rng = np.random.Generator(np.random.PCG64(seed))
    W = rng.integers(-2, 3, size=(M, K)).astype(np.float32)
    X = rng.integers(-2, 3, size=(K, N)).astype(np.float32)
    perm = (rng.permutation(K) if random_perm else np.arange(K)).astype(np.int32)
    return Workload(name=f"int_{M}x{K}x{N}_T{T}_s{seed}", M=M, K=K, N=N, T=T,
                    W_bits=f32_to_bf16_bits(W), X_bits=f32_to_bf16_bits(X), perm=perm,
                    t_s=t_s, v_s=v_s, meta=dict(seed=seed, integer=True))
