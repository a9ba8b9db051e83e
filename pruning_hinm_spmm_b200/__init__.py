"""Python binding of the HiNM C ABI (``include/hinm.h``, ``libhinm.so``).

The binding only marshals arguments: it allocates device buffers with PyTorch, passes
their raw pointers and the current CUDA stream to the C entry points of the same names,
and turns error statuses into exceptions.  Every step of the path runs in the library's
CUDA kernels; there is no CPU fallback.  If ``libhinm.so`` has not been built, importing
this package raises ImportError.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional, Tuple

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libhinm.so")

HINM_OK = 0
HINM_ERR_INVALID_ARG = 1
HINM_ERR_SHAPE = 2
HINM_ERR_ALIGNMENT = 3
HINM_ERR_UNSUPPORTED = 4
HINM_ERR_CUDA = 5
HINM_ERR_DEVICE_TIMEOUT = 6
HINM_ERR_BAD_MASK = 7
HINM_ERR_WORKSPACE = 8
HINM_LAYOUT_VERSION = 2
HINM_SPMM_TILE_PAIRS = 1   # hinm_spmm_ex flag
HINM_ACT_NONE, HINM_ACT_RELU, HINM_ACT_SILU, HINM_ACT_GELU = 0, 1, 2, 3

REGION_PRUNED, REGION_24, REGION_DENSE = 0, 1, 2

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python pruning_hinm_spmm_b200/build_lib.py` "
        "(the HiNM path has no CPU fallback)")

_lib = ctypes.CDLL(LIB_PATH)

_vp, _i32, _f64, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_double, ctypes.c_size_t
_szp = ctypes.POINTER(ctypes.c_size_t)


class hinm_layout(ctypes.Structure):
    _fields_ = [("layout_version", ctypes.c_int32), ("M", ctypes.c_int32), ("K", ctypes.c_int32),
                ("T", ctypes.c_int32), ("num_tiles", ctypes.c_int32),
                ("max_dense_blocks", ctypes.c_int32), ("max_sparse_blocks", ctypes.c_int32),
                ("tile_info", _vp), ("vals_dense", _vp), ("vals_sparse", _vp), ("meta", _vp),
                ("idx_dense", _vp), ("idx_sparse", _vp), ("run_dense", _vp), ("run_sparse", _vp)]


class hinm_layout_sizes(ctypes.Structure):
    _fields_ = [("max_dense_blocks", ctypes.c_int32), ("max_sparse_blocks", ctypes.c_int32),
                ("tile_info_bytes", _sz), ("vals_dense_bytes", _sz), ("vals_sparse_bytes", _sz),
                ("meta_bytes", _sz), ("idx_dense_bytes", _sz), ("idx_sparse_bytes", _sz),
                ("run_dense_bytes", _sz), ("run_sparse_bytes", _sz)]


_SIGS = {
    "hinm_status_string": (ctypes.c_char_p, [_i32]),
    "hinm_last_error": (ctypes.c_char_p, []),
    "hinm_abi_version": (_i32, []),
    "hinm_importance_workspace_size": (_i32, [_i32, _i32, _i32, _szp]),
    "hinm_importance": (_i32, [_vp, _vp, _i32, _i32, _i32, _vp, _vp, _sz, _vp]),
    "hinm_importance_noalloc": (_i32, [_vp, _vp, _i32, _i32, _i32, _vp, _vp]),
    "hinm_tile_stats_size": (_i32, [_i32, _i32, _i32, _szp]),
    "hinm_importance_stats": (_i32, [_vp, _vp, _i32, _i32, _i32, _i32, _vp, _vp, _sz, _vp, _sz,
                                     _vp]),
    "hinm_boundary_search_stats": (_i32, [_vp, _vp, _sz, _vp, _i32, _i32, _i32, _f64, _f64, _vp,
                                          _vp, _vp, _vp, _vp, _sz, _vp]),
    "hinm_selftest_wait_timeout": (_i32, [ctypes.c_ulonglong, _vp]),
    "hinm_counts_from_vs": (_i32, [_i32, _f64, _f64, ctypes.POINTER(ctypes.c_int32)]),
    "hinm_search_num_candidates": (_i32, [_i32, _f64, _f64, ctypes.POINTER(ctypes.c_int32)]),
    "hinm_search_workspace_size": (_i32, [_i32, _i32, _i32, _f64, _f64, _szp]),
    "hinm_boundary_search": (_i32, [_vp, _vp, _i32, _i32, _i32, _f64, _f64, _vp, _vp, _vp, _vp,
                                    _vp, _sz, _vp]),
    "hinm_boundary_search_ex": (_i32, [_vp, _vp, _vp, _sz, _vp, _i32, _i32, _i32, _i32, _f64, _f64,
                                       _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "hinm_mask_ex": (_i32, [_vp, _vp, _vp, _sz, _vp, _i32, _vp, _vp, _i32, _i32, _i32, _vp, _vp,
                            _vp, _sz, _vp]),
    "hinm_compress_ex": (_i32, [_vp, _vp, _vp, _vp, _i32, _vp, _i32, _i32, _i32,
                                ctypes.POINTER(hinm_layout), _vp, _sz, _vp]),
    "hinm_mask_workspace_size": (_i32, [_i32, _i32, _i32, _szp]),
    "hinm_mask": (_i32, [_vp, _vp, _vp, _vp, _i32, _i32, _i32, _vp, _vp, _vp, _sz, _vp]),
    "hinm_compress_size": (_i32, [_vp, _i32, _i32, _i32, ctypes.POINTER(hinm_layout_sizes)]),
    "hinm_compress_workspace_size": (_i32, [_i32, _i32, _i32, _szp]),
    "hinm_compress": (_i32, [_vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32,
                             ctypes.POINTER(hinm_layout), _vp, _sz, _vp]),
    "hinm_translate_index": (_i32, [ctypes.POINTER(hinm_layout), _vp, _vp]),
    "hinm_gyro_input_round_host": (_i32, [_vp, _i32, _i32, _vp, _i32, _vp, _vp, _i32, _i32,
                                           _i32, _vp]),
    "hinm_gyro_band_cost_host": (_i32, [_vp, _i32, _i32, _vp, _i32, _vp]),
    "hinm_gyro_cost_matrix": (_i32, [_vp, _i32, _i32, _i32, _vp, _i32, _vp, _vp, _vp, _i32, _i32,
                                      _vp, _vp]),
    "hinm_gyro_output_round_host": (_i32, [_vp, _i32, _i32, _i32, _vp, _vp, _vp, _vp, _i32, _i32,
                                            _i32, _vp]),
    "hinm_hard_concrete_forward": (_i32, [_vp, _vp, ctypes.c_longlong, ctypes.c_float, _vp, _vp,
                                          _vp, _vp]),
    "hinm_spmm": (_i32, [ctypes.POINTER(hinm_layout), _vp, _i32, _vp, _vp]),
    "hinm_spmm_ex": (_i32, [ctypes.POINTER(hinm_layout), _vp, _i32, _vp, _i32, _vp]),
    "hinm_spmm_epilogue": (_i32, [ctypes.POINTER(hinm_layout), _vp, _i32, _vp, _vp, _i32, _i32,
                                  _i32, _vp]),
    "hinm_device_status": (_i32, [_vp, ctypes.POINTER(ctypes.c_int32)]),
}
for _name, (_res, _args) in _SIGS.items():
    _f = getattr(_lib, _name)
    _f.restype = _res
    _f.argtypes = _args


def lib() -> ctypes.CDLL:
    return _lib


class HinmError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = _lib.hinm_last_error().decode(errors="replace")
        name = _lib.hinm_status_string(status).decode()
        super().__init__(f"{where}: {name}: {msg}")


def _check(status: int, where: str) -> None:
    if status != HINM_OK:
        raise HinmError(status, where)


def _torch():
    import torch
    return torch


def _stream(stream=None) -> int:
    torch = _torch()
    s = stream if stream is not None else torch.cuda.current_stream()
    return int(s.cuda_stream)


def _ptr(t) -> Optional[int]:
    return None if t is None else int(t.data_ptr())


def _size(fn, *args) -> int:
    out = ctypes.c_size_t(0)
    _check(fn(*args, ctypes.byref(out)), fn.__name__)
    return int(out.value)


def _per_tile(perm) -> int:
    """1 when perm holds one working order per tile ([M/T, K]), 0 for one shared order [K]."""
    return 1 if perm is not None and perm.dim() == 2 else 0


def _empty_bytes(nbytes: int, device):
    torch = _torch()
    return torch.empty(max(int(nbytes), 16), dtype=torch.uint8, device=device)


# ----------------------------------------------------------------------------- a1
def hinm_importance(W, X, I_out=None, workspace=None, stream=None):
    """I = fl32(fl32(w^2) * s_c), s_c = sum_n x_cn^2 (fp64, ascending).  W [M,K], X [K,N] bf16."""
    torch = _torch()
    M, K = W.shape
    N = X.shape[1]
    if I_out is None:
        I_out = torch.empty((M, K), dtype=torch.float32, device=W.device)
    if workspace is None:
        workspace = _empty_bytes(_size(_lib.hinm_importance_workspace_size, M, K, N), W.device)
    _check(_lib.hinm_importance(_ptr(W), _ptr(X), M, K, N, _ptr(I_out), _ptr(workspace),
                                workspace.numel(), _stream(stream)), "hinm_importance")
    return I_out


def hinm_tile_stats_size(M: int, K: int, T: int) -> int:
    return _size(_lib.hinm_tile_stats_size, M, K, T)


def hinm_importance_stats(W, X, T: int, I_out=None, stats_out=None, workspace=None, stream=None,
                          materialize: bool = True):
    """hinm_importance that also writes the boundary search's tile statistics (V, the tile
    maxima and the channel energies) in the same pass.  Returns (I, stats); stats is an
    opaque uint8 buffer for hinm_boundary_search / hinm_mask (..., stats=stats).  With
    materialize=False I is not written (returned as None): the search and the mask then
    recompute it from W and stats."""
    torch = _torch()
    M, K = W.shape
    N = X.shape[1]
    if I_out is None and materialize:
        I_out = torch.empty((M, K), dtype=torch.float32, device=W.device)
    if stats_out is None:
        stats_out = _empty_bytes(hinm_tile_stats_size(M, K, T), W.device)
    if workspace is None:
        workspace = _empty_bytes(_size(_lib.hinm_importance_workspace_size, M, K, N), W.device)
    _check(_lib.hinm_importance_stats(_ptr(W), _ptr(X), M, K, N, T, _ptr(I_out), _ptr(stats_out),
                                      stats_out.numel(), _ptr(workspace), workspace.numel(),
                                      _stream(stream)), "hinm_importance_stats")
    return I_out, stats_out


def tile_stats_views(stats, M: int, K: int, T: int):
    """(V fp64 [M/T, K], tile maxima int32 [M/T]) as views of a stats buffer (for tests)."""
    torch = _torch()
    nt = M // T
    v_bytes = (nt * K * 8 + 255) & ~255
    V = stats[:nt * K * 8].view(torch.float64).view(nt, K)
    pmax = stats[v_bytes:v_bytes + nt * 4].view(torch.int32)
    return V, pmax


def hinm_selftest_wait_timeout(limit_ns: int, stream=None):
    """Launches the bounded-wait self test (see hinm.h); read the outcome with
    hinm_device_status()."""
    _check(_lib.hinm_selftest_wait_timeout(int(limit_ns), _stream(stream)),
           "hinm_selftest_wait_timeout")


def hinm_importance_noalloc(W, X, I_out, stream=None):
    """hinm_importance with its scratch in the library's static per-device array
    (K <= 16384; overlapping calls on one device race).  I_out is caller-provided."""
    M, K = W.shape
    N = X.shape[1]
    _check(_lib.hinm_importance_noalloc(_ptr(W), _ptr(X), M, K, N, _ptr(I_out),
                                        _stream(stream)), "hinm_importance_noalloc")
    return I_out


# ----------------------------------------------------------------------------- counts
def hinm_counts_from_vs(K: int, t_s: float, v_s: float) -> Tuple[int, int, int]:
    out = (ctypes.c_int32 * 3)()
    _check(_lib.hinm_counts_from_vs(K, t_s, v_s, out), "hinm_counts_from_vs")
    return int(out[0]), int(out[1]), int(out[2])


# ----------------------------------------------------------------------------- a2/a3
def hinm_search_workspace_size(M, K, T, t_s, alpha) -> int:
    return _size(_lib.hinm_search_workspace_size, M, K, T, t_s, alpha)


def hinm_search_num_candidates(K: int, t_s: float, alpha: float = 1.0 / 32.0) -> int:
    out = ctypes.c_int32(0)
    _check(_lib.hinm_search_num_candidates(K, t_s, alpha, ctypes.byref(out)),
           "hinm_search_num_candidates")
    return int(out.value)


def hinm_boundary_search(I, perm, T: int, t_s: float, alpha: float = 1.0 / 32.0,
                         counts_out=None, vs_out=None, rank_out=None, workspace=None,
                         want_rank: bool = True, retained_out=None, stream=None, stats=None,
                         W=None):
    """Per-tile first-drop scan of v_s.  Returns (counts int32 [M/T,3], v_s fp64 [M/T], rank).
    ``retained_out`` (fp64 [M/T, n_cand]) optionally receives R(m) of every candidate;
    ``stats`` (from hinm_importance_stats for this I and T) spares the search its pass over
    I for V.  ``perm``: int32 [K] (every tile) or [M/T, K] (one working order per tile), or
    None (identity).  I may be None when W and stats are given (I recomputed from them)."""
    torch = _torch()
    M, K = (I if I is not None else W).shape
    nt = M // T
    dev = (I if I is not None else W).device
    if counts_out is None:
        counts_out = torch.empty((nt, 3), dtype=torch.int32, device=dev)
    if vs_out is None:
        vs_out = torch.empty((nt,), dtype=torch.float64, device=dev)
    if rank_out is None and want_rank:
        rank_out = torch.empty((nt, K), dtype=torch.int32, device=dev)
    if workspace is None:
        workspace = _empty_bytes(hinm_search_workspace_size(M, K, T, t_s, alpha), dev)
    _check(_lib.hinm_boundary_search_ex(_ptr(I), _ptr(W), _ptr(stats),
                                        0 if stats is None else stats.numel(),
                                        _ptr(perm), _per_tile(perm), M, K, T, t_s, alpha,
                                        _ptr(counts_out), _ptr(vs_out), _ptr(rank_out),
                                        _ptr(retained_out), _ptr(workspace), workspace.numel(),
                                        _stream(stream)), "hinm_boundary_search_ex")
    return counts_out, vs_out, rank_out


# ----------------------------------------------------------------------------- a4
def hinm_mask_workspace_size(M, K, T) -> int:
    return _size(_lib.hinm_mask_workspace_size, M, K, T)


def hinm_mask(I, perm, counts, T: int, rank=None, bitmask_out=None, region_out=None,
              workspace=None, stream=None, W=None, stats=None):
    """Bit-packed mask uint32 [M, ceil(K/32)] (as int32) and region int8 [M/T, K].  I may be
    None when W and stats (from hinm_importance_stats) are given."""
    torch = _torch()
    M, K = (I if I is not None else W).shape
    dev = (I if I is not None else W).device
    words = (K + 31) // 32
    if bitmask_out is None:
        bitmask_out = torch.empty((M, words), dtype=torch.int32, device=dev)
    if region_out is None:
        region_out = torch.empty((M // T, K), dtype=torch.int8, device=dev)
    if workspace is None:
        workspace = _empty_bytes(hinm_mask_workspace_size(M, K, T), dev)
    _check(_lib.hinm_mask_ex(_ptr(I), _ptr(W), _ptr(stats), 0 if stats is None else stats.numel(),
                             _ptr(perm), _per_tile(perm), _ptr(counts), _ptr(rank), M, K, T,
                             _ptr(bitmask_out), _ptr(region_out), _ptr(workspace),
                             workspace.numel(), _stream(stream)), "hinm_mask_ex")
    return bitmask_out, region_out


# ----------------------------------------------------------------------------- a5
def hinm_compress_size(M: int, K: int, T: int, counts_host=None) -> hinm_layout_sizes:
    out = hinm_layout_sizes()
    arg = None
    if counts_host is not None:
        import numpy as np
        arr = np.ascontiguousarray(counts_host, dtype=np.int32)
        arg = arr.ctypes.data
    _check(_lib.hinm_compress_size(arg, M, K, T, ctypes.byref(out)), "hinm_compress_size")
    return out


@dataclass
class HinmLayout:
    """Device buffers of one compressed HiNM weight (caller-owned torch tensors)."""
    M: int
    K: int
    T: int
    max_dense_blocks: int
    max_sparse_blocks: int
    tile_info: object    # int32 [M/T, 4]
    vals_dense: object   # int16 (bf16 bits) [blocks, 8192]
    vals_sparse: object  # int16 [blocks, 8192]
    meta: object         # int32 [blocks, 512]
    idx_dense: object    # int32 [blocks, 64]
    idx_sparse: object   # int32 [blocks, 128]
    run_dense: object    # int32 [blocks]
    run_sparse: object   # int32 [blocks]

    @classmethod
    def allocate(cls, M: int, K: int, T: int, device, counts_host=None) -> "HinmLayout":
        torch = _torch()
        sz = hinm_compress_size(M, K, T, counts_host)
        nd, ns = sz.max_dense_blocks, sz.max_sparse_blocks
        return cls(M=M, K=K, T=T, max_dense_blocks=nd, max_sparse_blocks=ns,
                   tile_info=torch.zeros((M // T, 4), dtype=torch.int32, device=device),
                   vals_dense=torch.empty((nd, 8192), dtype=torch.int16, device=device),
                   vals_sparse=torch.empty((ns, 8192), dtype=torch.int16, device=device),
                   meta=torch.empty((ns, 512), dtype=torch.int32, device=device),
                   idx_dense=torch.empty((nd, 64), dtype=torch.int32, device=device),
                   idx_sparse=torch.empty((ns, 128), dtype=torch.int32, device=device),
                   run_dense=torch.empty((nd,), dtype=torch.int32, device=device),
                   run_sparse=torch.empty((ns,), dtype=torch.int32, device=device))

    def as_c(self) -> hinm_layout:
        return hinm_layout(HINM_LAYOUT_VERSION, self.M, self.K, self.T, self.M // self.T,
                           self.max_dense_blocks, self.max_sparse_blocks,
                           _ptr(self.tile_info), _ptr(self.vals_dense), _ptr(self.vals_sparse),
                           _ptr(self.meta), _ptr(self.idx_dense), _ptr(self.idx_sparse),
                           _ptr(self.run_dense), _ptr(self.run_sparse))


def hinm_compress_workspace_size(M, K, T) -> int:
    return _size(_lib.hinm_compress_workspace_size, M, K, T)


def hinm_compress(W, bitmask, region, perm, counts, T: int, layout: Optional[HinmLayout] = None,
                  workspace=None, stream=None) -> HinmLayout:
    M, K = W.shape
    if layout is None:
        layout = HinmLayout.allocate(M, K, T, W.device)
    if workspace is None:
        workspace = _empty_bytes(hinm_compress_workspace_size(M, K, T), W.device)
    c = layout.as_c()
    _check(_lib.hinm_compress_ex(_ptr(W), _ptr(bitmask), _ptr(region), _ptr(perm),
                                 _per_tile(perm), _ptr(counts), M, K, T, ctypes.byref(c),
                                 _ptr(workspace), workspace.numel(), _stream(stream)),
           "hinm_compress_ex")
    return layout


# ----------------------------------------------------------------------------- a6
def hinm_spmm(layout: HinmLayout, X, Y_out=None, stream=None, c_layout: Optional[hinm_layout] = None,
              tile_pairs: bool = False):
    """Y (fp32 [M, N]) = W_HiNM . X (X bf16 [K, N]).  ``tile_pairs``: the caller knows every
    tile selects the same X rows (HINM_SPMM_TILE_PAIRS; a hint, the result is the same)."""
    torch = _torch()
    N = X.shape[1]
    if Y_out is None:
        Y_out = torch.empty((layout.M, N), dtype=torch.float32, device=X.device)
    c = c_layout if c_layout is not None else layout.as_c()
    if tile_pairs:
        _check(_lib.hinm_spmm_ex(ctypes.byref(c), _ptr(X), N, _ptr(Y_out), HINM_SPMM_TILE_PAIRS,
                                 _stream(stream)), "hinm_spmm_ex")
    else:
        _check(_lib.hinm_spmm(ctypes.byref(c), _ptr(X), N, _ptr(Y_out), _stream(stream)),
               "hinm_spmm")
    return Y_out


def hinm_spmm_epilogue(layout: HinmLayout, X, bias=None, activation: int = HINM_ACT_NONE,
                       out_bf16: bool = False, Y_out=None, stream=None,
                       c_layout: Optional[hinm_layout] = None, tile_pairs: bool = False):
    """Y = act(W_HiNM . X + bias[row]) as fp32 or bf16 [M, N] (bias fp32 [M] or None)."""
    torch = _torch()
    N = X.shape[1]
    if Y_out is None:
        Y_out = torch.empty((layout.M, N), dtype=torch.bfloat16 if out_bf16 else torch.float32,
                            device=X.device)
    c = c_layout if c_layout is not None else layout.as_c()
    _check(_lib.hinm_spmm_epilogue(ctypes.byref(c), _ptr(X), N, _ptr(Y_out), _ptr(bias),
                                   int(activation), 1 if out_bf16 else 0,
                                   HINM_SPMM_TILE_PAIRS if tile_pairs else 0, _stream(stream)),
           "hinm_spmm_epilogue")
    return Y_out


def hinm_translate_index(layout: HinmLayout, row_of_channel, stream=None,
                         c_layout: Optional[hinm_layout] = None):
    """Rewrites the layout's indices in place for an X whose row r holds channel sigma[r]:
    row_of_channel = sigma^-1 (device int32 [K])."""
    c = c_layout if c_layout is not None else layout.as_c()
    _check(_lib.hinm_translate_index(ctypes.byref(c), _ptr(row_of_channel), _stream(stream)),
           "hinm_translate_index")
    return layout


def hinm_hard_concrete_forward(log_alpha, eps, tau: float, z_out=None, hard_out=None,
                               sums_out=None, stream=None):
    """Hard-Concrete soft 2:4 mask (fp32 [n], groups of 4): returns (z, hard uint8 [n],
    sums fp64 [2] = (sum z, sum over groups |sum z - 2|))."""
    torch = _torch()
    n = log_alpha.numel()
    dev = log_alpha.device
    if z_out is None:
        z_out = torch.empty(n, dtype=torch.float32, device=dev)
    if hard_out is None:
        hard_out = torch.empty(n, dtype=torch.uint8, device=dev)
    if sums_out is None:
        sums_out = torch.empty(2, dtype=torch.float64, device=dev)
    _check(_lib.hinm_hard_concrete_forward(_ptr(log_alpha), _ptr(eps), n, float(tau), _ptr(z_out),
                                           _ptr(hard_out), _ptr(sums_out), _stream(stream)),
           "hinm_hard_concrete_forward")
    return z_out, hard_out, sums_out


def _host_i32(a):
    import numpy as np
    return np.ascontiguousarray(a, dtype=np.int32)


def hinm_gyro_input_round_host(I_tile, band, groups, slots, kmeans_iters: int = 8):
    """One in-tile input-channel gyro round on the host (numpy in, numpy out): I_tile fp32
    [T, K], band int32 [n] (the tile's 2:4 channels in working order), groups int32 [G],
    slots int32 [G, k].  Returns (refined band, (cost before, cost after))."""
    import numpy as np
    I_tile = np.ascontiguousarray(I_tile, dtype=np.float32)
    band = _host_i32(band).copy()
    groups = _host_i32(groups).ravel()
    slots = _host_i32(slots)
    T, K = I_tile.shape
    G, k = slots.shape
    cost = np.zeros(2, dtype=np.float64)
    _check(_lib.hinm_gyro_input_round_host(I_tile.ctypes.data, T, K, band.ctypes.data, band.size,
                                           groups.ctypes.data, slots.ctypes.data, G, k,
                                           int(kmeans_iters), cost.ctypes.data),
           "hinm_gyro_input_round_host")
    return band, (float(cost[0]), float(cost[1]))


def hinm_gyro_band_cost_host(I_tile, band) -> float:
    import numpy as np
    I_tile = np.ascontiguousarray(I_tile, dtype=np.float32)
    band = _host_i32(band)
    out = ctypes.c_double(0.0)
    _check(_lib.hinm_gyro_band_cost_host(I_tile.ctypes.data, I_tile.shape[0], I_tile.shape[1],
                                         band.ctypes.data, band.size, ctypes.byref(out)),
           "hinm_gyro_band_cost_host")
    return float(out.value)


def hinm_gyro_cost_matrix(I, T: int, bands, groups, slots, clusters, cost_out=None, stream=None):
    """The input rounds' cost matrices of every tile on the GPU: I fp32 [M, K], bands int32
    [M/T, band_len], groups [M/T, G], slots / clusters [M/T, G, k] (device tensors).
    Returns cost fp64 [M/T, G, G]."""
    torch = _torch()
    M, K = I.shape
    G, k = slots.shape[1], slots.shape[2]
    if cost_out is None:
        cost_out = torch.empty((M // T, G, G), dtype=torch.float64, device=I.device)
    _check(_lib.hinm_gyro_cost_matrix(_ptr(I), M, K, T, _ptr(bands), bands.shape[1],
                                      _ptr(groups), _ptr(slots), _ptr(clusters), G, k,
                                      _ptr(cost_out), _stream(stream)), "hinm_gyro_cost_matrix")
    return cost_out


def tile_orders_with_bands(perm, region, bands):
    """Per-tile working orders int32 [M/T, K] for the hot path's perm after the in-tile gyro
    rounds: in tile t the working positions that hold 2:4-region channels (region by channel,
    ascending position) take the refined band bands[t] in order; the other positions keep
    their channels.  perm: int32 [K] or [M/T, K]; region: int8 [M/T, K]; bands: a list of
    int32 arrays (host numpy)."""
    import numpy as np
    region = np.asarray(region)
    nt, K = region.shape
    perm = np.asarray(perm, dtype=np.int32)
    out = np.empty((nt, K), dtype=np.int32)
    for t in range(nt):
        pt = perm if perm.ndim == 1 else perm[t]
        pos = np.nonzero(region[t][pt] == REGION_24)[0]
        out[t] = pt
        out[t, pos] = np.asarray(bands[t], dtype=np.int32)
    return out


def hinm_gyro_output_round_host(I, T: int, n0, row_order, tiles, rows, kmeans_iters: int = 8):
    """One output-channel gyro round on the host: I fp32 [M, K], n0 int32 [M/T], row_order
    int32 [M], tiles int32 [G], rows int32 [G, k].  Returns (row order, (before, after))."""
    import numpy as np
    I = np.ascontiguousarray(I, dtype=np.float32)
    M, K = I.shape
    n0 = _host_i32(n0)
    order = _host_i32(row_order).copy()
    tiles = _host_i32(tiles).ravel()
    rows = _host_i32(rows)
    G, k = rows.shape
    cost = np.zeros(2, dtype=np.float64)
    _check(_lib.hinm_gyro_output_round_host(I.ctypes.data, M, K, T, n0.ctypes.data,
                                            order.ctypes.data, tiles.ctypes.data, rows.ctypes.data,
                                            G, k, int(kmeans_iters), cost.ctypes.data),
           "hinm_gyro_output_round_host")
    return order, (float(cost[0]), float(cost[1]))


def hinm_device_status(stream=None) -> int:
    out = ctypes.c_int32(0)
    _check(_lib.hinm_device_status(_stream(stream), ctypes.byref(out)), "hinm_device_status")
    return int(out.value)


def tile_pairs_hint(counts, perm, K: int) -> bool:
    """Whether hinm_spmm's ``tile_pairs`` hint holds for host-side counts (int32 [M/T, 3] or
    one row for every tile) and permutation (int32 [K] or None = identity): every tile has
    the same single region (all 2:4 or all dense) and the permutation is ascending, so every
    block of X that a tile reads is the same run of rows in every tile."""
    import numpy as np
    c = np.asarray(counts, dtype=np.int64).reshape(-1, 3)
    if not (c == c[0]).all():
        return False
    one_region = c[0, 1] == K or c[0, 2] == K
    ascending = perm is None or bool(np.array_equal(np.asarray(perm), np.arange(K)))
    return bool(one_region and ascending)


# ----------------------------------------------------------------------------- multi-GPU
def shard_tiles(M: int, T: int, world: int, rank: int) -> Tuple[int, int]:
    """Output rows [row0, row1) of W (and of Y) that rank ``rank`` of ``world`` takes when the
    tiles of one W are split across GPUs: every tile of T rows is computed independently
    (importance rows, boundary search, mask, compress and product need only the tile's rows
    of W and all of X), so rank r takes a contiguous run of whole tiles, the first
    (M/T) mod world ranks one tile more than the rest.  The ranges cover [0, M) exactly and
    in rank order; a rank may get none when there are fewer tiles than ranks."""
    if T <= 0 or M % T or world <= 0 or not 0 <= rank < world:
        raise ValueError(f"shard_tiles: M={M}, T={T}, world={world}, rank={rank}")
    nt = M // T
    base, extra = divmod(nt, world)
    t0 = rank * base + min(rank, extra)
    t1 = t0 + base + (1 if rank < extra else 0)
    return t0 * T, t1 * T


# ----------------------------------------------------------------------------- whole path
class HotPath:
    """Preallocated buffers for importance -> search -> mask -> compress -> spmm on one
    problem shape; run() enqueues the five steps on the current stream with no host sync."""

    def __init__(self, M: int, K: int, N: int, T: int, t_s: float, alpha: float = 1.0 / 32.0,
                 device="cuda", materialize_importance: bool = True):
        torch = _torch()
        self.M, self.K, self.N, self.T, self.t_s, self.alpha = M, K, N, T, t_s, alpha
        nt = M // T
        # materialize_importance=False: I is never written; the search and the mask recompute
        # it from W and the tile statistics (half the bytes per weight)
        self.I = (torch.empty((M, K), dtype=torch.float32, device=device)
                  if materialize_importance else None)
        self.counts = torch.empty((nt, 3), dtype=torch.int32, device=device)
        self.vs = torch.empty((nt,), dtype=torch.float64, device=device)
        self.rank = torch.empty((nt, K), dtype=torch.int32, device=device)
        self.bitmask = torch.empty((M, (K + 31) // 32), dtype=torch.int32, device=device)
        self.region = torch.empty((nt, K), dtype=torch.int8, device=device)
        self.layout = HinmLayout.allocate(M, K, T, device)
        self.c_layout = self.layout.as_c()
        self.Y = torch.empty((M, N), dtype=torch.float32, device=device)
        ws = max(_size(_lib.hinm_importance_workspace_size, M, K, N),
                 hinm_search_workspace_size(M, K, T, t_s, alpha),
                 hinm_mask_workspace_size(M, K, T), hinm_compress_workspace_size(M, K, T))
        self.ws = _empty_bytes(ws, device)
        self.stats = _empty_bytes(hinm_tile_stats_size(M, K, T), device)

    def run(self, W, X, perm, fixed_counts=None, stream=None, tile_pairs=False):
        """One pass of the path.  The search always runs (its ranking feeds the mask);
        ``fixed_counts`` (int32 [M/T, 3]) replaces its counts when given; ``tile_pairs`` is
        the SpMM hint (hinm_spmm)."""
        hinm_importance_stats(W, X, self.T, self.I, self.stats, self.ws, stream,
                              materialize=self.I is not None)
        hinm_boundary_search(self.I, perm, self.T, self.t_s, self.alpha, self.counts, self.vs,
                             self.rank, self.ws, stream=stream, stats=self.stats, W=W)
        counts = self.counts if fixed_counts is None else fixed_counts
        hinm_mask(self.I, perm, counts, self.T, self.rank, self.bitmask, self.region, self.ws,
                  stream, W=W, stats=self.stats)
        hinm_compress(W, self.bitmask, self.region, perm, counts, self.T, self.layout, self.ws,
                      stream)
        hinm_spmm(self.layout, X, self.Y, stream, self.c_layout, tile_pairs)
        return self.Y
