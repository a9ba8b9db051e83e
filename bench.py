#!/usr/bin/env python
"""Benchmark of the HiNM hot path on B200: importance -> boundary search -> mask ->
compress -> SpMM, one pass per step.  The headline workload is the HiNM up-projection
(W 11008x4096 bf16 ~N(0,0.02), X 4096x4096 bf16 ~N(0,1), tile 128 rows, t_s = 0.75 with the
fixed boundary v_s = 0.6, a seeded input-channel permutation folded into the index);
the pure 2:4 (4096x4096x2048) and the decode down-projection (4096x11008x16) workloads are
measured in the same run as extra keys.

Prints ONE JSON line (rank 0).  `value` is the effective (dense-equivalent) TFLOP/s of the
whole step, 2*M*K*N of the whole problem / max-over-ranks step time; the per-kernel
breakdown, the roofline of the SpMM, the end-to-end number through host buffers and the
CPU oracle baseline are extra keys.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl {hinm,reference}]
Multi-GPU: launched with torch.distributed.run, one rank per GPU; the tiles of the one W
are split across the ranks (contiguous runs of whole tiles, X replicated, each rank writes
its row block of Y; --gather-y adds the NCCL all-gather of Y to every step): strong scaling.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import hinm_inputs as hi  # noqa: E402

METRIC = "HiNM SpMM TFLOP/s (eff.) and HBM GB/s, % of 2:4-sparse/HBM roofline"
WORKLOADS = {  # name -> seeded generator (seed 0: every rank draws the same problem)
    "pure24": lambda: hi.pure24(seed=0),
    "tiny": lambda: hi.tiny_hinm(seed=0),
    "up": lambda: hi.hinm_up_proj(seed=0),
    "decode": lambda: hi.decode_down_proj(seed=0),
}
UNIT = "TFLOP/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def max_over_ranks(x: float, dist, device) -> float:
    """The largest of every rank's x (the job's time is its slowest rank's); x itself on
    one rank.  Every rank must call it at the same point."""
    if dist is None:
        return x
    import torch
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_value(flops_total: float, t_max: float) -> float:
    """Whole-job throughput in TFLOP/s: the whole problem's FLOPs over the slowest rank's
    time (the ranks split one problem's tiles)."""
    return flops_total / t_max / 1e12


def gather_rows(Y_shard, M: int, T: int, world: int, dist, shard_tiles):
    """The optional collective of the tile-sharded run: every rank's row block of Y, padded
    to the largest shard, all-gathered (NCCL on GPUs, gloo on CPU) and cut back into the full
    M x N matrix in rank order.  Every rank calls it at the same point."""
    import torch
    rows = [shard_tiles(M, T, world, r) for r in range(world)]
    most = max(r1 - r0 for r0, r1 in rows)
    N = Y_shard.shape[1]
    pad = torch.zeros((most, N), dtype=Y_shard.dtype, device=Y_shard.device)
    pad[:Y_shard.shape[0]] = Y_shard
    parts = [torch.empty_like(pad) for _ in range(world)]
    dist.all_gather(parts, pad)
    return torch.cat([parts[r][:r1 - r0] for r, (r0, r1) in enumerate(rows)], dim=0)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ------------------------------------------------------------------ clocks sampling
class ClockSampler:
    """SM clock and throttle reasons of this rank's GPU, polled through NVML every few
    milliseconds while the timed region runs (read-only queries)."""
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, torch_device_index: int, period_s: float = 0.002):
        self.dev = torch_device_index
        self.period = period_s
        self.samples = []
        self.max_mhz = None
        self.err = None
        self._stop = threading.Event()
        self._thread = None
        self._h = None

    def start(self):
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            props = torch.cuda.get_device_properties(self.dev)
            self._h = pynvml.nvmlDeviceGetHandleByUUID("GPU-" + str(props.uuid))
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self._nvml = pynvml
        except Exception as e:  # noqa: BLE001 - sampling is best effort, reported below
            self.err = f"{type(e).__name__}: {e}"
            return
        self._thread = threading.Thread(target=self._run, daemon=True)
        self._thread.start()

    def _run(self):
        n = self._nvml
        while not self._stop.is_set():
            try:
                sm = n.nvmlDeviceGetClockInfo(self._h, n.NVML_CLOCK_SM)
                rs = n.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                self.samples.append((sm, rs))
            except Exception as e:  # noqa: BLE001
                self.err = f"{type(e).__name__}: {e}"
                return
            time.sleep(self.period)

    def stop(self):
        self._stop.set()
        if self._thread:
            self._thread.join(timeout=5)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unsampled"],
                    "samples": 0, "error": self.err}
        reasons = sorted({name for _, r in self.samples for bit, name in self.REASONS.items()
                          if r & bit})
        return {"sm_mhz": statistics.median(sm for sm, _ in self.samples),
                "sm_max_mhz": self.max_mhz, "reasons": reasons, "samples": len(self.samples)}


# ------------------------------------------------------------------ workload accounting
def workload_model(M, K, N, T, counts):
    """Algorithmic FLOPs and bytes per step from the region counts actually used."""
    n0, n24, n4 = (int(x) for x in np.asarray(counts).sum(axis=0))  # summed over tiles
    nt = M // T
    kept = T * (n4 + n24 // 2)                       # kept weights
    flops_eff = 2.0 * M * K * N                      # dense-equivalent
    flops_dense = 2.0 * T * n4 * N                   # real dense-region MACs x2
    flops_sparse_eq = 2.0 * T * n24 * N              # 2:4 region, dense-equivalent
    spmm_bytes = (2.0 * kept + T * n24 / 8.0 + 4.0 * (n4 + n24) + 2.0 * K * N + 4.0 * M * N)
    return dict(
        flops_eff=flops_eff, flops_actual=2.0 * kept * N, flops_dense=flops_dense,
        flops_sparse_eq=flops_sparse_eq, kept=kept,
        # the step does not materialize I: the importance pass reads W and X and writes the
        # tile statistics (V, tile maxima, s_c); the search and the mask read W (2 B per
        # weight) and recompute the importance from it
        bytes=dict(importance=2.0 * M * K + 2.0 * K * N + 8.0 * nt * K + 4.0 * nt + 4.0 * K,
                   search=2.0 * M * K + 4.0 * nt * K,
                   mask=2.0 * M * K + M * ((K + 31) // 32) * 4.0 + nt * K,
                   compress=2.0 * M * K + M * ((K + 31) // 32) * 4.0 + nt * K
                   + 2.0 * kept + T * n24 / 8.0 + 4.0 * (n4 + n24),
                   spmm=spmm_bytes))


def roofline_for(phase, t_s, model, peaks, peak_kind):
    """(bound, achieved, peak, unit, frac) of one kernel phase."""
    hbm = peaks["hbm_gbs"]
    if phase == "spmm":
        # tensor time at the measured dense bf16 peak and twice it for the 2:4 region
        # (the nominal 2:4 ratio); report the dense-equivalent rate against the mix.
        dense_peak = peaks["bf16_tflops"]
        t_tensor = (model["flops_dense"] / (dense_peak * 1e12)
                    + model["flops_sparse_eq"] / (2.0 * dense_peak * 1e12))
        t_hbm = model["bytes"]["spmm"] / (hbm * 1e9)
        if t_tensor >= t_hbm:
            eff_peak = (model["flops_dense"] + model["flops_sparse_eq"]) / t_tensor / 1e12
            achieved = (model["flops_dense"] + model["flops_sparse_eq"]) / t_s / 1e12
            return "tensor", achieved, eff_peak, "TFLOP/s", achieved / eff_peak
        achieved = model["bytes"]["spmm"] / t_s / 1e9
        return "hbm", achieved, hbm, "GB/s", achieved / hbm
    achieved = model["bytes"][phase] / t_s / 1e9
    return "hbm", achieved, hbm, "GB/s", achieved / hbm


# ------------------------------------------------------------------ reference arm
def cpu_oracle_sample(w, tiles_n: int):
    """Run the CPU oracle on `tiles_n` tiles of the workload; returns (seconds, flops_eff)."""
    from oracle import hinm_oracle as O
    M, K, N, T = w.M, w.K, w.N, w.T
    tiles = list(range(tiles_n))
    rows = np.arange(0, tiles_n * T)
    t0 = time.perf_counter()
    I = np.zeros((M, K), dtype=np.float32)
    I[rows] = O.importance_rows(w.W_bits, w.X_bits, rows)
    sr = O.boundary_search(I, w.perm, T, w.t_s, w.alpha, tiles=tiles)
    counts = sr.counts  # the GPU arm's rule: a fixed boundary's counts where the workload has one
    if w.v_s is not None:
        counts = np.tile(np.array(O.counts_from_vs(K, w.t_s, w.v_s), dtype=np.int32), (M // T, 1))
    bm, reg = O.mask(I, w.perm, T, counts, tiles=tiles)
    O.compress(w.W_bits, bm, reg, w.perm, counts, T, tiles=tiles)
    O.spmm_reference(w.W_bits, bm, w.X_bits, rows=rows)
    dt = time.perf_counter() - t0
    return dt, 2.0 * len(rows) * K * N


def cpu_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def run_reference(args, w):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from threadpoolctl import threadpool_limits
    cores = cpu_cores()
    tiles_n = 2
    with threadpool_limits(limits=cores):
        for _ in range(args.warmup):
            cpu_oracle_sample(w, 1)
        times, flops = [], 0.0
        for _ in range(args.steps):
            dt, fl = cpu_oracle_sample(w, tiles_n)
            times.append(dt)
            flops = fl
    t = statistics.mean(times)
    value = flops / t / 1e12
    sample = (f"{tiles_n} of {w.M // w.T} tiles ({tiles_n * w.T} output rows) of {w.name} per step: "
              "channel energies over all of X, then importance, search, mask, compress and the "
              "fp64 masked product for those rows")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": t * 1e3, "higher_is_better": True,
            "scaling": "strong", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.name, "M": w.M, "K": w.K, "N": w.N, "T": w.T,
                       "t_s": w.t_s, "alpha": w.alpha},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ LLaMA-shaped sweep
SWEEP_SHAPES = (("q", 4), ("gate", 2), ("down", 1))  # distinct shapes, linears per layer


def run_sweep(args):
    """The LLaMA-2-7B-shaped layer sweep on one GPU: the three distinct linear shapes of
    layer 0 (q/k/v/o 4096x4096, gate/up 11008x4096, down 4096x11008), each at every
    N in {16, 512, 4096} and t_s in {0.5, 0.625, 0.75} with the boundary from the search.
    Each case times K graph-replayed steps (L2 flushed between them); a layer's time is
    4 x q + 2 x gate + 1 x down.  `value` = the layers' dense-equivalent FLOPs over their
    total time."""
    import torch
    import pruning_hinm_spmm_b200 as H
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    sampler = ClockSampler(0)
    sampler.start()
    rows, tot_flops, tot_s = [], 0.0, 0.0
    for t_s in (0.5, 0.625, 0.75):
        for N in (16, 512, 4096):
            layer_s, layer_flops, per = 0.0, 0.0, {}
            for name, mult in SWEEP_SHAPES:
                w = hi.llama_sweep_layer(0, name, N, t_s)
                M, K, T = w.M, w.K, w.T
                W = torch.from_numpy(w.W_bits.view(np.int16)).to(dev).view(torch.bfloat16)
                X = torch.from_numpy(w.X_bits.view(np.int16)).to(dev).view(torch.bfloat16)
                perm = torch.from_numpy(w.perm).to(dev)
                hp = H.HotPath(M, K, N, T, w.t_s, w.alpha, device=dev,
                               materialize_importance=False)
                for _ in range(args.warmup):
                    hp.run(W, X, perm)
                torch.cuda.synchronize()
                graph = torch.cuda.CUDAGraph()
                with torch.cuda.graph(graph):
                    hp.run(W, X, perm)
                torch.cuda.synchronize()
                ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)]
                      for _ in range(args.steps)]
                for k in range(args.steps):
                    flush.zero_()
                    ev[k][0].record(stream)
                    graph.replay()
                    ev[k][1].record(stream)
                torch.cuda.synchronize()
                if H.hinm_device_status() != 0:
                    raise RuntimeError(f"device status after {w.name}")
                t = statistics.mean(e[0].elapsed_time(e[1]) * 1e-3 for e in ev)
                del graph
                per[name] = {"M": M, "K": K, "ms": t * 1e3,
                             "v_s_searched": sorted(set(np.round(hp.vs.cpu().numpy(), 6).tolist()))}
                layer_s += mult * t
                layer_flops += mult * 2.0 * M * K * N
            rows.append({"t_s": t_s, "N": N, "layer_ms": layer_s * 1e3,
                         "layer_tflops_eff": layer_flops / layer_s / 1e12, "by_shape": per})
            tot_flops += layer_flops
            tot_s += layer_s
    sampler.stop()
    line = {"metric": METRIC, "value": tot_flops / tot_s / 1e12, "unit": UNIT, "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": tot_s * 1e3 / len(rows), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": "llama7b_layer0_sweep",
                       "step": "importance+search+mask+compress+spmm per linear, searched v_s",
                       "layer": "4 x (4096x4096) + 2 x (11008x4096) + 1 x (4096x11008)",
                       "l2": "flushed between timed steps (256 MB write)",
                       "step_exec": "CUDA graph replay"},
            "sweep": rows, "clocks": sampler.summary()}
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ GPU arm
def time_index_translate(H, hp, K, stream, reps=20):
    """The cross-layer index translation on this workload's layout, with the identity map
    (every index rewritten to itself, every run flag recomputed): CUDA events over `reps`
    back-to-back calls after 3 untimed ones.  Bytes: 4 B read + 4 B written per index entry,
    4 B read from the map per entry, 4 B written per block."""
    import torch
    ident = torch.arange(K, dtype=torch.int32, device=hp.counts.device)
    info = hp.layout.tile_info.cpu().numpy()
    nd, ns = int(info[:, 0].sum()), int(info[:, 1].sum())
    entries = nd * 64 + ns * 128
    for _ in range(3):
        H.hinm_translate_index(hp.layout, ident, None, hp.c_layout)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(reps):
        H.hinm_translate_index(hp.layout, ident, None, hp.c_layout)
    e1.record(stream)
    torch.cuda.synchronize()
    st = H.hinm_device_status()
    if st != 0:
        raise RuntimeError(f"device status {st} after the index translation")
    t = e0.elapsed_time(e1) / 1e3 / reps
    nbytes = entries * 12 + (nd + ns) * 4
    return {"us_per_call": t * 1e6, "index_entries": entries, "blocks": nd + ns,
            "gbs": nbytes / t / 1e9, "kernel": "translate_index_kernel", "launches": 1,
            "note": "identity map on the step's layout; back-to-back calls (L2-warm)"}


def time_epilogue(H, hp, X, M, N, tile_pairs, flush, stream, reps=10):
    """The SpMM with the fused epilogue (per-row bias, GELU, bf16 Y) against the plain fp32
    SpMM on this step's layout: each call timed alone by CUDA events after the 256 MB L2
    flush, the median of `reps`; Y bytes halve (4 -> 2 per output)."""
    import torch
    bias = torch.linspace(-0.1, 0.1, M, device=X.device, dtype=torch.float32)
    yb = torch.empty((M, N), dtype=torch.bfloat16, device=X.device)

    def timed(fn):
        ts = []
        for i in range(reps + 2):
            flush.fill_(i & 0xFF)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            fn()
            e1.record(stream)
            torch.cuda.synchronize()
            if i >= 2:
                ts.append(e0.elapsed_time(e1) * 1e3)
        return float(np.median(ts))

    t_plain = timed(lambda: H.hinm_spmm(hp.layout, X, hp.Y, None, hp.c_layout, tile_pairs))
    t_epi = timed(lambda: H.hinm_spmm_epilogue(hp.layout, X, bias, H.HINM_ACT_GELU, True, yb,
                                               None, hp.c_layout, tile_pairs))
    st = H.hinm_device_status()
    if st != 0:
        raise RuntimeError(f"device status {st} after the epilogue timing")
    return {"us_plain_fp32": t_plain, "us_bias_gelu_bf16": t_epi,
            "y_bytes_fp32": 4 * M * N, "y_bytes_bf16": 2 * M * N,
            "kernel": "same SpMM kernel, epilogue fused", "launches": 1,
            "note": "one call per timing after the L2 flush; median of %d" % reps}


def time_dense_context(M, K, N, flush, stream, reps=10):
    """Context, not a target: a dense bf16 GEMM of the same shape (torch.matmul, cuBLAS, fp32
    accumulation, bf16 output) on random operands, one call per timing after the L2 flush,
    the median of `reps`."""
    import torch
    A = torch.randn(M, K, device="cuda").to(torch.bfloat16)
    B = torch.randn(K, N, device="cuda").to(torch.bfloat16)
    ts = []
    for i in range(reps + 2):
        flush.fill_(i & 0xFF)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        torch.matmul(A, B)
        e1.record(stream)
        torch.cuda.synchronize()
        if i >= 2:
            ts.append(e0.elapsed_time(e1) * 1e3)
    t = float(np.median(ts))
    return {"torch_matmul_dense_bf16_us": t, "tflops": 2.0 * M * K * N / (t * 1e-6) / 1e12,
            "note": "dense W (no pruning) through cuBLAS, same M, K, N; context only"}


def time_sparse24_context(M, K, N, flush, stream, reps=10):
    """Context, not a target: torch's own 2:4 semi-structured product (torch.sparse's
    to_sparse_semi_structured, whatever backend this torch build uses) on a random W with the
    2:4 pattern, same M, K, N, one call per timing after the L2 flush, the median of `reps`.
    Reported as unavailable, with the reason, when this torch build has no such kernel here."""
    import torch
    try:
        from torch.sparse import to_sparse_semi_structured
        keep = torch.tensor([1, 1, 0, 0], dtype=torch.bfloat16, device="cuda").repeat(M, K // 4)
        A = to_sparse_semi_structured((torch.randn(M, K, device="cuda") * keep).to(torch.bfloat16))
        B = torch.randn(K, N, device="cuda").to(torch.bfloat16)
        torch.mm(A, B)
        torch.cuda.synchronize()
        ts = []
        for i in range(reps + 2):
            flush.fill_(i & 0xFF)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            torch.mm(A, B)
            e1.record(stream)
            torch.cuda.synchronize()
            if i >= 2:
                ts.append(e0.elapsed_time(e1) * 1e3)
        t = float(np.median(ts))
        return {"torch_semi_structured_24_us": t, "tflops_eff": 2.0 * M * K * N / (t * 1e-6) / 1e12,
                "note": "torch's 2:4 semi-structured matmul, same M, K, N; context only"}
    except Exception as ex:  # this torch build has no 2:4 kernel for this GPU
        return {"torch_semi_structured_24": "unavailable",
                "reason": f"{type(ex).__name__}: {str(ex)[:200]}"}


def time_gyro(H, hp, W, X, perm, T, K, G=16, k=2, rounds=4):
    """The library's in-tile gyro rounds (host) on tile 0 of this step: its importance rows,
    its 2:4 band in working order (from the step's regions), `rounds` rounds of G sampled
    groups x k slots (seeded draws); wall-clock time on one host core, and the band's
    pruning cost before and after."""
    import time
    I_tile = H.hinm_importance(W[:T], X).cpu().numpy()
    region0 = hp.region[0].cpu().numpy()
    band = np.array([c for c in perm if region0[c] == 1], dtype=np.int32)
    ng = band.size // 4
    if ng < 2:
        return {"note": "tile 0 has no 2:4 band to refine"}
    G = min(G, ng)
    rng = np.random.default_rng(7)
    c0 = H.hinm_gyro_band_cost_host(I_tile, band)
    t0 = time.perf_counter()
    for _ in range(rounds):
        groups = rng.choice(ng, G, replace=False).astype(np.int32)
        slots = np.stack([rng.choice(4, k, replace=False) for _ in range(G)]).astype(np.int32)
        band, _ = H.hinm_gyro_input_round_host(I_tile, band, groups, slots)
    dt = time.perf_counter() - t0
    c1 = H.hinm_gyro_band_cost_host(I_tile, band)
    return {"ms_per_round": dt / rounds * 1e3, "groups": ng, "sampled_groups": G,
            "slots_per_group": k, "rounds": rounds, "pruning_cost_change": c1 / c0 - 1.0,
            "where": "host (offline, once per layer)", "cores": 1}


def time_hard_concrete(H, n, peaks, stream, reps=10):
    """The Hard-Concrete forward over n = M*K elements (logits N(0, 2), noise U(0, 1), drawn
    on the device from a fixed seed; tau = 2/3): CUDA events over `reps` back-to-back calls
    after 3 untimed ones.  Algorithmic bytes: 4 (log alpha) + 4 (eps) in, 4 (z) + 1 (hard)
    out per element; the arrays (13 B x n) exceed L2 at the benchmark sizes."""
    import torch
    g = torch.Generator(device="cuda").manual_seed(1234)
    la = torch.randn(n, generator=g, device="cuda") * 2.0
    eps = torch.rand(n, generator=g, device="cuda")
    z = torch.empty(n, dtype=torch.float32, device="cuda")
    hard = torch.empty(n, dtype=torch.uint8, device="cuda")
    sums = torch.empty(2, dtype=torch.float64, device="cuda")
    for _ in range(3):
        H.hinm_hard_concrete_forward(la, eps, 2.0 / 3.0, z, hard, sums)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(reps):
        H.hinm_hard_concrete_forward(la, eps, 2.0 / 3.0, z, hard, sums)
    e1.record(stream)
    torch.cuda.synchronize()
    t = e0.elapsed_time(e1) / 1e3 / reps
    gbs = 13.0 * n / t / 1e9
    peak = peaks.get("hbm_gbs") if peaks else None
    return {"us_per_call": t * 1e6, "elements": n, "gbs": gbs, "bound": "hbm",
            "peak_gbs": peak, "frac": (gbs / peak) if peak else None,
            "kernel": "hard_concrete_kernel", "launches": 1,
            "note": "back-to-back calls; 13 B per element, arrays larger than L2"}


# ------------------------------------------------------------------ SpMM operand ingest
# The SpMM kernel's operand traffic from L2 into shared memory, per launch, by the kernel the
# library picks for (N, T, hint): every tile's A blocks (16 KB, plus 2 KB of metadata for a
# 2:4 block) once per column block of BN columns, and every tile's gathered X rows
# (64 per dense block, 128 per 2:4 block) x the block's columns x 2 bytes; with the tile-pair
# hint a pair whose blocks are the same runs reads each X block once for both tiles.
def spmm_plan(N: int, T: int, tile_pairs: bool):
    if N <= 16:
        return "spmm_kernel<16>", 16
    if N <= 32:
        return "spmm_kernel<32>", 32
    if N <= 64:
        return "spmm_kernel<64>", 64
    if N < 256:
        return "spmm_kernel<128>", 128
    if tile_pairs and T == 128 and N >= 1024:
        return "spmm_pair_kernel", 240
    return "spmm_kernel<192>", 192


def l2_to_sm_bytes(M: int, N: int, T: int, counts, tile_pairs: bool) -> float:
    c = np.asarray(counts, dtype=np.int64).reshape(-1, 3)
    nd = -(-c[:, 2] // 64)
    ns = -(-c[:, 1] // 128)
    name, bn = spmm_plan(N, T, tile_pairs)
    ncol = -(-N // bn)
    a_bytes = float(((nd + ns) * 16384 + ns * 2048).sum()) * ncol
    x_rows = (nd * 64 + ns * 128).astype(np.float64)
    x_bytes = float(x_rows.sum()) * N * 2.0
    if name == "spmm_pair_kernel":
        # shared pairs (identical run lists: the hint's case) read each X block once
        x_bytes = float(x_rows[::2].sum()) * N * 2.0
    return a_bytes + x_bytes


def count_graph_kernels(graph):
    """(kernel launches one replay of the captured step issues, their function names),
    counted on the captured cudaGraph_t through the CUDA runtime; (None, []) if the query is
    not available."""
    try:
        import cuda.bindings.runtime as rt
        g = rt.cudaGraph_t(init_value=graph.raw_cuda_graph())
        err, _, n = rt.cudaGraphGetNodes(g, 0)
        err, nodes, n = rt.cudaGraphGetNodes(g, n)
        names, count = set(), 0
        for node in nodes[:n]:
            err, kind = rt.cudaGraphNodeGetType(node)
            if kind != rt.cudaGraphNodeType.cudaGraphNodeTypeKernel:
                continue
            count += 1
            try:
                err, prm = rt.cudaGraphKernelNodeGetParams(node)
                err, nm = rt.cudaFuncGetName(prm.func)
                names.add(nm.decode() if isinstance(nm, bytes) else str(nm))
            except Exception:  # noqa: BLE001 - names are informative only
                pass
        return count, sorted(names)
    except Exception:  # noqa: BLE001
        return None, []


# ------------------------------------------------------------------ one workload on the GPU
def measure(H, w, args, dev, flush, stream, rows=None, dist=None, sampler=None):
    """Time the five-call step of workload w on this rank's rows [r0, r1) of W (all rows on
    one GPU): K CUDA-graph replays (L2 flushed between them) and K eager passes with events
    between the phases.  Returns the measurements and the state the caller reuses."""
    import torch
    M, K, N, T = w.M, w.K, w.N, w.T
    r0, r1 = rows if rows is not None else (0, M)
    Ms = r1 - r0
    have = Ms > 0
    out = dict(rows=(r0, r1))
    if have:
        W = torch.from_numpy(np.ascontiguousarray(w.W_bits[r0:r1]).view(np.int16)).to(dev).view(torch.bfloat16)
        X = torch.from_numpy(w.X_bits.view(np.int16)).to(dev).view(torch.bfloat16)
        perm = torch.from_numpy(w.perm).to(dev)
        # the importance is not materialized: the search and the mask recompute it from W
        hp = H.HotPath(Ms, K, N, T, w.t_s, w.alpha, device=dev, materialize_importance=False)
        # Workloads specified with a fixed boundary v_s use its closed-form counts; the search
        # still runs every step (its ranking feeds the mask).  Otherwise the search's counts.
        fixed = c = None
        if w.v_s is not None:
            c = H.hinm_counts_from_vs(K, w.t_s, w.v_s)
            fixed = torch.tensor([c] * (Ms // T), dtype=torch.int32, device=dev)
        counts_used = fixed if fixed is not None else hp.counts
        # fixed counts known on the host: tell the SpMM when every tile reads the same X rows
        tile_pairs = fixed is not None and H.tile_pairs_hint(c, w.perm, K)
        Yfull = torch.empty((M, N), dtype=torch.float32, device=dev) if args.gather_y else None

        def step(ev=None):
            if ev is not None:
                ev[0].record(stream)
            H.hinm_importance_stats(W, X, T, None, hp.stats, hp.ws, materialize=False)
            if ev is not None:
                ev[1].record(stream)
            H.hinm_boundary_search(None, perm, T, w.t_s, w.alpha, hp.counts, hp.vs, hp.rank,
                                   hp.ws, stats=hp.stats, W=W)
            if ev is not None:
                ev[2].record(stream)
            H.hinm_mask(None, perm, counts_used, T, hp.rank, hp.bitmask, hp.region, hp.ws,
                        W=W, stats=hp.stats)
            if ev is not None:
                ev[3].record(stream)
            H.hinm_compress(W, hp.bitmask, hp.region, perm, counts_used, T, hp.layout, hp.ws)
            if ev is not None:
                ev[4].record(stream)
            H.hinm_spmm(hp.layout, X, hp.Y, None, hp.c_layout, tile_pairs)
            if ev is not None:
                ev[5].record(stream)

        for _ in range(args.warmup):
            step()
        torch.cuda.synchronize()
        st = H.hinm_device_status()
        if st != 0:
            raise RuntimeError(f"device status {st} after warm-up")
        counts = counts_used.cpu().numpy()
        out.update(W=W, X=X, perm=perm, hp=hp, fixed=fixed, tile_pairs=tile_pairs, counts=counts,
                   vs=hp.vs.cpu().numpy())
        try:
            graph = torch.cuda.CUDAGraph(keep_graph=True)
        except TypeError:
            graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            step()
        launches, kernel_names = count_graph_kernels(graph)
        if hasattr(graph, "instantiate"):
            try:
                graph.instantiate()
            except RuntimeError:
                pass
        torch.cuda.synchronize()
    else:
        graph = step = None
        launches, kernel_names = 0, []
    out.update(launches_per_step=launches, kernel_names=kernel_names)
    gev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(args.steps)]
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    if sampler is not None:
        sampler.start()
        time.sleep(0.4)
    for k in range(args.steps):
        flush.zero_()                     # evict L2 (256 MB > 126 MB) between timed steps
        gev[k][0].record(stream)
        if have:
            graph.replay()
        if args.gather_y and dist:
            gathered = gather_rows(hp.Y if have else torch.zeros((0, N), device=dev), M, T,
                                   dist.get_world_size(), dist, H.shard_tiles)
            if have:
                Yfull.copy_(gathered)
        gev[k][1].record(stream)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    step_s = [gev[k][0].elapsed_time(gev[k][1]) * 1e-3 for k in range(args.steps)]
    if have:
        for k in range(args.steps):
            flush.zero_()
            step(evs[k])
        torch.cuda.synchronize()
        if H.hinm_device_status() != 0:
            raise RuntimeError("device status after the timed passes")
    if sampler is not None:
        sampler.stop()
    if dist:
        dist.barrier()
    phases = ["importance", "search", "mask", "compress", "spmm"]
    if have:
        out["per_phase"] = {p: statistics.mean(evs[k][i].elapsed_time(evs[k][i + 1]) * 1e-3
                                               for k in range(args.steps))
                            for i, p in enumerate(phases)}
        out["t_eager"] = statistics.mean(evs[k][0].elapsed_time(evs[k][5]) * 1e-3
                                         for k in range(args.steps))
    out["t_step"] = statistics.mean(step_s)
    if graph is not None:
        del graph
    return out


def spmm_roofline(M, K, N, T, counts, tile_pairs, t_spmm, peaks, peak_kind, traffic):
    model = workload_model(M, K, N, T, counts)
    bound, ach, pk, unit, frac = roofline_for("spmm", t_spmm, model, peaks, peak_kind)
    name, bn = spmm_plan(N, T, tile_pairs)
    ing = l2_to_sm_bytes(M, N, T, counts, tile_pairs)
    return model, {
        "bound": bound, "achieved": ach, "peak": pk, "unit": unit, "frac": frac,
        "traffic": traffic, "kernel": name,
        "peak_source": f"{peak_kind} (MEASURED_PEAKS.json burst; 2:4 = 2x dense bf16)",
        "l2_to_sm": {"bytes_per_launch": ing, "achieved_tbs": ing / t_spmm / 1e12,
                     "ceiling_tbs": L2_TO_SM_CEILING_TBS,
                     "frac": ing / t_spmm / 1e12 / L2_TO_SM_CEILING_TBS,
                     "ceiling_source": L2_TO_SM_CEILING_SOURCE,
                     "basis": "A blocks (+metadata) once per BN-column block, gathered X rows "
                              "x columns x 2 B per tile"}}


# The L2 -> shared-memory ceiling the SpMM's operand stream is compared with: ncu's
# peak-sustained rate of the L2 slices' output to the crossbar on this B200, derived from
# the up-proj capture of spmm_kernel<256> (lts__lts2xbar_cycles_active 28.27 % of peak at
# 6.48 TB/s of lts2xbar bytes).
L2_TO_SM_CEILING_TBS = 22.9
L2_TO_SM_CEILING_SOURCE = ("ncu peak-sustained lts2xbar rate on this B200 (28.27 % = 6.48 TB/s, "
                           "up-proj spmm_kernel<256> capture)")


def traffic_for(name, kernel):
    tr_path = os.path.join(ROOT, "profiles", "traffic.json")
    if os.path.exists(tr_path):
        return json.load(open(tr_path)).get(name, {}).get(kernel)
    return None


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="hinm", choices=["hinm", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-next-rows", action="store_true",
                    help="skip the extra timings of the index translation, the fused epilogue, "
                         "the Hard-Concrete forward and the gyro refinement")
    ap.add_argument("--no-other-configs", action="store_true",
                    help="skip the pure 2:4 and decode workloads measured beside the headline")
    ap.add_argument("--gather-y", action="store_true",
                    help="multi-GPU: all-gather Y (NCCL) at the end of every timed step")
    ap.add_argument("--workload", default="up", choices=sorted(WORKLOADS) + ["sweep"],
                    help="synthetic workload (default: the HiNM up-proj 11008x4096x4096); "
                         "'sweep' times the LLaMA-2-7B-shaped layer sweep")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.workload == "sweep":
        if world > 1 or args.impl == "reference":
            raise SystemExit("--workload sweep runs on one GPU with the CUDA arm only")
        return run_sweep(args)
    w = WORKLOADS[args.workload]()
    if args.impl == "reference":
        return run_reference(args, w)

    import torch
    import pruning_hinm_spmm_b200 as H

    torch.cuda.set_device(local_rank)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))

    M, K, N, T = w.M, w.K, w.N, w.T
    dev = torch.device("cuda", local_rank)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    rows = H.shard_tiles(M, T, world, rank)
    sampler = ClockSampler(local_rank)
    m = measure(H, w, args, dev, flush, stream, rows=rows, dist=dist, sampler=sampler)
    have = rows[1] > rows[0]
    t_step = max_over_ranks(m["t_step"], dist, dev)
    value = job_value(2.0 * M * K * N, t_step)

    # ---------------- end to end through the public API with host buffers
    # Every step copies this rank's inputs in from pinned host memory (its rows of W, all of
    # X, the permutation) and its rows of Y out.  Two device buffer sets (each with its own
    # HotPath) let step k+1's upload and step k-1's download run on their own streams while
    # step k computes: the figure is the pipelined steady-state throughput, not the latency
    # of one call.
    r0, r1 = rows
    Ms = r1 - r0
    e2e_steps = max(4, min(args.steps, 10))
    h2d = d2h = 0
    t_e2e = 0.0
    if have:
        W_h = torch.from_numpy(np.ascontiguousarray(w.W_bits[r0:r1]).view(np.int16)).pin_memory()
        X_h = torch.from_numpy(w.X_bits.view(np.int16)).pin_memory()
        P_h = torch.from_numpy(w.perm).pin_memory()
        hp0 = m["hp"]
        sets = []
        for b in range(2):
            hp_b = hp0 if b == 0 else H.HotPath(Ms, K, N, T, w.t_s, w.alpha, device=dev,
                                                materialize_importance=False)
            sets.append(dict(hp=hp_b, W=torch.empty_like(m["W"]), X=torch.empty_like(m["X"]),
                             P=torch.empty_like(m["perm"]),
                             Y=torch.empty((Ms, N), dtype=torch.float32).pin_memory(),
                             consumed=torch.cuda.Event(), read=torch.cuda.Event(),
                             loaded=torch.cuda.Event()))
        s_up, s_comp, s_down = (torch.cuda.Stream(dev), torch.cuda.Stream(dev),
                                torch.cuda.Stream(dev))
        for st in sets:  # both sets start free
            st["consumed"].record(s_comp)
            st["read"].record(s_down)

        def e2e_step(k):
            st = sets[k % 2]
            s_up.wait_event(st["consumed"])
            with torch.cuda.stream(s_up):
                st["W"].view(torch.int16).copy_(W_h, non_blocking=True)
                st["X"].view(torch.int16).copy_(X_h, non_blocking=True)
                st["P"].copy_(P_h, non_blocking=True)
            st["loaded"].record(s_up)
            s_comp.wait_event(st["loaded"])
            s_comp.wait_event(st["read"])
            with torch.cuda.stream(s_comp):
                st["hp"].run(st["W"], st["X"], st["P"], fixed_counts=m["fixed"], stream=s_comp,
                             tile_pairs=m["tile_pairs"])
            st["consumed"].record(s_comp)
            s_down.wait_event(st["consumed"])
            with torch.cuda.stream(s_down):
                st["Y"].copy_(st["hp"].Y, non_blocking=True)
            st["read"].record(s_down)

        for k in range(2):
            e2e_step(k)
        torch.cuda.synchronize()
        e_start = torch.cuda.Event(enable_timing=True)
        e_end = torch.cuda.Event(enable_timing=True)
        if dist:
            dist.barrier()
        e_start.record(s_up)
        for k in range(e2e_steps):
            e2e_step(k)
        e_end.record(s_down)
        torch.cuda.synchronize()
        t_e2e = e_start.elapsed_time(e_end) * 1e-3 / e2e_steps
        h2d = W_h.numel() * 2 + X_h.numel() * 2 + P_h.numel() * 4
        d2h = sets[0]["Y"].numel() * 4
        # the e2e outputs must match the device-resident path
        for st in sets:
            assert torch.equal(st["Y"], hp0.Y.cpu())
    elif dist:
        dist.barrier()
    t_e2e = max_over_ranks(t_e2e, dist, dev)
    launches = m["launches_per_step"]

    if dist:
        dist.destroy_process_group()
    if rank != 0:
        return 0

    peaks, peak_kind = load_peaks()
    counts = m["counts"]
    Ms0 = rows[1] - rows[0]
    model = workload_model(Ms0, K, N, T, counts)
    kernels = {}
    for p, t in m["per_phase"].items():
        bound, ach, pk, unit, frac = roofline_for(p, t, model, peaks, peak_kind)
        kernels[p] = {"ms": t * 1e3, "bound": bound, "achieved": ach, "peak": pk,
                      "unit": unit, "frac": frac}
    spmm_t = m["per_phase"]["spmm"]
    name0, _ = spmm_plan(N, T, m["tile_pairs"])
    _, roof = spmm_roofline(Ms0, K, N, T, counts, m["tile_pairs"], spmm_t, peaks, peak_kind,
                            traffic_for(w.name, name0.split("<")[0]))
    roof["longest_phase"] = max(m["per_phase"], key=lambda p: m["per_phase"][p])
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        from threadpoolctl import threadpool_limits
        cores = cpu_cores()
        with threadpool_limits(limits=cores):
            dt, fl = cpu_oracle_sample(w, 4)
        cpu = {"value": fl / dt / 1e12, "unit": UNIT, "cores": cores, "kind": "oracle",
               "sample": f"4 of {M // T} tiles ({4 * T} output rows) of {w.name}: channel "
                         "energies, importance, search, mask, compress and fp64 masked product",
               "seconds": dt}
    clocks = sampler.summary()
    next_rows = context = others = None
    if world == 1 and not args.no_next_rows:
        hp = m["hp"]
        context = time_dense_context(M, K, N, flush, stream)
        next_rows = {"index_translate": time_index_translate(H, hp, K, stream),
                     "hard_concrete": time_hard_concrete(H, M * K, peaks, stream),
                     "epilogue_bf16": time_epilogue(H, hp, m["X"], M, N, m["tile_pairs"], flush,
                                                    stream),
                     "gyro_refine_host": time_gyro(H, hp, m["W"], m["X"], w.perm, T, K)}
    if world == 1 and not args.no_other_configs:
        others = {}
        for oname in ("pure24", "decode"):
            if oname == args.workload:
                continue
            wo = WORKLOADS[oname]()
            mo = measure(H, wo, args, dev, flush, stream)
            so = mo["per_phase"]["spmm"]
            cn, _ = spmm_plan(wo.N, wo.T, mo["tile_pairs"])
            _, ro = spmm_roofline(wo.M, wo.K, wo.N, wo.T, mo["counts"], mo["tile_pairs"], so,
                                  peaks, peak_kind, traffic_for(wo.name, cn.split("<")[0]))
            others[wo.name] = {
                "ms_per_step": mo["t_step"] * 1e3,
                "value": job_value(2.0 * wo.M * wo.K * wo.N, mo["t_step"]), "unit": UNIT,
                "phases_ms": {p: t * 1e3 for p, t in mo["per_phase"].items()},
                "spmm_ms": so * 1e3, "roofline": ro,
                "launches_per_step": mo["launches_per_step"],
                "config": {"M": wo.M, "K": wo.K, "N": wo.N, "T": wo.T, "t_s": wo.t_s,
                           "v_s_used": wo.v_s, "counts_tile0": mo["counts"][0].tolist()}}
            if oname == "pure24" and not args.no_next_rows:
                others[wo.name]["context"] = {
                    "dense": time_dense_context(wo.M, wo.K, wo.N, flush, stream),
                    "semi_structured_24": time_sparse24_context(wo.M, wo.K, wo.N, flush, stream)}
            del mo
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": t_step * 1e3, "higher_is_better": True,
        "ms_per_step_eager": m["t_eager"] * 1e3,
        "scaling": "strong", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": w.name, "M": M, "K": K, "N": N, "T": T, "t_s": w.t_s,
                   "alpha": w.alpha, "v_s_searched": sorted(set(np.round(m["vs"], 6).tolist())),
                   "v_s_used": w.v_s if w.v_s is not None else "searched",
                   "counts_tile0": counts[0].tolist(),
                   "l2": "flushed between timed steps (256 MB write)",
                   "step": "importance+search+mask+compress+spmm",
                   "importance": "not materialized: the search and the mask recompute it from "
                                 "W and the channel energies (the same bits)",
                   "step_exec": "CUDA graph replay of the five calls (phase times: eager pass)",
                   "parallelism": (f"tiles sharded over {world} GPUs, X replicated"
                                   + (", Y all-gathered (NCCL) every step" if args.gather_y
                                      else ", each rank keeps its rows of Y"))
                   if world > 1 else "1 GPU",
                   "rank0_rows": list(rows)},
        "spmm_only": {"ms": spmm_t * 1e3, "tflops_eff": model["flops_eff"] / spmm_t / 1e12,
                      "tflops_actual": model["flops_actual"] / spmm_t / 1e12,
                      "gbs": model["bytes"]["spmm"] / spmm_t / 1e9},
        "kernels": kernels,
        "roofline": roof,
        "cpu_baseline": cpu,
        "e2e": {"value": job_value(2.0 * M * K * N, t_e2e), "unit": UNIT,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": t_e2e * 1e3,
                "kind": "pipelined steady-state throughput through the public API (two buffer "
                        "sets; upload, compute and download on their own streams)"},
        "gpu_launches": (launches * args.steps) if launches is not None else None,
        "gpu_launches_counted": "kernel nodes of the captured step graph (CUDA runtime) x "
                                "timed replays, rank 0",
        "kernels_in_step": m["kernel_names"],
        "other_configs": others,
        "next_rows": next_rows,
        "context": context,
        "clocks": {"sm_mhz": clocks["sm_mhz"], "sm_max_mhz": clocks["sm_max_mhz"],
                   "reasons": clocks["reasons"], "samples": clocks["samples"]},
    }
    print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
