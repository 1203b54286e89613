#!/usr/bin/env python
"""Benchmark of the DualQuant dual-scale W4A4 hot path on B200.

Headline workload (qwen32b_mlp_nvfp4): the Qwen-32B-shaped MLP weights
27648x5120 and 5120x27648 bf16 (Student-t), NVFP4, 50 BCD rounds;
activations M x K bf16 with 1 % outlier channels x100, M = 8192 (prefill)
and M in {1, 8, 64} (decode).  One step is the whole path:
    for each M, each weight : dq_quantize_act -> dq_w4a4_linear
    for each weight         : dq_solve_scales (T = 50) -> dq_quantize_weight
The linears run first in the step, on the weights packed by the previous
step, right after an L2 flush (a 256 MiB write outside the timed events), so
they read their weights cold.  Inputs are resident in HBM before timing.

`value` = W4A4 linear TFLOP/s of the prefill linears (M = 8192, both
weights, activation quantiser + GEMM: 2 M N K over their device time).  The
solver, the decode linears and the packer are reported beside it, each with
its own roofline fraction; ms_per_step covers the whole step.  Events sit
only around the prefill linears, the decode linears and each solver call (an
event record costs the GPU microseconds).  Per-kernel figures are taken
after the timed steps from launches back to back on copies of their inputs
that together exceed L2.  The other workloads (the Llama-3.1-8B-shaped
attention and MX MLP layers, the tiny layer, the 224-weight sweep in four
formats) and the MXFP8 linear are measured after that and reported under
`configs` / `mxfp8`.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
"""
import argparse
import json
import os
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from w4a4_post_quantization_dual_b200 import dist, synth  # noqa: E402

WORKLOAD = "qwen32b_mlp_nvfp4"
METRIC = "W4A4 linear TFLOP/s & % of FP4 peak; BCD solver GB/s & % HBM peak"
FMT_NAME = "nvfp4"


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d["hbm_gbs"], d["bf16_tflops"], d.get("bf16_tflops_sustained"), d.get(
            "sm_max_mhz", 1965.0), "measured"
    return 6650.0, 1590.0, 1400.0, 1965.0, "fallback"


def measured_traffic(key, files):
    """DRAM bytes per launch from the committed ncu capture of this kernel,
    or None when the kernel's source changed since the capture."""
    import hashlib
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    rec = json.load(open(p)).get(key)
    if not rec:
        return None
    h = hashlib.sha256()
    for f in files:
        h.update(open(os.path.join(ROOT, "w4a4_post_quantization_dual_b200", "csrc", f), "rb").read())
    return rec["dram_bytes"] if h.hexdigest()[:16] == rec["source_hash"] else None


class ClockSampler:
    """SM clock and clock-event reasons sampled through NVML (read-only)
    every 5 ms while the timed region runs."""

    REASONS = {"hw_slowdown": 0x8, "hw_thermal_slowdown": 0x40, "sw_thermal_slowdown": 0x20,
               "sw_power_cap": 0x4, "hw_power_brake_slowdown": 0x80}

    def __init__(self, cuda_index):
        self.samples, self.reasons, self.err = [], set(), None
        self.stop_ev = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            uuid = str(torch.cuda.get_device_properties(cuda_index).uuid).lower().replace("gpu-", "")
            self.h = None
            for i in range(pynvml.nvmlDeviceGetCount()):
                h = pynvml.nvmlDeviceGetHandleByIndex(i)
                u = pynvml.nvmlDeviceGetUUID(h)
                u = (u.decode() if isinstance(u, bytes) else u).lower().replace("gpu-", "")
                if u == uuid:
                    self.h = h
            if self.h is None:
                self.h = pynvml.nvmlDeviceGetHandleByIndex(0)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # noqa: BLE001 -- no NVML: report it, never fail the bench
            self.err = repr(e)

    def _run(self):
        nv = self.nv
        while not self.stop_ev.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for name, bit in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception as e:  # noqa: BLE001
                self.err = repr(e)
                return
            time.sleep(0.005)

    def start(self):
        if self.err is None:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()

    def stop(self):
        if self.err is not None and not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "error": self.err}
        self.stop_ev.set()
        self.t.join(timeout=2)
        return {"sm_mhz": float(np.median(self.samples)) if self.samples else None,
                "sm_max_mhz": float(self.max_mhz), "reasons": sorted(self.reasons),
                "samples": len(self.samples), "source": "NVML"}


# ---------------------------------------------------------------------------
# Inputs
# ---------------------------------------------------------------------------
def workload_inputs(name, fmt_name=None):
    """Host inputs of a workload: weights and, per weight, its activations
    for every M of the workload (K = the weight's input width)."""
    wl = synth.WORKLOADS[name]
    Ws = [synth.weight(name, i)[0] for i in range(len(wl["weights"]))]
    Xs = {}
    for j, W in enumerate(Ws):
        K = W.shape[1]
        for M in wl["M"]:
            Xs[(M, j)] = synth.acts(name, M, K, index=j)[0]
    return wl, Ws, Xs


def ev():
    return torch.cuda.Event(enable_timing=True)


L2_BYTES = 126 * 1024 * 1024


def per_launch_us(fn_of_copy, n_copies, reps=2):
    """Average duration of fn_of_copy(i) launched back to back between two
    events (i cycling over n_copies input copies, so that the launches read
    cold data when the copies together exceed L2)."""
    st = torch.cuda.current_stream()
    for i in range(n_copies):
        fn_of_copy(i)
    torch.cuda.synchronize()
    torch.cuda._sleep(60_000 * reps * n_copies)  # the launches queue up behind it
    k0, k1 = ev(), ev()
    k0.record(st)
    for _ in range(reps):
        for i in range(n_copies):
            fn_of_copy(i)
    k1.record(st)
    torch.cuda.synchronize()
    return 1e3 * k0.elapsed_time(k1) / (reps * n_copies)


def n_copies(nbytes, lo=2, hi=64):
    """Copies of an input whose total exceeds twice L2."""
    return int(max(lo, min(hi, -(-2 * L2_BYTES // max(nbytes, 1)))))


def act_bytes(M, K, fmt, G):
    """Algorithmic bytes of one activation rescale+quantise: bf16 in, codes,
    block scales (and the fp32 per-token scale for NVFP4) out."""
    from w4a4_post_quantization_dual_b200 import dq
    code = 1.0 if dq._fmt(fmt) in dq.EIGHT_BIT else 0.5
    return M * K * (2 + code + 1.0 / G) + (4 * M if dq._fmt(fmt) == dq.DQ_NVFP4 else 0)


def decode_bytes(M, N, K, G):
    """Algorithmic bytes of a 4-bit linear at small M (weight-bandwidth bound):
    weight codes + block scales, activation codes + scales + per-token
    scales, bf16 output."""
    return N * K / 2 + N * K / G + M * K / 2 + M * K / G + 4 * M + 2 * M * N


class Layer:
    """Device buffers of one weight: the weight, its scales, its packed form."""

    def __init__(self, W, fmt, G, dev):
        from w4a4_post_quantization_dual_b200 import dq
        self.W = W
        m, n = W.shape
        eight = dq._fmt(fmt) in dq.EIGHT_BIT
        self.r = torch.empty((m, n // G), dtype=torch.float32, device=dev)
        self.c = torch.empty(n, dtype=torch.float32, device=dev)
        self.sT = torch.empty(1, dtype=torch.float32, device=dev)
        self.codes = torch.empty((m, n if eight else n // 2), dtype=torch.uint8, device=dev)
        self.scales = torch.empty(dq.scales_bytes(m, n, fmt, G), dtype=torch.uint8, device=dev)

    def solve(self, fmt, T, ws, G):
        from w4a4_post_quantization_dual_b200 import dq
        dq.dq_solve_scales(self.W, fmt, T, self.r, self.c, self.sT, None, ws, group=G)

    def pack(self, fmt, G):
        from w4a4_post_quantization_dual_b200 import dq
        dq.dq_quantize_weight(self.W, fmt, self.r, self.c, self.sT, self.codes, self.scales,
                              group=G)


class Act:
    """Device buffers of one activation and its quantised form."""

    def __init__(self, X, fmt, G, N, dev):
        from w4a4_post_quantization_dual_b200 import dq
        M, K = X.shape
        eight = dq._fmt(fmt) in dq.EIGHT_BIT
        self.X = X
        self.A = torch.empty((M, K if eight else K // 2), dtype=torch.uint8, device=dev)
        self.sA = torch.empty(dq.scales_bytes(M, K, fmt, G), dtype=torch.uint8, device=dev)
        self.st = (torch.empty(M, dtype=torch.float32, device=dev)
                   if dq._fmt(fmt) == dq.DQ_NVFP4 else None)
        self.Y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)

    def linear(self, L, fmt, G, X=None):
        from w4a4_post_quantization_dual_b200 import dq
        dq.dq_quantize_act(self.X if X is None else X, fmt, L.c, self.A, self.sA, self.st, group=G)
        dq.dq_w4a4_linear(self.A, self.sA, self.st, L.codes, L.scales, L.sT, self.Y, fmt)

    def gemm(self, fmt, codes, scales, sT):
        from w4a4_post_quantization_dual_b200 import dq
        dq.dq_w4a4_linear(self.A, self.sA, self.st, codes, scales, sT, self.Y, fmt)


def time_linear(L, a, fmt, G, peak_tf):
    """Activation quantiser and GEMM of one (activation, weight) pair, each
    launched back to back on cold copies of its input (activations for the
    quantiser, packed weights for the GEMM)."""
    M, K = a.X.shape
    N = L.W.shape[0]
    from w4a4_post_quantization_dual_b200 import dq
    nx = n_copies(a.X.numel() * 2, hi=16)
    Xc = [a.X.clone() for _ in range(nx)]
    t_act = per_launch_us(lambda i: dq.dq_quantize_act(Xc[i], fmt, L.c, a.A, a.sA, a.st,
                                                       group=G), nx)
    del Xc
    a.linear(L, fmt, G)
    nw = n_copies(L.codes.numel() + L.scales.numel())
    Bc = [(L.codes.clone(), L.scales.clone()) for _ in range(nw)]
    t_gemm = per_launch_us(lambda i: a.gemm(fmt, Bc[i][0], Bc[i][1], L.sT), nw)
    del Bc
    fl = 2.0 * M * N * K
    ab = act_bytes(M, K, fmt, G)
    return {"M": M, "N": N, "K": K, "act_us": t_act, "gemm_us": t_gemm,
            # the captures are of the NVFP4 kernels
            "gemm_traffic": (measured_traffic(f"gemm_nvfp4_{M}x{N}x{K}", ["dq_gemm.cu", "dq_device.cuh"])
                             if dq._fmt(fmt) == dq.DQ_NVFP4 else None),
            "act_traffic": (measured_traffic(f"act_nvfp4_{M}x{K}", ["dq_quant.cu", "dq_device.cuh"])
                            if dq._fmt(fmt) == dq.DQ_NVFP4 else None),
            "gemm_tflops": fl / (t_gemm * 1e-6) / 1e12, "gemm_frac": fl / (t_gemm * 1e-6) / 1e12 / peak_tf,
            "act_gbs": ab / (t_act * 1e-6) / 1e9, "linear_tflops": fl / ((t_act + t_gemm) * 1e-6) / 1e12}


# ---------------------------------------------------------------------------
# Reference arm / CPU baseline: the oracle as it stands, on host cores.
# ---------------------------------------------------------------------------
_ORACLE_PACKED = {}


def oracle_prepare(Ws):
    """Offline part for the oracle legs: Algorithm 1's initial scales of every
    tile (T = 0) and the packed weights, computed once and cached."""
    import oracle as O
    if not _ORACLE_PACKED:
        for i, W in enumerate(Ws):
            res = O.solve(W, O.NVFP4, 16, 0)
            B, sB = O.pack_weight(W, O.NVFP4, 16, res["r"], res["c"], res["s_T"])
            _ORACLE_PACKED[i] = (res, B, sB)
    return _ORACLE_PACKED


SAMPLE_COLS = 2048


def oracle_linear_sample(Ws, Xs, M, rows):
    """The oracle's inference path on a bounded sample of the prefill
    linears: activation rescale+quantise of `rows` token rows, then the
    dequantised fp64 matmul for SAMPLE_COLS seeded output columns, for both
    weights.  Returns (TFLOP/s of the sampled outputs, seconds)."""
    import oracle as O
    packed = oracle_prepare(Ws)
    flops, t0 = 0.0, time.perf_counter()
    for j, W in enumerate(Ws):
        N, K = W.shape
        res, B, sB = packed[j]
        X = Xs[(M, j)][:rows]
        A, sA, st = O.quantize_act(X, res["c"], O.NVFP4, 16)
        cols = np.random.default_rng(j).choice(N, size=min(SAMPLE_COLS, N), replace=False)
        O.linear_rows(A, sA, st, B, sB, res["s_T"], np.arange(rows), rows, N, K, O.NVFP4,
                      cols=cols)
        flops += 2.0 * rows * len(cols) * K
    dt = time.perf_counter() - t0
    return flops / dt / 1e12, dt


LINEAR_SAMPLE_DESC = ("oracle (C + numpy fp64): activation rescale+quantise of {rows} of the "
                      "{M} prefill token rows and the dequantised fp64 matmul for " +
                      str(SAMPLE_COLS) + " sampled output columns, both weights (weights "
                      "packed once beforehand, outside the timing)")


def _oracle_tile(args):
    import oracle as O
    Wt, T = args
    t0 = time.perf_counter()
    O.solve(Wt, O.NVFP4, 16, T)
    return time.perf_counter() - t0


def oracle_solver_sample(W, T, procs):
    """Algorithm 1 (T rounds) on whole m x 16 column tiles of the weight:
    one tile on one core, then one tile per process on `procs` host cores
    (spawned processes).  Each tile is solved on its own columns (its
    initial scales and tensor scale from those columns).  Returns effective
    GB/s (T * tile bytes / time) for both and the seconds."""
    import multiprocessing as mp
    m = W.shape[0]
    tile = lambda b: np.ascontiguousarray(W[:, 16 * b:16 * b + 16])
    one = _oracle_tile((tile(0), T))
    ctx = mp.get_context("spawn")
    t0 = time.perf_counter()
    with ctx.Pool(procs) as pool:
        pool.map(_oracle_tile, [(tile(b), T) for b in range(procs)])
    wall = time.perf_counter() - t0
    tb = T * m * 16 * 2.0
    return {"one_core_gbs": tb / one / 1e9, "one_core_s": one,
            "all_cores_gbs": procs * tb / wall / 1e9, "all_cores_s": wall, "cores": procs}


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        return max([d.get("num_threads", 1) for d in threadpool_info()] + [1])
    except Exception:
        return os.cpu_count() or 1


def run_reference(args, rank, world):
    if rank != 0:
        return
    wl, Ws, Xs = workload_inputs(args.workload)
    M = max(wl["M"])
    oracle_prepare(Ws)
    for _ in range(args.warmup):
        oracle_linear_sample(Ws, Xs, M, rows=16)
    flops_t, dt = 0.0, 0.0
    for _ in range(args.steps):
        v, d = oracle_linear_sample(Ws, Xs, M, rows=16)
        flops_t += v * d
        dt += d
    value = flops_t / dt
    desc = LINEAR_SAMPLE_DESC.format(rows=16, M=M)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": dt / max(args.steps, 1) * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": args.workload, "format": FMT_NAME, "M": M, "sample_rows": 16,
                   "sample_cols": SAMPLE_COLS},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": blas_threads(),
                         "kind": "oracle", "sample": desc},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# Our arm
# ---------------------------------------------------------------------------
def side_config(name, fmts, dev, ws_T, ws, peaks_):
    """Solver time and linear throughput of another workload (not timed in the
    step): per format, each weight solved (T rounds) and packed, then the
    activation quantiser and GEMM of every M of the workload."""
    from w4a4_post_quantization_dual_b200 import dq
    hbm, fp4_peak, fp8_peak, alu_peak = peaks_
    wl, Ws, Xs = workload_inputs(name)
    T = wl["T"]
    Wd = [torch.from_numpy(W).to(torch.bfloat16).to(dev) for W in Ws]
    out = {"weights": [list(W.shape) for W in Ws], "M": wl["M"], "T": T}
    for f in fmts:
        fmt = dq.FORMATS[f]
        G = dq.native_group(fmt)
        peak = fp8_peak if f in ("mxint4", "mxfp8") else fp4_peak
        res = {"solver": {}, "linear": {}}
        Ls = [Layer(W, fmt, G, dev) for W in Wd]
        for L in Ls:
            ms = 1e-3 * per_launch_us(lambda i: L.solve(fmt, T, ws, G), 2)
            m_, n_ = L.W.shape
            tops = 12.0 * m_ * n_ * T / (ms * 1e-3) / 1e12
            res["solver"][f"{m_}x{n_}"] = {"ms": ms, "tops": tops, "frac_alu": tops / alu_peak}
            L.pack(fmt, G)
        for (M, j), X in Xs.items():
            a = Act(torch.from_numpy(X).to(torch.bfloat16).to(dev), fmt, G, Ls[j].W.shape[0], dev)
            res["linear"][f"M{M}_N{Ls[j].W.shape[0]}_K{Ls[j].W.shape[1]}"] = time_linear(
                Ls[j], a, fmt, G, peak)
            del a
        res["peak_tflops"] = peak
        out[f] = res
        del Ls
    return out


def run_ours(args, rank, world, local_rank):
    from w4a4_post_quantization_dual_b200 import dq, sweep
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    dq.lib()
    wl, Ws, Xs = workload_inputs(args.workload)
    fmt, T = dq.DQ_NVFP4, wl["T"]
    G = dq.native_group(fmt)
    st = torch.cuda.current_stream()
    Mp = max(wl["M"])                     # prefill
    Mds = sorted(M for M in wl["M"] if M != Mp)  # decode

    Ls = [Layer(torch.from_numpy(W).to(torch.bfloat16).to(dev), fmt, G, dev) for W in Ws]
    acts = {(M, j): Act(torch.from_numpy(X).to(torch.bfloat16).to(dev), fmt, G,
                        Ls[j].W.shape[0], dev) for (M, j), X in Xs.items()}
    ws = torch.empty(dq.solve_workspace_size(max(T, 64)), dtype=torch.uint8, device=dev)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    flops_p = sum(2.0 * Mp * L.W.shape[0] * L.W.shape[1] for L in Ls)
    launches_per_step = 2 * len(Ls) * len(wl["M"]) + 3 * len(Ls)

    def step(rec):
        # linears first, on the weights the previous step packed, right after
        # the L2 flush (cold weights); events only around the prefill
        # linears, the decode linears and each solver call
        e0, e1, e2, e3 = ev(), ev(), ev(), ev()
        e0.record(st)
        for j, L in enumerate(Ls):
            acts[(Mp, j)].linear(L, fmt, G)
        e1.record(st)
        for M in Mds:
            for j, L in enumerate(Ls):
                acts[(M, j)].linear(L, fmt, G)
        e2.record(st)
        for L in Ls:
            s0, s1 = ev(), ev()
            s0.record(st)
            L.solve(fmt, T, ws, G)
            s1.record(st)
            L.pack(fmt, G)
            rec["solve"].append((s0, s1))
        e3.record(st)
        rec["step"].append((e0, e3))
        rec["prefill"].append((e0, e1))
        rec["decode"].append((e1, e2))

    dist.barrier()
    for _ in range(args.warmup):
        flush.fill_(1)
        step({"solve": [], "step": [], "prefill": [], "decode": []})
    torch.cuda.synchronize()
    dist.barrier()
    torch.cuda.synchronize()

    sampler = ClockSampler(local_rank)
    sampler.start()
    rec = {"solve": [], "step": [], "prefill": [], "decode": []}
    for _ in range(args.steps):
        flush.fill_(rank + 1)      # L2 flush, outside the timed events
        step(rec)
    torch.cuda.synchronize()
    dist.barrier()
    torch.cuda.synchronize()
    clocks = sampler.stop()
    if dq.dq_device_error(clear=True) != 0:
        raise RuntimeError("device error word set during the bench")

    el = lambda p: p[0].elapsed_time(p[1])  # ms
    step_ms = sum(el(p) for p in rec["step"])
    pre_ms = sum(el(p) for p in rec["prefill"])
    dec_ms = sum(el(p) for p in rec["decode"])
    solve_each = [el(p) for p in rec["solve"]]
    solve_ms = sum(solve_each)
    step_ms, pre_ms, dec_ms, solve_ms = dist.max_over_ranks([step_ms, pre_ms, dec_ms, solve_ms],
                                                            device=dev)
    # whole-job throughput: every rank runs the same per-GPU workload (weak
    # scaling); the time is the slowest rank's
    value = world * flops_p * args.steps / (pre_ms * 1e-3) / 1e12

    hbm, bf16_tf, bf16_sus, sm_max, peak_kind = peaks()
    fp4_peak = 4.0 * bf16_tf            # nominal fp4 : bf16 dense ratio 9 : 2.25
    fp8_peak = 2.0 * bf16_tf            # nominal fp8 : bf16 dense ratio 4.5 : 2.25
    # solver: 12 algorithmic fp32 ops per element per round (two
    # quantisations, two scale products, four reduction FMAs); ALU peak =
    # 148 SMs x 128 fp32 lanes x max SM clock (derived, not measured)
    alu_peak = 148 * 128 * sm_max * 1e6 / 1e12  # T lane-ops/s

    # ---- per-kernel durations (after the timed steps)
    solver = {}
    for j, L in enumerate(Ls):
        m_, n_ = L.W.shape
        ms = float(np.mean(solve_each[j::len(Ls)]))
        tops = 12.0 * m_ * n_ * T / (ms * 1e-3) / 1e12
        gbs = T * m_ * n_ * 2.0 / (ms * 1e-3) / 1e9
        solver[f"{m_}x{n_}"] = {"ms": ms, "tops": tops, "frac_alu": tops / alu_peak,
                                "gbs_effective": gbs, "frac_hbm_effective": gbs / hbm}
    prefill = {f"N{L.W.shape[0]}_K{L.W.shape[1]}": time_linear(L, acts[(Mp, j)], fmt, G, fp4_peak)
               for j, L in enumerate(Ls)}
    decode = {}
    for M in Mds:
        for j, L in enumerate(Ls):
            a = acts[(M, j)]
            N, K = L.W.shape
            nw = n_copies(L.codes.numel() + L.scales.numel())
            Bc = [(L.codes.clone(), L.scales.clone()) for _ in range(nw)]
            a.linear(L, fmt, G)
            t_gemm = per_launch_us(lambda i: a.gemm(fmt, Bc[i][0], Bc[i][1], L.sT), nw)

            def pair(i):
                dq.dq_quantize_act(a.X, fmt, L.c, a.A, a.sA, a.st, group=G)
                a.gemm(fmt, Bc[i][0], Bc[i][1], L.sT)

            def fused(i):
                dq.dq_w4a4_linear_fused(a.X, L.c, Bc[i][0], Bc[i][1], L.sT, a.Y, fmt)

            t_pair = per_launch_us(pair, nw)
            try:    # the fused kernel takes the shapes whose K split fits its stages
                t_fused = per_launch_us(fused, nw)
            except dq.DQError:
                t_fused = None
            del Bc
            b_ = decode_bytes(M, N, K, G)
            decode[f"M{M}_N{N}_K{K}"] = {
                "kernel": ("w4a4_gemv_kernel (CUDA cores)" if M == 1 and K % 1024 == 0 and
                           fmt in (dq.DQ_NVFP4, dq.DQ_MXFP4) else "tcgen05 GEMM"),
                "gemm_us": t_gemm, "act_plus_gemm_us": t_pair, "fused_us": t_fused,
                "gemm_traffic": (measured_traffic(f"gemv_nvfp4_{M}x{N}x{K}", ["dq_gemv.cu", "dq_device.cuh"])
                                 if M == 1 and dq._fmt(fmt) == dq.DQ_NVFP4 else None),
                "algorithmic_bytes": b_, "gemm_gbs": b_ / (t_gemm * 1e-6) / 1e9,
                "gemm_frac_hbm": b_ / (t_gemm * 1e-6) / 1e9 / hbm,
                "pair_gbs": b_ / (t_pair * 1e-6) / 1e9,
                "fused_gbs": b_ / (t_fused * 1e-6) / 1e9 if t_fused else None,
                "fused_frac_hbm": b_ / (t_fused * 1e-6) / 1e9 / hbm if t_fused else None}
    pack = {}
    for L in Ls:
        m_, n_ = L.W.shape
        t = per_launch_us(lambda i: L.pack(fmt, G), 2)
        b_ = m_ * n_ * (2 + 0.5 + 1.0 / G)
        pack[f"{m_}x{n_}"] = {"us": t, "gbs": b_ / (t * 1e-6) / 1e9,
                              "frac_hbm": b_ / (t * 1e-6) / 1e9 / hbm}

    # ---- solver ablation modes (Table 4 arms) on the first weight
    L0 = Ls[0]
    modes = {"both": 0, "alpha_only": dq.DQ_SOLVE_ALPHA_ONLY, "beta_only": dq.DQ_SOLVE_BETA_ONLY}
    mode_ms = {name: 1e-3 * per_launch_us(lambda i: dq.dq_solve_scales_ex(
        L0.W, fmt, T, L0.r, L0.c, L0.sT, flags=flags, workspace=ws, group=G), 2)
        for name, flags in modes.items()}
    L0.solve(fmt, T, ws, G)   # restore the step's scales of that weight
    L0.pack(fmt, G)

    # ---- activation SQNR of the prefill activations with each weight's
    # column scales (beta) and without them (Appendix E, Table 6)
    act_sqnr = {}
    for j, L in enumerate(Ls):
        X = acts[(Mp, j)].X
        w_ = dq.act_sqnr_db(X, fmt, L.c, group=G)
        wo = dq.act_sqnr_db(X, fmt, None, group=G)
        act_sqnr[f"K{X.shape[1]}"] = {"with_beta_db": w_, "without_beta_db": wo,
                                      "delta_db": w_ - wo}
    torch.cuda.synchronize()
    if dq.dq_device_error(clear=True) != 0:
        raise RuntimeError("device error word set during the per-kernel timing")

    # ---- the other workloads (reported beside the headline, not in the step)
    peaks_ = (hbm, fp4_peak, fp8_peak, alu_peak)
    configs = {}
    if rank == 0 and not args.headline_only:
        configs["llama8b_attn_nvfp4"] = side_config("llama8b_attn_nvfp4", ["nvfp4"], dev, T, ws,
                                                    peaks_)
        configs["llama8b_mlp_mx"] = side_config("llama8b_mlp_mx", ["mxfp4", "mxint4"], dev, T,
                                                ws, peaks_)
        configs["tiny_layer_256"] = side_config("tiny_layer_256", ["nvfp4"], dev, T, ws, peaks_)
        # whole-model sweep: the 224 linears of a Llama-3.1-8B-shaped model,
        # random bf16 Student-t weights, solved (T = 50) and packed per format
        lin = sweep.llama8b_linears()
        SW = [sweep.student_t_weight(m_, n_, 10_000 + i, dev) for i, (_, m_, n_) in enumerate(lin)]
        sw = {"weights": len(SW), "params": int(sum(W.numel() for W in SW)), "T": 50}
        for f, g in (("int4", 128), ("mxint4", 0), ("mxfp4", 0), ("nvfp4", 0)):
            torch.cuda.synchronize()
            s0, s1 = ev(), ev()
            s0.record(st)
            qs = sweep.solve_and_pack(SW, dq.FORMATS[f], 50, group=g)
            s1.record(st)
            torch.cuda.synchronize()
            sec = 1e-3 * s0.elapsed_time(s1)
            sw[f] = {"group": g or dq.native_group(dq.FORMATS[f]), "seconds": sec,
                     "weights_per_s": len(SW) / sec,
                     "packed_bytes": int(sum(q.codes.numel() + q.scales.numel() for q in qs))}
            del qs
        del SW
        configs["llama8b_sweep_224"] = sw
        torch.cuda.synchronize()
        if dq.dq_device_error(clear=True) != 0:
            raise RuntimeError("device error word set during the side configurations")

    # ---- 8-bit variant (Appendix G.2): MXFP8 linear at the prefill shape of
    # the first weight.  Auxiliary: an error is reported, not raised.
    mxfp8 = None
    if rank == 0 and not args.headline_only:
        try:
            L8 = Layer(Ls[0].W, dq.DQ_MXFP8, 32, dev)
            L8.solve(dq.DQ_MXFP8, T, ws, 32)
            L8.pack(dq.DQ_MXFP8, 32)
            a8 = Act(acts[(Mp, 0)].X, dq.DQ_MXFP8, 32, L8.W.shape[0], dev)
            mxfp8 = time_linear(L8, a8, dq.DQ_MXFP8, 32, fp8_peak)
            mxfp8["peak_tflops"] = fp8_peak
            mxfp8["device_error"] = dq.dq_device_error(clear=True)
            del L8, a8
        except Exception as ex:  # auxiliary measurement: report, do not fail the bench line
            mxfp8 = {"error": str(ex)[:300]}

    # ---- e2e through the public API with host buffers (pinned): the prefill
    # linears of both weights, X host -> device, Y device -> host, every step
    e2e = None
    Xh = [torch.from_numpy(Xs[(Mp, j)]).to(torch.bfloat16).pin_memory() for j in range(len(Ls))]
    Yh = [torch.empty((Mp, L.W.shape[0]), dtype=torch.bfloat16).pin_memory() for L in Ls]
    Xdev = [torch.empty_like(acts[(Mp, j)].X) for j in range(len(Ls))]

    def e2e_step():
        for j, L in enumerate(Ls):
            Xdev[j].copy_(Xh[j], non_blocking=True)
            acts[(Mp, j)].linear(L, fmt, G, X=Xdev[j])
            Yh[j].copy_(acts[(Mp, j)].Y, non_blocking=True)

    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize()
    tot = 0.0
    n_e2e = max(min(args.steps, 10), 3)
    for _ in range(n_e2e):
        flush.fill_(2)
        x0, x1 = ev(), ev()
        x0.record(st)
        e2e_step()
        x1.record(st)
        x1.synchronize()
        tot += x0.elapsed_time(x1)
    tot = dist.max_over_ranks([tot], device=dev)[0]
    e2e = {"value": world * flops_p * n_e2e / (tot * 1e-3) / 1e12, "unit": "TFLOP/s",
           "h2d_bytes_per_step": int(sum(x.numel() * 2 for x in Xh)),
           "d2h_bytes_per_step": int(sum(y.numel() * 2 for y in Yh)),
           "what": f"host bf16 X -> device, act quant + GEMM, bf16 Y -> host, both weights, "
                   f"prefill M={Mp}"}

    if rank != 0:
        return
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        oracle_prepare(Ws)
        v, secs = oracle_linear_sample(Ws, Xs, Mp, rows=64)
        procs = max(1, min(os.cpu_count() or 1, 32))
        sol = oracle_solver_sample(Ws[0], T, procs)
        cpu = {"value": v, "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
               "sample": LINEAR_SAMPLE_DESC.format(rows=64, M=Mp), "seconds": secs,
               "solver": dict(sol, sample=f"Algorithm 1, T={T}, whole {Ws[0].shape[0]}x16 "
                                          f"column tiles of the first weight: one tile on one "
                                          f"core, one tile per process on {procs} processes")}

    # dominant kernel of the step by device time: the solver
    big = max(solver, key=lambda k: solver[k]["ms"])
    m_, n_ = (int(v) for v in big.split("x"))
    sb = solver[big]
    first = f"N{Ls[0].W.shape[0]}_K{Ls[0].W.shape[1]}"
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "fp4(e2m1)",
        "data": "synthetic",
        "config": {"workload": args.workload, "format": FMT_NAME,
                   "weights": [list(L.W.shape) for L in Ls], "M_prefill": Mp, "M_decode": Mds,
                   "T": T, "l2": "flushed before every step (256 MiB write, outside the timed "
                                 "events); the linears run first in the step",
                   "value": "prefill linears (act quant + GEMM), both weights",
                   "parallelism": f"replicas x{world}"},
        "roofline": {"kernel": f"solve_bcd_kernel (+ solve_init_kernel), {big} bf16, T={T}",
                     "bound": "alu", "achieved": sb["tops"], "peak": alu_peak, "unit": "Tops/s",
                     "frac": sb["frac_alu"], "ms_per_launch": sb["ms"],
                     "share_of_step": solve_ms / step_ms,
                     "traffic": measured_traffic(f"solver_{big}_nvfp4_T50",
                                                 ["dq_solver.cu", "dq_device.cuh"]),
                     "algorithmic_bytes": m_ * n_ * 2 + m_ * n_ // 16 * 4 + n_ * 4,
                     "peak_kind": "derived: 148 SM x 128 fp32 lanes x max SM clock",
                     "note": "12 algorithmic fp32 ops / element / round"},
        "roofline_gemm": {"kernel": "w4a4_gemm", "bound": "tensor",
                          "achieved": prefill[first]["gemm_tflops"], "peak": fp4_peak,
                          "unit": "TFLOP/s", "frac": prefill[first]["gemm_frac"],
                          "us_per_launch": prefill[first]["gemm_us"],
                          "shape": f"M={Mp} x N={Ls[0].W.shape[0]} x K={Ls[0].W.shape[1]}",
                          "traffic": measured_traffic(f"gemm_nvfp4_{Mp}x{Ls[0].W.shape[0]}x"
                                                      f"{Ls[0].W.shape[1]}",
                                                      ["dq_gemm.cu", "dq_device.cuh"]),
                          "peak_kind": f"{peak_kind} bf16 burst x 4 (nominal fp4:bf16)"},
        "roofline_act": {"kernel": "quantize_act", "bound": "hbm",
                         "achieved": prefill[first]["act_gbs"], "peak": hbm, "unit": "GB/s",
                         "frac": prefill[first]["act_gbs"] / hbm,
                         "us_per_launch": prefill[first]["act_us"],
                         "algorithmic_bytes": act_bytes(Mp, Ls[0].W.shape[1], fmt, G),
                         "shape": f"M={Mp} x K={Ls[0].W.shape[1]}",
                         "traffic": measured_traffic(f"act_nvfp4_{Mp}x{Ls[0].W.shape[1]}",
                                                     ["dq_quant.cu", "dq_device.cuh"])},
        "solver": solver, "prefill": prefill, "decode": decode, "pack": pack,
        "per_kernel_timing": "after the timed steps: launches back to back between two events, "
                             "each on its own copy of its input (copies > 2x L2)",
        "step_ms": {"prefill_linears": pre_ms / args.steps, "decode_linears": dec_ms / args.steps,
                    "solve": solve_ms / args.steps},
        "solver_modes": {
            "weight": list(L0.W.shape), "T": T, "ms_per_call": mode_ms,
            "frac_alu": {k: (12.0 if k == "both" else 6.0) * L0.W.numel() * T
                         / (v * 1e-3) / 1e12 / alu_peak for k, v in mode_ms.items()},
            "note": "Table 4 arms through dq_solve_scales_ex; algorithmic fp32 ops per "
                    "element per round: 12 (both half-steps), 6 (one half-step)"},
        "configs": configs,
        "mxfp8": mxfp8,
        "act_sqnr": {"per_weight": act_sqnr, "rows": Mp,
                     "note": "SQNR of the dequantised activations mapped back by 1/c vs X, "
                             "measured on the device (dq_act_quant_error); synthetic inputs"},
        "peaks": {"hbm_gbs": hbm, "bf16_tflops": bf16_tf, "fp4_tflops": fp4_peak,
                  "fp8_tflops": fp8_peak, "alu_tops": alu_peak, "kind": peak_kind},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks,
        "e2e": e2e,
        "cpu_baseline": cpu,
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--workload", default=WORKLOAD, choices=[WORKLOAD, "llama8b_attn_nvfp4"],
                    help="the NVFP4 layer the step runs (prefill + decode linears, solve + pack)")
    ap.add_argument("--headline-only", action="store_true",
                    help="skip the other workloads and the MXFP8 line")
    args = ap.parse_args()
    rank, world, local_rank = dist.env_ranks()
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3
    backend = "nccl" if torch.cuda.is_available() and args.impl == "ours" else "gloo"
    dist.init(backend, timeout_s=300)
    try:
        if args.impl == "reference":
            run_reference(args, rank, world)
        else:
            run_ours(args, rank, world, local_rank)
    finally:
        dist.finalize()


if __name__ == "__main__":
    main()
