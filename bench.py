#!/usr/bin/env python3
"""Benchmark of the LLM.int8() mixed-precision decomposition matmul on B200.

One step = one call of the whole forward path (outlier scan + row quantize +
gather, int8 tcgen05 GEMM with the dequantize + fp16 outlier epilogue) on the
6.7B-style FFN up-projection prefill: X fp16 [2048, 4096] with 6 outlier
columns, W [4096, 16384] pre-quantized column-wise (weight conversion is
offline, timed separately).  Metric: effective TOPS = 2*M*N*K / time.

Arms:
  (default)          this library, inputs resident in HBM; ``e2e`` adds the
                     host->device copy of X and device->host copy of Y per step.
  --impl reference   the CPU oracle (plain C, OpenMP) on a bounded row sample.
Multi-GPU (torchrun): independent replicas, one per GPU (the path has no
exchange step); value = all ranks' operations / max-over-ranks time.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "effective TOPS (2MNK/s) of LLM.int8 mixed matmul; % of INT8/HBM roofline"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
INT8_PER_BF16 = 2.0  # nominal dense ratio, 4.5 POPS int8 / 2.25 PFLOP/s bf16
INT8_DATASHEET_TOPS = 4500.0  # B200 dense int8, datasheet
# supplementary configurations of the default line: (workload, threshold or None for its own)
SUPPLEMENTARY = [("hidden_175b", None), ("sweep8k_o0", None), ("sweep8k_o0p1", None), ("sweep8k_o1", None),
                 ("sweep8k_o1", float("inf")), ("ragged_1000x1000x1000", None), ("ragged_2047x4095x4100", None),
                 ("ragged_129x257x520", None), ("ragged_1x1001x1000", None), ("ragged_3x33x24", None)]


def parse_args():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=30)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="ffn_6p7b_prefill")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="CPU-baseline sample budget")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-decode", action="store_true",
                    help="skip the supplementary decode-shape measurement")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the supplementary 175B / sweep / ragged measurements")
    ap.add_argument("--configs", default="",
                    help="comma-separated subset of the supplementary configurations (default: all)")
    ap.add_argument("--leg-seconds", type=float, default=0.25,
                    help="device time each supplementary leg is replayed for (clock record; long enough that the "
                         "power cap applies: its fractions are also given against the sustained peak)")
    ap.add_argument("--graph", action="store_true",
                    help="capture the K timed steps in one CUDA graph (small, launch-bound workloads)")
    return ap.parse_args()


# ------------------------------------------------------------------ peaks
def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    except (OSError, KeyError, ValueError):
        return {"hbm_gbs": FALLBACK_HBM_GBS, "bf16_tflops": FALLBACK_BF16_TFLOPS,
                "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def algorithmic_bytes(M, N, K, n_o):
    """X read + Wq read + fp16 outlier rows of W + scales + Y write."""
    return 2 * M * K + N * K + 2 * n_o * N + 4 * (M + N) + 2 * M * N


# ------------------------------------------------------------------ clocks
REASON_BITS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
               0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}


class ClockSampler:
    """Polls SM clock and clock-event reasons through NVML (read only)."""

    def __init__(self, index: int, period_s: float = 0.002):
        self.samples = []
        self.period = period_s
        self._stop = threading.Event()
        self.ok = False
        self.max_mhz = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self._reasons = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                getattr(pynvml, "nvmlDeviceGetCurrentClocksThrottleReasons")
            self.ok = True
        except Exception as e:  # noqa: BLE001 - clocks are reported as unavailable
            self.err = repr(e)
        self.t = threading.Thread(target=self._run, daemon=True)

    def _run(self):
        while not self._stop.is_set():
            try:
                mhz = self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM)
                rs = int(self._reasons(self.h))
                self.samples.append((time.perf_counter(), mhz, rs))
            except Exception:  # noqa: BLE001
                pass
            time.sleep(self.period)

    def start(self):
        if self.ok:
            self.t.start()
        return self

    def stop(self):
        self._stop.set()
        if self.ok:
            self.t.join(timeout=2)

    def window(self, t0, t1):
        """Median SM clock, sample count and reasons seen inside [t0, t1]."""
        if not self.ok:
            return {"sm_mhz": None, "samples": 0, "reasons": []}
        win = [s for s in self.samples if t0 <= s[0] <= t1]
        reasons = sorted({name for _, _, r in win for bit, name in REASON_BITS.items() if r & bit})
        return {"sm_mhz": statistics.median([s[1] for s in win]) if win else None, "samples": len(win),
                "reasons": reasons}

    def summary(self, t0, t1):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "note": "NVML unavailable"}
        win = [s for s in self.samples if t0 <= s[0] <= t1]
        note = f"{len(win)} NVML samples inside the timed region"
        if len(win) < 3:  # short region: widen to the samples taken under load around it
            win = [s for s in self.samples if t0 - 1.0 <= s[0] <= t1 + 0.2]
            note += f"; widened to {len(win)} samples within 1 s before it"
        reasons = set()
        for _, _, r in win:
            for bit, name in REASON_BITS.items():
                if r & bit:
                    reasons.add(name)
        return {"sm_mhz": statistics.median([s[1] for s in win]) if win else None, "sm_max_mhz": self.max_mhz,
                "reasons": sorted(reasons), "note": note}


# ------------------------------------------------------------------ distributed plumbing
class Dist:
    """One process per GPU (torchrun's RANK / LOCAL_RANK / WORLD_SIZE): NCCL
    on GPUs; gloo when no GPU is present (the host-side logic under CPU
    tests).  Only used for the barrier around the timed region and the
    max-over-ranks of the timings: the path itself needs no exchange."""

    def __init__(self, backend=None):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.backend = backend
        self.pg = None

    def init(self, torch):
        backend = self.backend or ("nccl" if torch.cuda.is_available() else "gloo")
        self.backend = backend
        if self.world > 1:
            import datetime

            import torch.distributed as dist
            timeout = datetime.timedelta(seconds=120)  # ranks that wait on a lost peer end with an error
            if backend == "nccl":
                torch.cuda.set_device(self.local)
                dist.init_process_group("nccl", timeout=timeout, device_id=torch.device("cuda", self.local))
            else:
                dist.init_process_group(backend, timeout=timeout)
            self.pg = dist
        elif backend == "nccl":
            torch.cuda.set_device(0)

    def barrier(self, torch):
        if self.pg:
            self.pg.barrier()

    def max(self, torch, v: float) -> float:
        if not self.pg:
            return v
        t = torch.tensor([v], dtype=torch.float64, device="cuda" if self.backend == "nccl" else "cpu")
        self.pg.all_reduce(t, op=self.pg.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.pg:
            self.pg.destroy_process_group()


# ------------------------------------------------------------------ CPU oracle sample
def oracle_sample(X, W, tau, rows, weight):
    """Run the oracle's a1-a7 on the first `rows` rows; returns seconds."""
    import oracle
    Xs = X[:rows]
    t0 = time.perf_counter()
    oracle.mixed_matmul(Xs, W, tau, weight=weight)
    return time.perf_counter() - t0


def calibrate_rows(X, W, tau, weight, budget_s, M):
    """Rows of the oracle sample that take about budget_s on this host (the
    oracle parallelises over rows, so calibrate with one row per thread)."""
    import oracle
    nt = max(1, oracle.num_threads())
    rows0 = min(M, nt)
    t0 = oracle_sample(X, W, tau, rows0, weight)
    per_row = max(t0, 1e-6) / rows0
    rows = int(budget_s / per_row) // nt * nt
    return int(max(rows0, min(M, rows)))


def cpu_baseline(wl_, X, W, budget_s):
    import oracle
    weight = oracle.quantize_weight(W)  # offline conversion, not timed
    rows = calibrate_rows(X, W, wl_.tau, weight, budget_s, wl_.M)
    t = oracle_sample(X, W, wl_.tau, rows, weight)
    tops = 2.0 * rows * wl_.N * wl_.K / t / 1e12
    return {"value": tops, "unit": "TOPS", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"oracle a1-a7 on the first {rows} of {wl_.M} rows of X ({t:.2f} s); all steps are "
                      f"linear in the rows, so TOPS = 2*rows*N*K/t"}


# ------------------------------------------------------------------ reference arm
def run_reference(args, wl_, dist):
    if dist.rank != 0:
        return 0
    import numpy as np  # noqa: F401

    import oracle
    import workloads as wl
    X, W = wl.make_inputs(wl_)
    weight = oracle.quantize_weight(W)
    per_step = min(0.5, 150.0 / max(1, args.steps + args.warmup))
    rows = calibrate_rows(X, W, wl_.tau, weight, per_step, wl_.M)
    for _ in range(args.warmup):
        oracle_sample(X, W, wl_.tau, rows, weight)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_sample(X, W, wl_.tau, rows, weight)
    el = time.perf_counter() - t0
    tops = 2.0 * rows * wl_.N * wl_.K * args.steps / el / 1e12
    sample = (f"each step: oracle a1-a7 on the first {rows} of {wl_.M} rows (all steps are linear in the rows; "
              f"weights converted once, untimed)")
    line = {
        "impl": "reference", "metric": METRIC, "value": tops, "unit": "TOPS", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": el / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int8", "data": "synthetic",
        "config": config_of(wl_, None),
        "cpu_baseline": {"value": tops, "unit": "TOPS", "cores": oracle.num_threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": tops, "unit": "TOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def config_of(wl_, n_o, extra=None):
    c = {"workload": wl_.name, "M": wl_.M, "N": wl_.N, "K": wl_.K, "tau": wl_.tau,
         "outlier_columns_planted": int(wl_.n_planted if wl_.planted is None else len(wl_.planted)),
         "outlier_columns_detected": n_o, "global_batch": wl_.M, "parallelism": "replicas"}
    if extra:
        c.update(extra)
    return c


# ------------------------------------------------------------------ decode shapes
def measure_decode(L, torch, dev, peaks, names=("decode_m1", "decode_m8", "decode_m32"), reps=20):
    """Decode-shaped calls of llmint8_mixed_matmul (M <= 32, HBM-bound on
    streaming Wq): per-call time from a CUDA graph of one pass over rotating
    weight copies (together > 3x L2, so every call streams Wq from HBM),
    replayed `reps` times between CUDA events on the replaying stream."""
    import workloads as wl
    out = {}
    for name in names:
        w = wl.get(name)
        X_np, W_np = wl.make_inputs(w)
        W = torch.from_numpy(W_np).to(dev)
        X = torch.from_numpy(X_np).to(dev)
        Wq0, cs0 = L.quantize_weight_colwise(W)
        n_sets = max(2, math.ceil(3 * L2_BYTES / Wq0.numel()))
        sets = [(Wq0.clone(), cs0.clone(), torch.empty((w.M, w.N), dtype=torch.float16, device=dev),
                 L.empty_workspace(w.M, w.N, w.K, w.K, device=dev)) for _ in range(n_sets)]
        del Wq0, cs0

        def one_pass(on):
            for (q, c, y, ws) in sets:
                L.llmint8_mixed_matmul(X, q, c, W, w.tau, w.K, y, ws, on)

        for _ in range(3):
            one_pass(torch.cuda.current_stream())
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            one_pass(torch.cuda.current_stream())
        g.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            g.replay()
        e1.record()
        torch.cuda.synchronize()
        t = e0.elapsed_time(e1) * 1e-3 / (reps * n_sets)
        st, flags = L.llmint8_check_status(sets[0][3])
        if st != 0:
            raise RuntimeError(f"device status after the {name} run: {st} flags={flags}")
        n_o = int(L.workspace_views(sets[0][3], w.M, w.N, w.K, w.K)["n_outlier"].item())
        byts = algorithmic_bytes(w.M, w.N, w.K, n_o)
        out[name] = {"M": w.M, "N": w.N, "K": w.K, "us_per_call": t * 1e6, "achieved_gbs": byts / t / 1e9,
                     "frac_hbm": byts / t / 1e9 / peaks["hbm_gbs"],
                     "roofline_us": byts / (peaks["hbm_gbs"] * 1e9) * 1e6, "algorithmic_bytes": byts,
                     "kernels_per_call": L.llmint8_mixed_matmul_kernels(X, w.N),
                     "kernels": L.llmint8_mixed_matmul_path(X, sets[0][0], w.K), "n_outlier": n_o,
                     "timing": f"CUDA graph of {n_sets} calls on rotating Wq copies, replayed {reps}x"}
        del sets, g
    return out


# ------------------------------------------------------------------ supplementary configurations
def replay_for(torch, stream, graph, units_per_replay, seconds, clocks):
    """Replay `graph` back to back for about `seconds` of device time (at
    least 3 replays), timed by CUDA events on the replaying stream; returns
    (us per unit, clock record of the window)."""
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    graph.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    one = max(e0.elapsed_time(e1) * 1e-3, 1e-6)
    reps = max(3, int(math.ceil(seconds / one)))
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    e0.record(stream)
    for _ in range(reps):
        graph.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    t1 = time.perf_counter()
    us = e0.elapsed_time(e1) * 1e3 / (reps * units_per_replay)
    clk = clocks.window(t0, t1)
    clk["replays"] = reps
    return us, clk


def capture(torch, fn):
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn(torch.cuda.current_stream())
    g.replay()
    torch.cuda.synchronize()
    return g


def roofline_times(M, N, K, n_o, peaks):
    """T_roof = max(2MNK / int8 peak, algorithmic bytes / HBM bandwidth) for
    the measured peaks and for the datasheet ones."""
    ops = 2.0 * M * N * K
    byts = algorithmic_bytes(M, N, K, n_o)
    meas = (peaks["bf16_tflops"] * INT8_PER_BF16 * 1e12, peaks["hbm_gbs"] * 1e9)
    sust = (peaks["bf16_tflops_sustained"] * INT8_PER_BF16 * 1e12, peaks["hbm_gbs"] * 1e9)
    ds = (INT8_DATASHEET_TOPS * 1e12, 8000.0 * 1e9)
    out = {}
    # "measured": the burst figures (a kernel timed alone); "sustained": the
    # measured GEMM rate under the power cap (a kernel timed in a long run);
    # "datasheet": 4.5 POPS int8, 8 TB/s
    for tag, (p_int8, bw) in (("measured", meas), ("sustained", sust), ("datasheet", ds)):
        t_t, t_m = ops / p_int8, byts / bw
        out[tag] = {"t_roof_us": max(t_t, t_m) * 1e6, "bound": "tensor" if t_t >= t_m else "hbm",
                    "int8_tops": p_int8 / 1e12, "hbm_gbs": bw / 1e9}
    return out, byts


def measure_config(L, torch, dev, peaks, clocks, name, tau, leg_s):
    """One supplementary configuration: the whole call (one pass of
    llmint8_mixed_matmul over rotating input sets > 3x L2, as a CUDA graph),
    and for the multi-kernel paths the activation step and the GEMM alone,
    each replayed for about leg_s seconds with its own clock record."""
    import workloads as wl
    w = wl.get(name)
    tau = w.tau if tau is None else tau
    M, N, K = w.M, w.N, w.K
    X_np, W_np = wl.make_inputs(w)
    W = torch.from_numpy(W_np).to(dev)
    X0 = torch.from_numpy(X_np).to(dev)
    del W_np
    Wq0, cs0 = L.quantize_weight_colwise(W)
    ldq = L.round_up(K, 16)
    per_set = 2 * M * K + Wq0.numel() + 2 * M * N + M * ldq
    n_sets = max(2, min(16, math.ceil(3 * L2_BYTES / per_set)))
    sets = [{"X": X0 if i == 0 else X0.clone(), "Wq": Wq0 if i == 0 else Wq0.clone(),
             "cs": cs0 if i == 0 else cs0.clone(), "Y": torch.empty((M, N), dtype=torch.float16, device=dev),
             "ws": L.empty_workspace(M, N, K, K, device=dev)} for i in range(n_sets)]
    stream = torch.cuda.current_stream()

    def path_pass(on):
        for st in sets:
            L.llmint8_mixed_matmul(st["X"], st["Wq"], st["cs"], W, tau, K, st["Y"], st["ws"], on)

    for _ in range(2):
        path_pass(stream)
    torch.cuda.synchronize()
    st_, flags = L.llmint8_check_status(sets[0]["ws"])
    if st_ != 0:
        raise RuntimeError(f"device status after {name}: {st_} flags={flags}")
    n_o = int(L.workspace_views(sets[0]["ws"], M, N, K, K)["n_outlier"].item())
    kernels = L.llmint8_mixed_matmul_path(sets[0]["X"], sets[0]["Wq"], K)
    g = capture(torch, path_pass)
    t_path, clk_path = replay_for(torch, stream, g, n_sets, leg_s, clocks)
    del g
    roof, byts = roofline_times(M, N, K, n_o, peaks)
    ops = 2.0 * M * N * K
    out = {"M": M, "N": N, "K": K, "tau": tau, "n_outlier": n_o, "kernels": kernels, "us_per_step": t_path,
           "tops": ops / (t_path * 1e-6) / 1e12, "algorithmic_bytes": byts,
           "path_frac": {k: v["t_roof_us"] / t_path for k, v in roof.items()}, "roofline": roof,
           "rotating_sets": n_sets, "clocks": {"path": clk_path}}
    if len(kernels) > 1:
        acts = [{"Xq": torch.empty((M, ldq), dtype=torch.int8, device=dev),
                 "row_scale": torch.empty(M, dtype=torch.float32, device=dev),
                 "outlier_idx": torch.empty(K, dtype=torch.int32, device=dev),
                 "n_outlier": torch.empty(1, dtype=torch.int32, device=dev),
                 "Xo": torch.empty((M, K), dtype=torch.float16, device=dev)} for _ in sets]

        def act_pass(on):
            for st, a in zip(sets, acts):
                L.llmint8_quantize_act_rowwise_outliers(st["X"], tau, a["Xq"], a["row_scale"], a["outlier_idx"],
                                                        a["n_outlier"], a["Xo"], st["ws"], on)

        def gemm_pass(on):
            for st, a in zip(sets, acts):
                L.llmint8_mixed_gemm(a["Xq"], a["row_scale"], a["outlier_idx"], a["n_outlier"], a["Xo"], st["Wq"],
                                     st["cs"], W, K, st["Y"], st["ws"], on)

        act_pass(stream)
        gemm_pass(stream)
        torch.cuda.synchronize()
        g = capture(torch, act_pass)
        t_act, clk_act = replay_for(torch, stream, g, n_sets, leg_s, clocks)
        del g
        g = capture(torch, gemm_pass)
        t_gemm, clk_gemm = replay_for(torch, stream, g, n_sets, leg_s, clocks)
        del g, acts
        out.update({"activation_us": t_act, "gemm_us": t_gemm, "gemm_tops": ops / (t_gemm * 1e-6) / 1e12,
                    "gemm_frac": {k: ops / (t_gemm * 1e-6) / 1e12 / v["int8_tops"] for k, v in roof.items()},
                    "activation_gbs": 3 * M * K / (t_act * 1e-6) / 1e9})
        out["clocks"].update({"activation": clk_act, "gemm": clk_gemm})
    st_, flags = L.llmint8_check_status(sets[0]["ws"])
    if st_ != 0:
        raise RuntimeError(f"device status after {name}: {st_} flags={flags}")
    del sets, W, X0, Wq0, cs0
    torch.cuda.empty_cache()
    return out


def measure_supplementary(L, torch, dev, peaks, clocks, leg_s, only=""):
    out = {}
    pick = {x for x in only.split(",") if x}
    for name, tau in SUPPLEMENTARY:
        key = name if tau is None else f"{name}_tau_" + ("inf" if math.isinf(tau) else format(tau, "g"))
        if pick and key not in pick:
            continue
        out[key] = measure_config(L, torch, dev, peaks, clocks, name, tau, leg_s)
    return out


# ------------------------------------------------------------------ our arm
def source_digest(path):
    """First 16 hex digits of the sha256 of a C++ source with its comments
    removed and its white space collapsed: the code the counters were taken
    on, whatever its comments say."""
    with open(path) as f:
        src = f.read()
    src = re.sub(r"//[^\n]*", "", src)
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    src = re.sub(r"\s+", " ", src).strip()
    return hashlib.sha256(src.encode()).hexdigest()[:16]


def recorded_traffic(wl_name):
    """DRAM bytes per GEMM launch from a committed ncu summary, only if it was
    taken on the kernel source as it is now."""
    try:
        with open(os.path.join(ROOT, "profiles", "gemm_i8_traffic.json")) as f:
            d = json.load(f)
    except (OSError, ValueError):
        return None
    src = os.path.join(ROOT, "int8_quantized_matmul_colwise_b200", "csrc", "gemm_i8.cu")
    ent = d.get(wl_name)
    if not ent or ent.get("gemm_code_sha256_16") != source_digest(src):
        return None
    return ent.get("dram_bytes_per_launch")


def run_ours(args, wl_, dist):
    import numpy as np
    import torch

    import int8_quantized_matmul_colwise_b200 as L
    import workloads as wl

    dist.init(torch)
    dev = torch.device("cuda", torch.cuda.current_device())
    peaks = load_peaks()
    int8_peak = peaks["bf16_tflops"] * INT8_PER_BF16

    X_np, W_np = wl.make_inputs(wl_)
    M, N, K = wl_.M, wl_.N, wl_.K
    cap = K
    W = torch.from_numpy(W_np).to(dev)
    X0 = torch.from_numpy(X_np).to(dev)

    # offline weight conversion (reported, not part of the metric)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    Wq0, cs0 = L.quantize_weight_colwise(W)
    e1.record()
    torch.cuda.synchronize()
    wq_ms = e0.elapsed_time(e1)

    # the same conversion warm (the first call above also loads the module):
    # 2KN bytes read twice (column maxima, then codes) + KN written; reported
    # against the 2KN + KN algorithmic bytes
    reps_q = 5
    L.quantize_weight_colwise(W)  # untimed: its outputs are the blocks the timed calls reuse
    torch.cuda.synchronize()
    e0.record()
    for _ in range(reps_q):
        L.quantize_weight_colwise(W)
    e1.record()
    torch.cuda.synchronize()
    wq_warm_us = e0.elapsed_time(e1) * 1e3 / reps_q
    wq_bytes = 3 * K * N + 4 * N
    ws_bytes = L.llmint8_workspace_size(M, N, K, cap)
    per_set = 2 * M * K + Wq0.numel() + 2 * M * N + M * L.round_up(K, 16)
    n_sets = max(2, min(64, math.ceil(3 * L2_BYTES / per_set)))
    sets = []
    for i in range(n_sets):
        sets.append({
            "X": X0.clone(), "Wq": Wq0.clone(), "cs": cs0.clone(),
            "Y": torch.empty((M, N), dtype=torch.float16, device=dev),
            "ws": L.empty_workspace(M, N, K, cap, device=dev),
        })
    stream = torch.cuda.current_stream()

    def step(i, on=stream):
        s = sets[i % n_sets]
        L.llmint8_mixed_matmul(s["X"], s["Wq"], s["cs"], W, wl_.tau, cap, s["Y"], s["ws"], on)

    clocks = ClockSampler(torch.cuda.current_device()).start()
    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    st, flags = L.llmint8_check_status(sets[0]["ws"])
    if st != 0:
        raise RuntimeError(f"device status after warm-up: {st} flags={flags}")
    views = L.workspace_views(sets[0]["ws"], M, N, K, cap)
    n_o = int(views["n_outlier"].item())
    n_kern = L.llmint8_mixed_matmul_kernels(sets[0]["X"], N)  # 1: a one-kernel decode path
    kern_names = L.llmint8_mixed_matmul_path(sets[0]["X"], sets[0]["Wq"], K)

    graph = None
    if args.graph:  # the K timed steps as one CUDA graph, captured before the timed region
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):  # captured on torch's side stream, replayed on `stream`
            for i in range(args.steps):
                step(i, torch.cuda.current_stream())
        graph.replay()
        torch.cuda.synchronize()

    # ---- timed region: exactly K steps, inputs resident in HBM
    dist.barrier(torch)
    torch.cuda.synchronize()
    ev_a, ev_b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t_host0 = time.perf_counter()
    ev_a.record(stream)
    if graph is not None:
        graph.replay()
    else:
        for i in range(args.steps):
            step(i)
    ev_b.record(stream)
    torch.cuda.synchronize()
    t_host1 = time.perf_counter()
    dist.barrier(torch)
    el_ms = dist.max(torch, ev_a.elapsed_time(ev_b))
    clk = clocks.summary(t_host0, t_host1)

    ops = 2.0 * M * N * K
    value = dist.world * ops * args.steps / (el_ms / 1e3) / 1e12
    ms_per_step = el_ms / args.steps

    byts = algorithmic_bytes(M, N, K, n_o)
    if n_kern == 1:
        # one kernel per step: its duration is the step's, taken over the timed region
        t_step = ms_per_step * 1e-3
        gbs = byts / t_step / 1e9
        roofline = {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                    "frac": gbs / peaks["hbm_gbs"], "traffic": None,
                    "kernel": kern_names[0] + " (a1-a7 in one kernel)",
                    "peak_note": f"measured HBM copy bandwidth ({peaks['source']}); algorithmic bytes per launch "
                                 f"= 2MK + NK + 2*n_o*N + 4(M+N) + 2MN = {byts}"}
        path = {"t_roof_us": byts / (peaks["hbm_gbs"] * 1e9) * 1e6, "t_step_us": ms_per_step * 1e3,
                "frac": byts / (peaks["hbm_gbs"] * 1e9) / t_step, "algorithmic_bytes": byts,
                "int8_peak_tops": int8_peak, "hbm_gbs": peaks["hbm_gbs"]}
    else:
        # ---- per-kernel durations (same inputs, split entry points, events on the launching stream)
        acts = []
        for s in sets:
            acts.append({
                "Xq": torch.empty((M, L.round_up(K, 16)), dtype=torch.int8, device=dev),
                "row_scale": torch.empty(M, dtype=torch.float32, device=dev),
                "outlier_idx": torch.empty(cap, dtype=torch.int32, device=dev),
                "n_outlier": torch.empty(1, dtype=torch.int32, device=dev),
                "Xo": torch.empty((M, cap), dtype=torch.float16, device=dev),
            })
        n_k = max(10, min(args.steps, 200))
        for i in range(n_k):  # warm-up; leaves every set's activation quantized
            s, a = sets[i % n_sets], acts[i % n_sets]
            L.llmint8_quantize_act_rowwise_outliers(s["X"], wl_.tau, a["Xq"], a["row_scale"], a["outlier_idx"],
                                                    a["n_outlier"], a["Xo"], s["ws"], stream)
            L.llmint8_mixed_gemm(a["Xq"], a["row_scale"], a["outlier_idx"], a["n_outlier"], a["Xo"], s["Wq"],
                                 s["cs"], W, K, s["Y"], s["ws"], stream)
        torch.cuda.synchronize()
        # the GEMM alone: one CUDA graph of n_k launches back to back on the
        # rotating sets (the host's launch overhead stays out of the timing)
        g_gemm = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_gemm):
            cur = torch.cuda.current_stream()
            for i in range(n_k):
                s, a = sets[i % n_sets], acts[i % n_sets]
                L.llmint8_mixed_gemm(a["Xq"], a["row_scale"], a["outlier_idx"], a["n_outlier"], a["Xo"], s["Wq"],
                                     s["cs"], W, K, s["Y"], s["ws"], cur)
        g_gemm.replay()
        torch.cuda.synchronize()
        ev_a.record(stream)
        g_gemm.replay()
        ev_b.record(stream)
        torch.cuda.synchronize()
        t_gemm = dist.max(torch, ev_a.elapsed_time(ev_b) * 1e3 / n_k)  # us
        del g_gemm
        # the activation step is short next to the host's launch overhead: time
        # it as one CUDA graph of n_k calls (its two kernels back to back)
        g_act = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_act):
            cur = torch.cuda.current_stream()
            for i in range(n_k):
                s, a = sets[i % n_sets], acts[i % n_sets]
                L.llmint8_quantize_act_rowwise_outliers(s["X"], wl_.tau, a["Xq"], a["row_scale"], a["outlier_idx"],
                                                        a["n_outlier"], a["Xo"], s["ws"], cur)
        g_act.replay()
        torch.cuda.synchronize()
        ev_a.record(stream)
        g_act.replay()
        ev_b.record(stream)
        torch.cuda.synchronize()
        t_quant = ev_a.elapsed_time(ev_b) * 1e3 / n_k
        del g_act
        gemm_tops = ops / (t_gemm * 1e-6) / 1e12

        traffic = recorded_traffic(wl_.name)
        roofline = {"bound": "tensor", "achieved": gemm_tops, "peak": int8_peak, "unit": "TFLOP/s",
                    "frac": gemm_tops / int8_peak, "traffic": traffic,
                    "kernel": "gemm_i8_kernel (tcgen05 kind::i8 + dequant/outlier epilogue)",
                    "peak_note": f"int8 dense = {INT8_PER_BF16:g} x bf16 burst {peaks['bf16_tflops']:.1f} TFLOP/s "
                                 f"({peaks['source']}); algorithmic ops per launch = 2MNK = {ops:.4g}",
                    "peak_datasheet": INT8_DATASHEET_TOPS, "frac_datasheet": gemm_tops / INT8_DATASHEET_TOPS}
        roof2, _ = roofline_times(M, N, K, n_o, peaks)
        t_roof = roof2["measured"]["t_roof_us"] * 1e-6
        path = {"t_roof_us": t_roof * 1e6, "t_step_us": ms_per_step * 1e3, "frac": t_roof / (ms_per_step * 1e-3),
                "frac_datasheet": roof2["datasheet"]["t_roof_us"] / (ms_per_step * 1e3),
                "t_roof_datasheet_us": roof2["datasheet"]["t_roof_us"],
                "algorithmic_bytes": byts, "int8_peak_tops": int8_peak, "int8_datasheet_tops": INT8_DATASHEET_TOPS,
                "hbm_gbs": peaks["hbm_gbs"], "scan_quantize_us": t_quant, "gemm_us": t_gemm,
                "scan_quantize_gbs": (2 * M * K + M * K) / (t_quant * 1e-6) / 1e9,
                "legs_note": "gemm_us / scan_quantize_us: the split entry points replayed from CUDA graphs"}

    # ---- end to end through the public API with host buffers: every step
    # copies its X from pinned host memory and its Y back; the copies run on
    # two copy streams so that step i's compute overlaps the H2D of step i+1
    # and the D2H of step i-1 (events order each step's three parts)
    n_e = max(5, min(args.steps, 50))
    Xh = [torch.from_numpy(X_np).pin_memory() for _ in range(2)]
    Yh = [torch.empty((M, N), dtype=torch.float16).pin_memory() for _ in range(2)]
    h2d, d2h = torch.cuda.Stream(), torch.cuda.Stream()
    n_buf = min(n_sets, 3)

    def e2e_run(n):
        loaded = [torch.cuda.Event() for _ in range(n)]
        done = [torch.cuda.Event() for _ in range(n)]
        copied = [torch.cuda.Event() for _ in range(n)]
        for i in range(n):
            s = sets[i % n_buf]
            with torch.cuda.stream(h2d):
                if i >= n_buf:
                    h2d.wait_event(done[i - n_buf])  # the compute that read this X buffer has finished
                s["X"].copy_(Xh[i % 2], non_blocking=True)
                loaded[i].record(h2d)
            stream.wait_event(loaded[i])
            if i >= n_buf:
                stream.wait_event(copied[i - n_buf])  # the previous D2H of this Y buffer has finished
            L.llmint8_mixed_matmul(s["X"], s["Wq"], s["cs"], W, wl_.tau, cap, s["Y"], s["ws"], stream)
            done[i].record(stream)
            with torch.cuda.stream(d2h):
                d2h.wait_event(done[i])
                Yh[i % 2].copy_(s["Y"], non_blocking=True)
                copied[i].record(d2h)
        return copied[-1]

    e2e_run(3)
    torch.cuda.synchronize()
    ev_a.record(stream)
    h2d.wait_event(ev_a)
    last = e2e_run(n_e)
    stream.wait_event(last)
    ev_b.record(stream)
    torch.cuda.synchronize()
    e2e_ms = dist.max(torch, ev_a.elapsed_time(ev_b)) / n_e
    e2e = {"value": dist.world * ops / (e2e_ms * 1e-3) / 1e12, "unit": "TOPS",
           "h2d_bytes_per_step": Xh[0].numel() * 2, "d2h_bytes_per_step": Yh[0].numel() * 2,
           "ms_per_step": e2e_ms, "steps": n_e,
           "note": "X copied in and Y copied out every step on two copy streams, overlapping the neighbouring "
                   "steps' compute; timed from the first H2D to the last D2H"}

    st, flags = L.llmint8_check_status(sets[0]["ws"])
    if st != 0:
        raise RuntimeError(f"device status after the run: {st} flags={flags}")

    cpu = None
    if dist.rank == 0 and dist.world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(wl_, X_np, W_np, args.cpu_seconds)

    line = {
        "metric": METRIC, "value": value, "unit": "TOPS", "n_gpus": dist.world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "int8", "data": "synthetic",
        "config": config_of(wl_, n_o, {
            "l2": f"{n_sets} rotating input sets (X, Wq, Y, workspace) of {per_set / 2**20:.0f} MiB each "
                  f"> 3x L2; consecutive steps touch different buffers",
            "weight_quant_ms_offline": wq_ms, "weight_quant_warm_us": wq_warm_us,
            "weight_quant_hbm_frac": wq_bytes / (wq_warm_us * 1e-6) / (peaks["hbm_gbs"] * 1e9),
            "workspace_bytes": ws_bytes,
            "launch": ("llmint8_mixed_matmul: 1 kernel (a1-a7 fused)" if n_kern == 1 else
                       f"llmint8_mixed_matmul: {n_kern} kernels chained with programmatic dependent launch") +
                      ("; the K steps replayed from one CUDA graph" if args.graph else "")}),
        "roofline": roofline, "path_roofline": path, "cpu_baseline": cpu, "e2e": e2e,
        "gpu_launches": n_kern * args.steps, "clocks": clk,
    }
    if not args.no_decode and M > 32:
        line["decode"] = measure_decode(L, torch, dev, peaks)
    if not args.no_configs and M > 32 and dist.world == 1:
        sets.clear()
        torch.cuda.empty_cache()
        line["configs"] = measure_supplementary(L, torch, dev, peaks, clocks, args.leg_seconds, args.configs)
    clocks.stop()
    if dist.rank == 0:
        print(json.dumps(line), flush=True)
    dist.close()
    return 0


def main():
    args = parse_args()
    import workloads as wl
    wl_ = wl.get(args.workload)
    dist = Dist()
    if args.impl == "reference":
        return run_reference(args, wl_, dist)
    return run_ours(args, wl_, dist)


if __name__ == "__main__":
    sys.exit(main())
