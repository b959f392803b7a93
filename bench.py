"""Benchmark of the W4A16 + gated-EC layer on B200.

Step = one pass of the layer (quantised 4-bit weights, fused gated EC) over
one batch of synthetic input for the decode GEMV workload: the 7B-style MLP
up-projection (K=4096, N=11008, EC rank 64, b_g=-1, 5 % outlier tokens), run
at M = 1, 4 and 16 tokens (three calls, 21 tokens per step).  Every step
reads a different one of several identical weight copies whose total exceeds
twice the L2 size, so each call streams its weights from HBM.

Prints one JSON line (see the keys below).  Multi-GPU: one process per GPU
under torchrun; every rank runs the same replica workload (the layer needs
no collective), timing is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

K_, N_, R_ = 4096, 11008, 64
MS = (1, 4, 16)
METRIC = "W4+gated-EC layer tokens/s (decode GEMV, M in {1,4,16}, K=4096, N=11008, r=64)"


def alg_bytes(M, K, N, r):
    return K * N / 2 + 2 * N + 2 * M * K + 2 * M * N + (2 * (K * r + r * N + K) if r else 0)


def alg_flops(M, K, N, r):
    return 2 * M * K * N + (2 * M * K * r + 2 * M * r * N + 2 * M * K if r else 0)


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d.get("hbm_gbs", 6650.0), d.get("bf16_tflops", 1590.0), d.get("bf16_tflops_sustained", 1400.0), "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during a region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines: list[str] = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, FileNotFoundError):
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------------------
# reference arm: the CPU oracle on a bounded sample of the same workload
# ----------------------------------------------------------------------------

def oracle_sample_setup(n_cols: int):
    from oracle import spear_oracle as O
    from w4_gemm_gated_b200 import synth
    L = synth.decode(16, force_outlier=True)
    q, s = O.quantize_rtn(L.W, 0)
    cols = np.arange(n_cols)
    xs = {M: synth.decode(M, force_outlier=True).x for M in MS}
    return O, L, q[cols], s[cols], L.B[:, cols], xs


def oracle_step(O, L, q, s, B, xs):
    for M in MS:
        O.linear(xs[M], q, s, 0, L.A, B, L.w_g, L.b_g)


def cpu_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        n = [d.get("num_threads", 0) for d in info if d.get("internal_api") in ("openblas", "mkl", "blis")]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


def time_oracle(target_s: float = 15.0, n_cols: int = 1376):
    O, L, q, s, B, xs = oracle_sample_setup(n_cols)
    oracle_step(O, L, q, s, B, xs)  # warm
    t0 = time.perf_counter()
    n = 0
    while True:
        oracle_step(O, L, q, s, B, xs)
        n += 1
        el = time.perf_counter() - t0
        if el >= target_s or n >= 200:
            break
    frac = n_cols / N_
    tokens = sum(MS) * n * frac      # full-layer tokens equivalent of the computed columns
    return {"value": tokens / el, "unit": "tokens/s", "cores": cpu_threads(), "kind": "oracle",
            "sample": f"{n} oracle steps (M=1,4,16) on {n_cols} of {N_} output columns, "
                      f"{el:.1f} s, scaled to the full layer by column fraction"}


# DRAM bytes per decode launch from the ncu captures summarised in profiles/
# (dram__bytes_read.sum + dram__bytes_write.sum, one launch at M = 1 and at M = 16),
# valid only while the decode kernel sources are the ones captured.
DECODE_TRAFFIC = {"sources_sha1": "2b2f809a8cf32a5360f470a3cd29ed42a7616859",
                  "bytes_per_launch": {1: 24592384, 16: 24724992}}
DECODE_SOURCES = ("w4_gemm_gated_b200/csrc/decode3.cu", "w4_gemm_gated_b200/csrc/common.cuh",
                  "w4_gemm_gated_b200/csrc/tma.cuh")


def decode_traffic_per_step():
    """DRAM bytes of one step (M = 1, 4, 16) from the captures, or None if the
    kernel changed since (M = 4 runs the M = 1 instantiation; its x adds 24 KB)."""
    import hashlib
    h = hashlib.sha1()
    for f in DECODE_SOURCES:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    if h.hexdigest() != DECODE_TRAFFIC["sources_sha1"]:
        return None
    b = DECODE_TRAFFIC["bytes_per_launch"]
    return b[1] + (b[1] + 2 * 3 * 4096) + b[16]


def max_over_ranks(ms: float, world: int, device) -> float:
    """The slowest rank's elapsed time (every rank calls this, in the same order)."""
    import torch
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_step_per_rank: float, steps: int, world: int, max_ms: float) -> float:
    """Units processed by all ranks (replicas: every rank runs the same step) per second."""
    return units_per_step_per_rank * steps * world / (max_ms * 1e-3)


def run_reference(args, rank, world):
    if rank != 0:
        return
    n_cols = 1376
    O, L, q, s, B, xs = oracle_sample_setup(n_cols)
    for _ in range(args.warmup):
        oracle_step(O, L, q, s, B, xs)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_step(O, L, q, s, B, xs)
    el = time.perf_counter() - t0
    frac = n_cols / N_
    value = sum(MS) * args.steps * frac / el
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        # the time of the work actually done: each step computes n_cols of the N output columns
        "ms_per_step": el * 1e3 / args.steps,
        "ms_per_step_full_layer_extrapolated": el * 1e3 / args.steps / frac,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": "decode GEMV K=4096 N=11008 r=64, M in {1,4,16} (7B MLP up-projection)",
                   "sample_columns": n_cols},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cpu_threads(), "kind": "oracle",
                         "sample": f"each step on {n_cols} of {N_} output columns, scaled by column fraction"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------
# our arm
# ----------------------------------------------------------------------------

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-prefill", action="store_true")
    ap.add_argument("--no-stack", action="store_true", help="skip the 32-layer stack (config 4) key")
    ap.add_argument("--profile-case", choices=["decode", "prefill"], default=None,
                    help="run only --steps launches of one kernel on a small case (for ncu captures); "
                         "prints no bench line")
    ap.add_argument("--m", type=int, default=16, help="tokens of the --profile-case launch")
    ap.add_argument("--sweep", action="store_true",
                    help="dispatch sweep (M x (K, N) x r x scale kind): time every path, check the dispatcher")
    ap.add_argument("--stack", action="store_true",
                    help="32-layer decoder stack of W4 linears (ECs on layers 0, 1, 30, 31) at M=256")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if args.profile_case:
        run_profile_case(args)
        return
    if args.sweep:
        run_sweep(args)
        return
    if args.stack:
        run_stack(args)
        return

    import torch
    import torch.distributed as dist
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))
    torch.cuda.set_device(local)
    from w4_gemm_gated_b200 import spear as S   # raises if the CUDA library is missing
    from w4_gemm_gated_b200 import synth

    dev = torch.device("cuda", local)
    props = torch.cuda.get_device_properties(dev)
    l2 = getattr(props, "L2_cache_size", 126 << 20)

    def bf16(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(dev)

    L = synth.decode(16, force_outlier=True)
    base = S.prepare_layer(torch.from_numpy(L.W).to(dev), 0, bf16(L.A), bf16(L.B), bf16(L.w_g), L.b_g)
    layer_bytes = alg_bytes(0, K_, N_, R_)
    ncopy = max(4, int(np.ceil(2.2 * l2 / layer_bytes)))
    layers = [base] + [S.Layer(K_, N_, 0, R_, base.w_packed.clone(), base.scales.clone(), base.AgT.clone(),
                               base.BpT.clone(), base.b_g) for _ in range(ncopy - 1)]
    xs = {M: bf16(synth.decode(M, force_outlier=True).x) for M in MS}
    ys = {M: torch.empty((M, N_), dtype=torch.bfloat16, device=dev) for M in MS}
    ws = S.make_workspace(base, 16)
    stream = torch.cuda.Stream(device=dev)

    def step(i):
        # every launch reads its own weight copy: the copies rotate per launch,
        # not per step, so no launch finds its weights in L2 unless the call
        # before it warmed them; each call names the next call's layer
        # (prefetch_next), as a decoder's token step would
        for j, M in enumerate(MS):
            c = i * len(MS) + j
            S.forward(layers[c % ncopy], xs[M], ws, y=ys[M], stream=stream, prefetch_next=layers[(c + 1) % ncopy])

    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            step(i)
    stream.synchronize()
    assert S.read_status(ws, stream=stream) == S.OK

    # CUDA graph of a chunk of steps (host launch cost out of the timed region)
    chunk = min(args.steps, 3 * ncopy * 4)
    # the timed graph: a chunk of steps, launches back to back (consecutive
    # launches keep their programmatic, overlapping dependency; event nodes
    # between launches would serialise them and add several microseconds)
    g_plain = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_plain, stream=stream):
        for i in range(chunk):
            step(i)
    rem = args.steps % chunk
    g_rem = None
    if rem:
        g_rem = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_rem, stream=stream):
            for i in range(rem):
                step(i)
    with torch.cuda.stream(stream):
        for _ in range(2):
            g_plain.replay()
    stream.synchronize()

    sampler = ClockSampler(local)
    sampler.start()
    # soak of the same step so the clock record covers a steady state
    t_soak = time.perf_counter()
    while time.perf_counter() - t_soak < 1.5:
        with torch.cuda.stream(stream):
            g_plain.replay()
        stream.synchronize()

    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):       # graphs replay on the current stream
        e0.record(stream)
        for _ in range(args.steps // chunk):
            g_plain.replay()
        if g_rem is not None:
            g_rem.replay()
        e1.record(stream)
    e1.synchronize()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    el_ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    assert S.read_status(ws, stream=stream) == S.OK

    # The timed region holds nothing but decode-kernel launches (3 per step),
    # so its average launch duration is the kernel's: achieved = algorithmic
    # bytes of a step / step time.
    tot_bytes = sum(alg_bytes(M, K_, N_, R_) for M in MS)
    hbm_peak, tc_peak, tc_sust, peak_src = measured_peaks()
    achieved = tot_bytes / (el_ms * 1e-3 / args.steps) / 1e9

    # per-M launch durations (informative): event-free graphs of one M only
    def per_launch_stats(lays, M, reps=12):
        """Back-to-back launches of one M (a graph of 3 x copies launches, hinted):
        the mean launch time of each replay; median, p10 and p90 over replays."""
        n = 3 * ncopy
        gm = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gm, stream=stream):
            for i in range(n):
                S.forward(lays[i % ncopy], xs[M], ws, y=ys[M], stream=stream, prefetch_next=lays[(i + 1) % ncopy])
        vals = []
        with torch.cuda.stream(stream):
            gm.replay()
            for _ in range(reps):
                m0, m1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                m0.record(stream)
                gm.replay()
                m1.record(stream)
                m1.synchronize()
                vals.append(m0.elapsed_time(m1) * 1e3 / n)
        return {"median": float(np.median(vals)), "p10": float(np.percentile(vals, 10)),
                "p90": float(np.percentile(vals, 90))}

    def per_launch_us(lays, M):
        return per_launch_stats(lays, M)["median"]

    launch_stats = {M: per_launch_stats(layers, M) for M in MS}
    mean_us = {M: launch_stats[M]["median"] for M in MS}
    # the pages' per-rank gate gamma(t) (bottleneck h = 16) on the same layers
    rng = np.random.default_rng(7)
    rg = [torch.from_numpy(v.astype(np.float32)).to(dev) for v in
          (rng.standard_normal((16, R_)) / np.sqrt(R_), rng.standard_normal(16) * 0.1,
           rng.standard_normal((R_, 16)) / 4.0, rng.standard_normal(R_) - 0.5)]
    rank_layers = [S.with_rank_gate(lay, *rg, 1.0) for lay in layers]
    rank_us = {M: per_launch_us(rank_layers, M) for M in (1, 16)}
    assert S.read_status(ws, stream=stream) == S.OK

    tokens_per_step = sum(MS)
    value = whole_job_rate(tokens_per_step, args.steps, world, el_ms)

    # ---- end to end through the public API: pinned host x in, host y out ----
    hx = {M: xs[M].cpu().pin_memory() for M in MS}
    hy = {M: torch.empty((M, N_), dtype=torch.bfloat16).pin_memory() for M in MS}
    dx = {M: torch.empty_like(xs[M]) for M in MS}
    e2e_steps = min(args.steps, 500)
    with torch.cuda.stream(stream):
        def e2e_step(i):
            for j, M in enumerate(MS):
                dx[M].copy_(hx[M], non_blocking=True)
                c = i * len(MS) + j
                S.forward(layers[c % ncopy], dx[M], ws, y=ys[M], stream=stream, prefetch_next=layers[(c + 1) % ncopy])
                hy[M].copy_(ys[M], non_blocking=True)
        for i in range(3):
            e2e_step(i)
        stream.synchronize()
        if world > 1:
            dist.barrier()
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        for i in range(e2e_steps):
            e2e_step(i)
        a1.record(stream)
        a1.synchronize()
    e2e_value = whole_job_rate(tokens_per_step, e2e_steps, world, max_over_ranks(a0.elapsed_time(a1), world, dev))

    # ---- EC overhead: same kernel with the EC disabled ----
    plain = [S.Layer(K_, N_, 0, 0, lay.w_packed, lay.scales, None, None, 0.0) for lay in layers]
    noec_us = per_launch_us(plain, 16)
    noec_us_m1 = per_launch_us(plain, 1)

    prefill = None
    if not args.no_prefill and rank == 0:
        prefill = bench_prefill(S, synth, dev, stream, bf16, tc_peak)
    stack = None
    if not args.no_stack and rank == 0:
        try:
            stack = stack_measure(S, synth, 5)
            # device time of the linears: the graph replay (no host dispatch between kernels)
            lt = stack["graph"]["linears_tflops"]
            stack["roofline"] = {"bound": "tensor", "achieved": lt, "peak": tc_sust,
                                 "unit": "TFLOP/s", "frac": lt / tc_sust, "frac_of_burst": lt / tc_peak,
                                 "from": "graph-replayed linears",
                                 "peak_source": f"{peak_src} bf16_tflops_sustained (a long step)"}
        except Exception as e:  # report, do not hide the decode result
            stack = {"error": f"{type(e).__name__}: {e}"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = time_oracle()

    line = {
        "metric": METRIC,
        "value": value,
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": el_ms / args.steps,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16 x int4 -> fp32 accumulate, bf16 out",
        "data": "synthetic",
        "config": {"workload": "decode GEMV K=4096 N=11008 r=64, M in {1,4,16} per step (7B MLP up-projection)",
                   "tokens_per_step": tokens_per_step, "parallelism": f"replicas x{world}",
                   "l2": f"cold: {ncopy} weight copies rotating per launch ({ncopy * layer_bytes / 1e6:.0f} MB > 2x L2)",
                   "timing": f"CUDA-graph replay of {chunk}-step chunks (launches overlap through programmatic "
                             f"dependent launch), events on the launching stream",
                   "prefetch_hint": "each call names the next call's layer (prefetch_next): its kernel warms L2 "
                                    "with that layer's weights; DRAM bytes per step unchanged"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                     "frac": achieved / hbm_peak, "traffic": decode_traffic_per_step(),
                     "traffic_unit": "DRAM bytes per step (3 launches), ncu capture in profiles/",
                     "kernel": "decode_kernel (fused W4 GEMV + gated EC)",
                     "per_launch_us": mean_us,
                     "per_launch_us_p10_p50_p90": {M: [launch_stats[M]["p10"], launch_stats[M]["median"],
                                                       launch_stats[M]["p90"]] for M in MS},
                     "achieved_from": "algorithmic bytes of a step / timed step time (3 decode launches)",
                     "per_launch_timing": "event-free graphs of 3 x copies launches of one M, back to back; "
                                          "p10/p50/p90 over 12 replays of the mean launch time",
                     "algorithmic_bytes": {M: alg_bytes(M, K_, N_, R_) for M in MS},
                     "peak_source": f"{peak_src} hbm_gbs"},
        "ec_overhead": {"m16_with_ec_us": mean_us[16], "m16_ec_disabled_us": noec_us,
                        "overhead": mean_us[16] / noec_us - 1.0,
                        "m1_with_ec_us": mean_us[1], "m1_ec_disabled_us": noec_us_m1,
                        "overhead_m1": mean_us[1] / noec_us_m1 - 1.0},
        "rank_gate": {"per_launch_us": rank_us, "hidden": 16,
                      "vs_scalar_gate": {M: rank_us[M] / mean_us[M] - 1.0 for M in rank_us},
                      "form": "y = xW + alpha (t * sigmoid(W2 relu(W1 t + b1) + b2)) B, t = xA"},
        "e2e": {"value": e2e_value, "unit": "tokens/s",
                "h2d_bytes_per_step": sum(2 * M * K_ for M in MS), "d2h_bytes_per_step": sum(2 * M * N_ for M in MS),
                "steps": e2e_steps, "api": "w4_gemm_gated_b200.spear.forward (eager, pinned host buffers)"},
        "gpu_launches": 3 * args.steps,
        "clocks": clocks,
        "cpu_baseline": cpu,
    }
    if prefill is not None:
        line["prefill"] = prefill
    if stack is not None:
        line["stack"] = stack
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


SWEEP_MS = (1, 8, 32, 128, 512, 2048, 8192)
SWEEP_KN = ((4096, 4096), (4096, 14336), (14336, 4096))
SWEEP_R = (32, 128)


def run_sweep(args):
    """Dispatch sweep: every (K, N, r, scale kind) layer is tuned over the M list
    (spear_dispatch_tune: cold L2, CUDA events, median), then every eligible
    path is re-timed independently and the table's choice is checked against
    the fastest (within 5 %, or 2 us at small sizes)."""
    import torch
    from w4_gemm_gated_b200 import spear as S
    from w4_gemm_gated_b200 import synth

    def bf16(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()

    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()

    def median_us(layer, x, y, ws, path, reps):
        ts = []
        for i in range(reps + 3):
            flush.fill_(i & 0xFF)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            S.forward(layer, x, ws, y=y, path=path, stream=stream)
            b.record(stream)
            b.synchronize()
            if i >= 3:
                ts.append(a.elapsed_time(b) * 1e3)
        return float(np.median(ts))

    names = S.PATH_NAMES
    points, good, failures = [], 0, []
    S.dispatch_clear()
    t_start = time.perf_counter()
    for K, N in SWEEP_KN:
        L = synth.sweep_point(max(SWEEP_MS), K, N, 128)
        W = torch.from_numpy(L.W).cuda()
        x_all = bf16(L.x)
        for r in SWEEP_R:
            A, B, w_g = bf16(L.A[:, :r]), bf16(L.B[:r]), bf16(L.w_g)
            for group in (0, 128):
                layer = S.prepare_layer(W, group, A, B, w_g, L.b_g)
                ws = S.make_workspace(layer, max(SWEEP_MS))
                y_all = torch.empty((max(SWEEP_MS), N), dtype=torch.bfloat16, device="cuda")
                S.dispatch_tune(layer, list(SWEEP_MS), x_all, y_all, ws, flush=flush, reps=10)
                st = S.read_status(ws)
                if st != S.OK:
                    failures.append({"K": K, "N": N, "r": r, "group": group, "stage": "tune", "status": st})
                for M in SWEEP_MS:
                    paths = [S.PATH_FUSED, S.PATH_UNFUSED, S.PATH_SEMIFUSED] + ([S.PATH_DECODE] if M <= 16 else [])
                    x = x_all[:M].contiguous()
                    t = {}
                    for p in paths:
                        t[p] = median_us(layer, x, y_all[:M], ws, p, 10)
                        st = S.read_status(ws)
                        if st != S.OK:
                            failures.append({"K": K, "N": N, "r": r, "group": group, "M": M, "path": names[p],
                                             "status": st})
                    choice = S.dispatch_choice(layer, M)
                    best = min(t.values())
                    ok = t[choice] <= max(1.05 * best, best + 2.0)
                    good += ok
                    fl = 2.0 * M * K * N + 2.0 * M * K * (r + 1) + 2.0 * M * r * N
                    points.append({"M": M, "K": K, "N": N, "r": r, "group": group,
                                   "us": {names[p]: round(v, 2) for p, v in t.items()},
                                   "choice": names[choice], "choice_ok": bool(ok),
                                   "tflops_best": round(fl / (best * 1e-6) / 1e12, 2)})
                del layer, ws, y_all
        del W, x_all
    S.dispatch_clear()
    print(json.dumps({"sweep": "dispatch (M x (K,N) x r x scale kind)", "points": len(points),
                      "dispatcher_within_5pct": good, "seconds": round(time.perf_counter() - t_start, 1),
                      "device_status_failures": failures,
                      "timing": "median of 10 launches, L2 flushed (256 MB write) before each",
                      "table": points}))
    if failures:
        sys.exit(1)


STACK_SHAPES = ((4096, 4096), (4096, 4096), (4096, 4096), (4096, 4096),  # q, k, v, o
                (4096, 11008), (4096, 11008), (11008, 4096))              # gate, up, down
STACK_EC_LAYERS = (0, 1, 30, 31)


def stack_glue(S, layers, x, ws, eps=1e-6, n_layers=32):
    """One pass of the synthetic decoder stack through the W4 (+EC) linears.
    Per layer: h = RMSNorm(x); q, k, v = Wq h, Wk h, Wv h; x = x + Wo v (the
    attention mixing is replaced by v); h2 = RMSNorm(x); x = x + Wd(silu(Wg h2) * Wu h2).
    The glue between linears is plain tensor arithmetic (fp32, bf16 activations)."""
    import torch

    def rms(t):
        tf = t.float()
        return (tf * torch.rsqrt(tf.pow(2).mean(-1, keepdim=True) + eps)).to(torch.bfloat16)

    for l in range(n_layers):
        Lq, Lk, Lv, Lo, Lg, Lu, Ld = layers[l]
        h = rms(x)
        S.forward(Lq, h, ws)
        S.forward(Lk, h, ws)
        v = S.forward(Lv, h, ws)
        x = (x.float() + S.forward(Lo, v, ws).float()).to(torch.bfloat16)
        h2 = rms(x)
        gte = S.forward(Lg, h2, ws).float()
        up = S.forward(Lu, h2, ws).float()
        act = (gte * torch.sigmoid(gte) * up).to(torch.bfloat16)
        x = (x.float() + S.forward(Ld, act, ws).float()).to(torch.bfloat16)
    return x


def run_stack(args):
    from w4_gemm_gated_b200 import spear as S
    from w4_gemm_gated_b200 import synth
    print(json.dumps(stack_measure(S, synth, max(1, min(args.steps, 5)))))


def stack_measure(S, synth, reps):
    """Config 4: 32 decoder layers x 7 per-channel W4 linears, ECs (r=64) on all
    linears of layers 0, 1, 30, 31, M=256 tokens pushed through all 224 linears.
    Weights are drawn on the device (seeded per projection) and quantised and
    packed by the library.  Reports the time of the linears alone and of the
    whole stack with the glue (mean of `reps` passes, with p10/p90)."""
    import torch

    M, R = 256, 64
    dev = torch.device("cuda")
    layers, packed_bytes, ec_params = [], 0, 0
    t0 = time.perf_counter()
    for l in range(32):
        row = []
        for proj, (K, N) in enumerate(STACK_SHAPES):
            g = torch.Generator(device=dev).manual_seed(synth.stack_layer_seed(0, l, proj))
            W = torch.randn((K, N), generator=g, device=dev, dtype=torch.float32) * 0.02
            if l in STACK_EC_LAYERS:
                A = (torch.randn((K, R), generator=g, device=dev) * 0.01).to(torch.bfloat16)
                B = (torch.randn((R, N), generator=g, device=dev) * 0.01).to(torch.bfloat16)
                w_g = (torch.randn(K, generator=g, device=dev) / np.sqrt(K)).to(torch.bfloat16)
                lay = S.prepare_layer(W, 0, A, B, w_g, -1.0)
                ec_params += K * R + R * N + K
            else:
                lay = S.prepare_layer(W, 0, None, None, None, 0.0)
            packed_bytes += K * N // 2
            row.append(lay)
            del W
        layers.append(row)
    prep_s = time.perf_counter() - t0
    # one zeroed workspace large enough for every linear of the stack
    ws = torch.zeros(max(S.workspace_bytes(lay, M) for row in layers for lay in row), dtype=torch.uint8, device=dev)
    x0 = torch.randn((M, 4096), generator=torch.Generator(device=dev).manual_seed(7), device=dev).to(torch.bfloat16)
    stream = torch.cuda.current_stream()

    # the linears alone, inputs prepared once per shape
    xs = {4096: x0, 11008: torch.randn((M, 11008), device=dev).to(torch.bfloat16)}
    for _ in range(2):
        for row in layers:
            for lay in row:
                S.forward(lay, xs[lay.K], ws)
    torch.cuda.synchronize()
    lin = []
    for _ in range(reps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for row in layers:
            for lay in row:
                S.forward(lay, xs[lay.K], ws)
        b.record(stream)
        b.synchronize()
        lin.append(a.elapsed_time(b))
    lin_ms = float(np.mean(lin))

    # the whole stack with the glue
    for _ in range(2):
        out = stack_glue(S, layers, x0, ws)
    torch.cuda.synchronize()
    full = []
    for _ in range(reps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        out = stack_glue(S, layers, x0, ws)
        b.record(stream)
        b.synchronize()
        full.append(a.elapsed_time(b))
    e2e_ms = float(np.mean(full))
    assert S.read_status(ws) == S.OK
    finite = bool(torch.isfinite(out.float()).all().item())

    # the same two measurements replayed from CUDA graphs (one pass captured),
    # as a serving engine runs a step: no host dispatch between the kernels
    def graph_ms(fn):
        side = torch.cuda.Stream()
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            fn()
            side.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=side):
                fn()
            g.replay()
            side.synchronize()
            ts = []
            for _ in range(reps):
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(side)
                g.replay()
                b.record(side)
                b.synchronize()
                ts.append(a.elapsed_time(b))
        stream.wait_stream(side)
        del g
        return ts

    def lin_pass():
        for row in layers:
            for lay in row:
                S.forward(lay, xs[lay.K], ws)

    lin_g = graph_ms(lin_pass)
    full_g = graph_ms(lambda: stack_glue(S, layers, x0, ws))
    assert S.read_status(ws) == S.OK
    lin_g_ms, full_g_ms = float(np.mean(lin_g)), float(np.mean(full_g))
    flops = sum(2.0 * M * K * N for (K, N) in STACK_SHAPES) * 32 + \
        len(STACK_EC_LAYERS) * sum(2.0 * M * K * (R + 1) + 2.0 * M * R * N for (K, N) in STACK_SHAPES)
    del layers, ws
    torch.cuda.empty_cache()
    return {
        "stack": "32 decoder layers x 7 W4 linears, ECs r=64 on layers 0,1,30,31", "M": M,
        "linears_ms": lin_ms, "stack_ms": e2e_ms, "tokens_per_s": M / (e2e_ms * 1e-3),
        "linears_ms_p10_p90": [float(np.percentile(lin, 10)), float(np.percentile(lin, 90))],
        "stack_ms_p10_p90": [float(np.percentile(full, 10)), float(np.percentile(full, 90))],
        "linears_tflops": flops / (lin_ms * 1e-3) / 1e12,
        "graph": {"linears_ms": lin_g_ms, "stack_ms": full_g_ms, "tokens_per_s": M / (full_g_ms * 1e-3),
                  "linears_ms_p10_p90": [float(np.percentile(lin_g, 10)), float(np.percentile(lin_g, 90))],
                  "stack_ms_p10_p90": [float(np.percentile(full_g, 10)), float(np.percentile(full_g, 90))],
                  "linears_tflops": flops / (lin_g_ms * 1e-3) / 1e12,
                  "timing": f"one pass captured in a CUDA graph, mean of {reps} replays"},
        "packed_weight_bytes": packed_bytes, "ec_params": ec_params,
        "ec_params_fraction_of_packed_bytes": ec_params / packed_bytes,
        "ec_bytes_fraction_of_packed_bytes": 2 * ec_params / packed_bytes,
        "output_finite": finite, "prep_seconds": round(prep_s, 1),
        "timing": f"mean of {reps} passes, weights 3.24 GB (no L2 reuse across passes)"}


def run_profile_case(args):
    """A few launches of one kernel for a profiler: the decode kernel on the
    7B up-projection (K=4096, N=11008, r=64) or the tensor-core kernel on the
    o-projection shape (K=N=4096, r=64), at --m tokens."""
    import torch
    from w4_gemm_gated_b200 import spear as S
    from w4_gemm_gated_b200 import synth

    def bf16(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()

    M = args.m
    if args.profile_case == "decode":
        L = synth.decode(16, force_outlier=True)
        x = bf16(L.x[:M])
        path = S.PATH_DECODE
    else:
        L = synth.prefill(M=M)
        x = bf16(L.x)
        path = S.PATH_FUSED
    lay = S.prepare_layer(torch.from_numpy(L.W).cuda(), 0, bf16(L.A), bf16(L.B), bf16(L.w_g), L.b_g)
    ws = S.make_workspace(lay, max(M, 16))
    for _ in range(args.steps):
        S.forward(lay, x, ws, path=path)
    torch.cuda.synchronize()
    st = S.read_status(ws)
    print(json.dumps({"profile_case": args.profile_case, "M": M, "launches": args.steps, "status": st}))
    if st != S.OK:
        sys.exit(1)


def bench_prefill(S, synth, dev, stream, bf16, tc_peak):
    """Prefill GEMM (M=2048, K=N=4096, r=64): fused tensor-core path."""
    import torch
    try:
        L = synth.prefill()
        lay = S.prepare_layer(torch.from_numpy(L.W).to(dev), 0, bf16(L.A), bf16(L.B), bf16(L.w_g), L.b_g)
        plain = S.Layer(4096, 4096, 0, 0, lay.w_packed, lay.scales, None, None, 0.0)
        rng = np.random.default_rng(7)
        rank = S.with_rank_gate(lay, *[torch.from_numpy(v.astype(np.float32)) for v in
                                       (rng.standard_normal((16, 64)) / 8.0, rng.standard_normal(16) * 0.1,
                                        rng.standard_normal((64, 16)) / 4.0, rng.standard_normal(64) - 0.5)], 1.0)
        x = bf16(L.x)
        y = torch.empty((2048, 4096), dtype=torch.bfloat16, device=dev)
        ws = S.make_workspace(lay, 2048)
        flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
        res = {}
        for name, ly, path in (("fused", lay, S.PATH_FUSED), ("unfused", lay, S.PATH_UNFUSED),
                               ("semifused", lay, S.PATH_SEMIFUSED), ("ec_disabled", plain, S.PATH_FUSED),
                               ("fused_rank_gate", rank, S.PATH_FUSED)):
            ts = []
            with torch.cuda.stream(stream):
                for i in range(13):
                    flush.fill_(i)
                    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    a.record(stream)
                    S.forward(ly, x, ws, y=y, path=path, stream=stream)
                    b.record(stream)
                    b.synchronize()
                    if i >= 3:
                        ts.append(a.elapsed_time(b) * 1e3)
            res[name] = float(np.median(ts))
            res[name + "_p10_p90"] = [float(np.percentile(ts, 10)), float(np.percentile(ts, 90))]
        if S.read_status(ws, stream=stream) != S.OK:
            return {"error": "device status not OK"}
        fl = alg_flops(2048, 4096, 4096, 64)
        tf = fl / (res["fused"] * 1e-6) / 1e12
        return {"workload": "prefill GEMM M=2048 K=N=4096 r=64 (attention o-projection)",
                "fused_us": res["fused"], "unfused_us": res["unfused"], "semifused_us": res["semifused"],
                "ec_disabled_us": res["ec_disabled"], "fused_rank_gate_us": res["fused_rank_gate"],
                "tokens_per_s": 2048 / (res["fused"] * 1e-6), "tflops": tf,
                "roofline": {"bound": "tensor", "achieved": tf, "peak": tc_peak, "unit": "TFLOP/s",
                             "frac": tf / tc_peak},
                "ec_overhead": res["fused"] / res["ec_disabled"] - 1.0,
                "fused_us_p10_p90": res["fused_p10_p90"], "ec_disabled_us_p10_p90": res["ec_disabled_p10_p90"],
                "timing": "median of 10 single launches, L2 flushed (256 MB write) before each"}
    except Exception as e:  # report, do not hide the decode result
        return {"error": f"{type(e).__name__}: {e}"}


if __name__ == "__main__":
    main()
