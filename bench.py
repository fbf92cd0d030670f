#!/usr/bin/env python
"""Benchmark of the tensor-parallel MLP pair on B200.

One step = one pass of the whole layer-pair path over one batch of synthetic
tokens, with all tp_degree shards on one GPU: slice every shard of W_up,
b_up and W_down (a1), the colwise FFN-in GEMM with bias + GELU for every shard
(a2, a3), and the rowwise FFN-out GEMM whose accumulator sums every shard's
partial plus the bias once (a4).  These are the five C-ABI calls that the
one-shot ``tp_mlp_pair`` makes, issued one by one so that each kernel's
duration is measured with CUDA events inside the timed region (a GPU test
checks that the sequence is bit-identical to ``tp_mlp_pair``).

Usage:  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
Under torchrun (N > 1) every rank runs the same workload on its own tokens
(independent replicas: the layer pair has no exchange step when all shards of
a layer live on one GPU), so per-GPU work is fixed ("weak" scaling) and the
job value is the sum of all ranks' work over the slowest rank's time.

``--impl reference`` times the fp64 CPU oracle on the same workload (a bounded
sample of token rows per step), on rank 0 only.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "TP layer-pair bf16 TFLOP/s and % of dense-BF16 tensor peak on 1 B200"
UNIT = "TFLOP/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_BYTES = 126 << 20


# --------------------------------------------------------------------------- distributed helpers
def dist_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")),
            int(os.environ.get("WORLD_SIZE", "1")))


def max_over_ranks(x: float) -> float:
    """Max of a per-rank scalar over all ranks (a host-side timing reduction)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    dev = torch.device("cuda", torch.cuda.current_device()) if dist.get_backend() == "nccl" else torch.device("cpu")
    t = torch.tensor([float(x)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier():
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.barrier()


def job_value(flops_per_rank_step: float, n_ranks: int, steps: int, max_seconds: float) -> float:
    """Whole-job TFLOP/s: every rank's work over the slowest rank's time."""
    return flops_per_rank_step * n_ranks * steps / max_seconds / 1e12


# --------------------------------------------------------------------------- peaks, clocks, traffic
def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


REASON_BITS = {
    0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
    0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
    0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
}


class ClockSampler:
    """Samples the SM clock and the clock-event reasons through NVML (the
    library behind nvidia-smi) every `period` seconds while running."""

    def __init__(self, local_index: int, period: float = 0.002):
        self.period = period
        self.samples = []
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None
        self._h = None
        try:
            import pynvml
            pynvml.nvmlInit()
            idx = local_index
            vis = os.environ.get("CUDA_VISIBLE_DEVICES")
            if vis:
                ids = [v.strip() for v in vis.split(",") if v.strip()]
                if local_index < len(ids) and ids[local_index].isdigit():
                    idx = int(ids[local_index])
            self._nvml = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(idx)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:  # noqa: BLE001 - no NVML: report no clocks
            self._h = None

    def _reasons(self):
        n = self._nvml
        for name in ("nvmlDeviceGetCurrentClocksEventReasons", "nvmlDeviceGetCurrentClocksThrottleReasons"):
            f = getattr(n, name, None)
            if f is not None:
                return f(self._h)
        return 0

    def _run(self):
        n = self._nvml
        while not self._stop.is_set():
            try:
                self.samples.append((n.nvmlDeviceGetClockInfo(self._h, n.NVML_CLOCK_SM), int(self._reasons())))
            except Exception:  # noqa: BLE001
                pass
            time.sleep(self.period)

    def start(self):
        if self._h is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()

    def stop(self) -> dict:
        if self._thread is not None:
            self._stop.set()
            self._thread.join()
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        mhz = [s[0] for s in self.samples]
        bits = 0
        for _, r in self.samples:
            bits |= r
        reasons = [name for b, name in REASON_BITS.items() if bits & b and name != "gpu_idle"]
        return {"sm_mhz": statistics.median(mhz), "sm_max_mhz": self.max_mhz, "reasons": reasons,
                "samples": len(mhz)}


def source_sha(*names) -> str:
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(ROOT, "tensor_transformer_layers_b200", "csrc", n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    the current kernel source (else None)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(f"{kernel}@{workload}")
    if not e or e.get("source_sha") != source_sha(*e.get("sources", [])):
        return None
    return e.get("dram_bytes_per_launch")


# --------------------------------------------------------------------------- workload
def workload_cfg():
    import synthetic as syn
    return syn.CONFIGS["flux_mlp"]


def make_inputs(cfg, rank: int):
    import synthetic as syn
    M, D, F = cfg["M"], cfg["D"], cfg["F"]
    d = syn.mlp_inputs(M, D, F, cfg["seed"])
    if rank:
        # every replica gets its own tokens; the weights are the layer's
        d["X"] = syn.normal_bf16((M, D), 1.0, seed=cfg["seed"] + 1000 * rank, tid=syn.TID["X"])
    return d


def flops_mlp(M, D, F):
    return 4.0 * M * D * F


# --------------------------------------------------------------------------- CPU oracle legs
def oracle_rows_run(d, rows: int, T: int):
    import oracle as o
    import synthetic as syn
    f = {k: syn.bf16_bits_to_f64(v) for k, v in d.items() if k != "X"}
    X = syn.bf16_bits_to_f64(d["X"][:rows])
    t0 = time.perf_counter()
    o.mlp_sharded_summed(X, f["W_up"], f["b_up"], f["W_down"], f["b_down"], T)
    return time.perf_counter() - t0


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads") for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:  # noqa: BLE001
        pass
    return os.cpu_count() or 1


def cpu_baseline(d, cfg, budget_s: float = 12.0):
    """The oracle as it stands, on a bounded sample of the workload's token rows."""
    M, D, F, T = cfg["M"], cfg["D"], cfg["F"], cfg["T"]
    probe = 64
    oracle_rows_run(d, probe, T)  # warm
    t = oracle_rows_run(d, probe, T)
    rows = int(min(M, max(probe, probe * budget_s / max(t, 1e-6))))
    t = oracle_rows_run(d, rows, T)
    return {"value": flops_mlp(rows, D, F) / t / 1e12, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
            "sample": f"{rows} of {M} token rows of the workload through the fp64 oracle "
                      f"(mlp_sharded_summed, tp_degree {T}), {t:.1f} s"}


def run_reference(args, cfg, rank, world):
    if rank != 0:
        return None  # rank 0 alone runs the CPU reference
    d = make_inputs(cfg, 0)
    M, D, F, T = cfg["M"], cfg["D"], cfg["F"], cfg["T"]
    probe = 32
    oracle_rows_run(d, probe, T)
    t = oracle_rows_run(d, probe, T)
    per_step = max(0.2, min(5.0, 120.0 / max(1, args.steps + args.warmup)))
    rows = int(min(M, max(8, probe * per_step / max(t, 1e-6))))
    for _ in range(args.warmup):
        oracle_rows_run(d, rows, T)
    times = [oracle_rows_run(d, rows, T) for _ in range(args.steps)]
    total = sum(times)
    value = flops_mlp(rows, D, F) * args.steps / total / 1e12
    sample = (f"{rows} of {M} token rows per step through the fp64 oracle (mlp_sharded_summed, "
              f"tp_degree {T}) on host cores")
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": config_dict(cfg, world),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": blas_threads(), "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def config_dict(cfg, world):
    return {"workload": (f"flux_mlp: TP MLP pair (colwise FFN-in + GELU(tanh), rowwise FFN-out with the "
                         f"cross-shard sum fused), all tp_degree shards on one GPU; M={cfg['M']} tokens "
                         f"(4096 image + 512 text), D={cfg['D']}, F={cfg['F']}"),
            "M": cfg["M"], "D": cfg["D"], "F": cfg["F"], "tp_degree": cfg["T"], "global_batch_tokens": cfg["M"] * world,
            "l2": ("not flushed: inputs larger than L2 (each step reads 179 MB of inputs, > 126 MB L2, "
                   "and moves about 0.6 GB in total)"),
            "parallelism": "single GPU" if world == 1 else f"{world} independent replicas (one per GPU)"}


# --------------------------------------------------------------------------- GPU leg
def run_ours(args, cfg, rank, local_rank, world):
    import numpy as np
    import torch

    import tensor_transformer_layers_b200 as tp

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    M, D, F, T = cfg["M"], cfg["D"], cfg["F"], cfg["T"]
    Fs = F // T
    d = make_inputs(cfg, rank)
    host = {k: torch.from_numpy(np.ascontiguousarray(v).view(np.int16)).pin_memory() for k, v in d.items()}
    g = {k: v.to(dev) for k, v in host.items()}
    w_up = torch.empty((T, Fs, D), dtype=torch.int16, device=dev)
    b_up = torch.empty((T, Fs), dtype=torch.int16, device=dev)
    w_down = torch.empty((T, D, Fs), dtype=torch.int16, device=dev)
    H = torch.empty((T, M, Fs), dtype=torch.int16, device=dev)
    Y = torch.empty((M, D), dtype=torch.int16, device=dev)
    input_bytes = sum(v.numel() * v.element_size() for v in g.values())
    assert input_bytes > L2_BYTES, "the step's inputs must exceed L2 (no flush between steps)"
    check = tp._check

    names = ["slice_w_up", "slice_b_up", "slice_w_down", "colwise_gemm", "rowwise_gemm"]

    def step(ev):
        ev[0].record()
        check(tp.tp_shard_weight_all(g["W_up"], F, D, tp.TP_COLWISE, T, w_up), "slice W_up")
        ev[1].record()
        check(tp.tp_shard_weight_all(g["b_up"], T, Fs, tp.TP_COLWISE, T, b_up), "slice b_up")
        ev[2].record()
        check(tp.tp_shard_weight_all(g["W_down"], D, F, tp.TP_ROWWISE, T, w_down), "slice W_down")
        ev[3].record()
        check(tp.tp_colwise_linear(g["X"], M, D, w_up, b_up, Fs, T, 1, tp.TP_OUT_BF16, H), "colwise")
        ev[4].record()
        check(tp.tp_rowwise_linear_sum(H, M, Fs, w_down, D, g["b_down"], T, Y), "rowwise")
        ev[5].record()

    def new_events():
        return [torch.cuda.Event(enable_timing=True) for _ in range(6)]

    for _ in range(args.warmup):
        step(new_events())
    torch.cuda.synchronize()

    sampler = ClockSampler(local_rank)
    evs = [new_events() for _ in range(args.steps)]
    barrier()
    torch.cuda.synchronize()
    launches0 = tp.tp_kernel_launches()
    sampler.start()
    t_wall0 = time.perf_counter()
    for i in range(args.steps):
        step(evs[i])
    torch.cuda.synchronize()
    t_wall = time.perf_counter() - t_wall0
    clocks = sampler.stop()
    launches = tp.tp_kernel_launches() - launches0
    barrier()
    assert tp.tp_check_device_error() == 0

    per_kernel = {n: [] for n in names}
    step_ms = []
    for ev in evs:
        for j, n in enumerate(names):
            per_kernel[n].append(ev[j].elapsed_time(ev[j + 1]))
        step_ms.append(ev[0].elapsed_time(ev[5]))
    local_s = sum(step_ms) / 1e3
    max_s = max_over_ranks(local_s)
    flops = flops_mlp(M, D, F)
    value = job_value(flops, world, args.steps, max_s)

    peaks, peak_src = load_peaks()
    tc_peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    hbm_peak = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    kinfo = {}
    algo = {
        "slice_w_up": ("GB/s", 2.0 * F * D * 2),
        "slice_b_up": ("GB/s", 2.0 * F * 2),
        "slice_w_down": ("GB/s", 2.0 * D * F * 2),
        "colwise_gemm": ("TFLOP/s", 2.0 * M * D * F),
        "rowwise_gemm": ("TFLOP/s", 2.0 * M * F * D),
    }
    tot = sum(statistics.mean(v) for v in per_kernel.values())
    for n in names:
        ms = statistics.mean(per_kernel[n])
        unit, work = algo[n]
        ach = work / (ms / 1e3) / (1e12 if unit == "TFLOP/s" else 1e9)
        pk = tc_peak if unit == "TFLOP/s" else hbm_peak
        kinfo[n] = {"ms": round(ms, 5), "share": round(ms / tot, 4), "achieved": round(ach, 1), "unit": unit,
                    "frac": round(ach / pk, 4)}
    dom = max(("colwise_gemm", "rowwise_gemm"), key=lambda n: kinfo[n]["ms"])
    roofline = {"kernel": dom, "bound": "tensor", "achieved": kinfo[dom]["achieved"], "peak": tc_peak,
                "unit": "TFLOP/s", "frac": kinfo[dom]["frac"],
                "traffic": recorded_traffic(dom, "flux_mlp"),
                "peak_source": f"{peak_src} (bf16 burst; {'MEASURED_PEAKS.json' if peak_src == 'measured' else 'recipe fallback'})",
                "algorithmic_flops_per_launch": algo[dom][1]}

    # ---- end to end: the one-shot public call with host buffers copied in and the result copied out.
    ws = torch.empty(tp.tp_mlp_workspace_bytes(M, D, F, T), dtype=torch.uint8, device=dev)
    y_host = torch.empty((M, D), dtype=torch.int16).pin_memory()
    gi = {k: torch.empty_like(v, device=dev) for k, v in host.items()}
    h2d = sum(v.numel() * v.element_size() for v in host.values())
    d2h = y_host.numel() * 2

    def e2e_step():
        for k in host:
            gi[k].copy_(host[k], non_blocking=True)
        check(tp.tp_mlp_pair(gi["X"], M, D, F, gi["W_up"], gi["b_up"], gi["W_down"], gi["b_down"], T, Y, ws,
                             ws.numel()), "tp_mlp_pair")
        y_host.copy_(Y, non_blocking=True)

    for _ in range(max(1, args.warmup)):
        e2e_step()
    torch.cuda.synchronize()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n_e2e = args.steps
    e0.record()
    for _ in range(n_e2e):
        e2e_step()
    e1.record()
    torch.cuda.synchronize()
    e2e_s = max_over_ranks(e0.elapsed_time(e1) / 1e3)
    barrier()
    e2e = {"value": job_value(flops, world, n_e2e, e2e_s), "unit": UNIT, "h2d_bytes_per_step": h2d,
           "d2h_bytes_per_step": d2h,
           "call": "tp_mlp_pair with X, W_up, b_up, W_down, b_down copied from pinned host memory and Y copied back"}

    out = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1e3 * max_s / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded)",
        "config": config_dict(cfg, world),
        "frac_of_nominal_dense_bf16": round(value / world / 2250.0, 4),
        "frac_of_measured_bf16": round(value / world / tc_peak, 4),
        "roofline": roofline, "kernels": kinfo, "clocks": clocks, "e2e": e2e,
        "gpu_launches": int(launches), "wall_s_timed_region": round(t_wall, 4),
        "cpu_baseline": None,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(d, cfg)
    return out


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true",
                    help="leave out the CPU oracle leg (cpu_baseline is then null)")
    args = ap.parse_args(argv)
    rank, local_rank, world = dist_env()
    cfg = workload_cfg()

    if world > 1 and args.impl == "ours":
        import datetime

        import torch
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local_rank)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    try:
        if args.impl == "reference":
            out = run_reference(args, cfg, rank, world)
        else:
            out = run_ours(args, cfg, rank, local_rank, world)
        if rank == 0 and out is not None:
            print(json.dumps(out), flush=True)
    finally:
        if world > 1 and args.impl == "ours":
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
