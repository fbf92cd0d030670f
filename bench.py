#!/usr/bin/env python
"""Benchmark of the tensor-parallel MLP pair on B200.

One step = one pass of the layer-pair path over one batch of synthetic
tokens, with all tp_degree shards on one GPU and the shards prepared at load
time (each rank slices its weights once when the model is loaded, then runs
the layer every step): the colwise FFN-in GEMM with bias + GELU for every
shard (a2, a3) and the rowwise FFN-out GEMM whose accumulator sums every
shard's partial plus the bias once (a4) -- the two launches ``tp_mlp_run``
makes on a prepared handle.  The load-time slicing of W_up, b_up and W_down
(a1, one launch) runs in the same timed loop, between steps, and is reported
as its own kernel entry; ``one_shot_value`` counts it too, as the one-shot
``tp_mlp_pair`` (slice + both GEMMs every call) would.  Each kernel is timed
with CUDA events inside the timed region (GPU tests check that these
step-level calls are bit-identical to ``tp_mlp_run`` and ``tp_mlp_pair``).

Usage:  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                       [--workload flux_mlp|flux_mlp_sweep|flux_attn|wide_block|flux_reduce|flux_swiglu|
                                   flux_split_input|flux_joint_attn|flux_ring_attn|flux_ulysses_attn]
                       [--mode replicas|tp] [--no-cpu-baseline] [--headline-only] [--context-torch]
The default workload (flux_mlp) is the headline line.  The others time the
remaining rows the same way: flux_mlp_sweep (the same pair at tp_degree 1, 2,
4 and 8, one kernel set per degree), flux_attn (QKV head split, QKV GEMM, SDPA,
out-projection), wide_block (attention then MLP pair at tp_degree 8, every
row), flux_reduce (the standalone partial-sum reduction, GB/s), flux_swiglu
(the SwiGLU pair: packed gate/up slicing, SwiGLU colwise GEMM, rowwise GEMM)
flux_split_input (rowwise_split_input on an FFN-out-sized projection) and
flux_joint_attn (dual-stream joint attention, 4096 image + 512 text tokens),
flux_ring_attn / flux_ulysses_attn (context-parallel attention, ranks emulated
on one GPU).  A default one-GPU run also times every other workload after
the headline measurement, with short loops, and adds them to the same line
as ``other_configs`` (``--headline-only`` leaves them out).
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


def has_context_row(wl) -> bool:
    """Whether the workload's line carries the torch / cuBLAS context row: the headline MLP pair only (the
    other workloads subclass it but are other layers)."""
    return type(wl).__name__ == "MlpWorkload"


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


# --------------------------------------------------------------------------- workloads
def oracle_threads():
    """Host threads the C++ oracle computes with (OpenMP; all cores by default)."""
    import oracle as o
    return o.num_threads()


def _f64(d, keys):
    import synthetic as syn
    return {k: syn.bf16_bits_to_f64(d[k]) for k in keys}


class Kernel:
    """One timed entry in a step: a name, its unit (TFLOP/s or GB/s), its
    algorithmic work per step, and the C-ABI calls that make it.

    ``exchange`` marks a stand-in for a collective that several GPUs would run
    (device copies emulating an all-to-all between ranks that share one GPU):
    timed and reported, but not counted in ``value``.

    ``load`` marks load-time work (shard slicing): in the pages' design each
    rank slices its weights once, when the model is loaded, and then runs the
    layer every step.  Load-time kernels run in the same timed loop and get
    their own entry in the JSON line, but the headline ``value`` counts only the
    per-step kernels (the prepared layer); ``one_shot_value`` counts both, as a
    one-shot call that slices every time would.

    ``composite`` marks one call of the prepared layer that launches several
    kernels (and may run some side by side); ``breakdown`` marks the step-level
    calls that time the same kernels one at a time in the same loop.  The step
    is then the composite call; breakdown entries are reported (and the
    dominant kernel's roofline is taken among them) but not counted in
    ``value``."""

    def __init__(self, name, unit, work, fn, load=False, group=None, exchange=False, breakdown=False,
                 composite=False):
        self.name, self.unit, self.work, self.fn = name, unit, float(work), fn
        self.load, self.group, self.exchange = load, group, exchange
        self.breakdown, self.composite = breakdown, composite


class MlpWorkload:
    """flux_mlp (the default line): the MLP pair, a1..a4."""
    key = "flux_mlp"
    metric = METRIC
    unit = UNIT

    def __init__(self, cfg=None):
        import synthetic as syn
        self.cfg = cfg or syn.CONFIGS["flux_mlp"]

    def host_inputs(self, rank):
        import synthetic as syn
        c = self.cfg
        d = syn.mlp_inputs(c["M"], c["D"], c["F"], c["seed"])
        if rank:  # every replica gets its own tokens; the weights are the layer's
            d["X"] = syn.normal_bf16((c["M"], c["D"]), 1.0, seed=c["seed"] + 1000 * rank, tid=syn.TID["X"])
        return d

    def work(self):
        c = self.cfg
        return 4.0 * c["M"] * c["D"] * c["F"]

    def kernels(self, tp, g, dev):
        import torch
        M, D, F, T = self.cfg["M"], self.cfg["D"], self.cfg["F"], self.cfg["T"]
        Fs = F // T
        b = {"w_up": torch.empty((T, Fs, D), dtype=torch.int16, device=dev),
             "b_up": torch.empty((T, Fs), dtype=torch.int16, device=dev),
             "w_down": torch.empty((T, D, Fs), dtype=torch.int16, device=dev),
             "H": torch.empty((T, M, Fs), dtype=torch.int16, device=dev),
             "Y": torch.empty((M, D), dtype=torch.int16, device=dev)}
        ck = tp._check
        self.bufs = b
        jobs = [(g["W_up"], F, D, tp.TP_COLWISE, b["w_up"]), (g["W_down"], D, F, tp.TP_ROWWISE, b["w_down"]),
                (g["b_up"], T, Fs, tp.TP_COLWISE, b["b_up"])]
        return [
            Kernel("slice_weights", "GB/s", 2.0 * (F * D + D * F + F) * 2,
                   lambda: ck(tp.tp_shard_weights_batch(jobs, T), "slice W_up, W_down, b_up"), load=True),
            Kernel("colwise_gemm", "TFLOP/s", 2.0 * M * D * F,
                   lambda: ck(tp.tp_colwise_linear(g["X"], M, D, b["w_up"], b["b_up"], Fs, T, 1, tp.TP_OUT_BF16,
                                                   b["H"]), "colwise")),
            Kernel("rowwise_gemm", "TFLOP/s", 2.0 * M * F * D,
                   lambda: ck(tp.tp_rowwise_linear_sum(b["H"], M, Fs, b["w_down"], D, g["b_down"], T, b["Y"]),
                              "rowwise")),
        ]

    def context(self, g, dev):
        """The same pair through torch (cuBLAS GEMMs with the bias in their epilogue, GELU as its own
        kernel): a timed context row only, outside the library and the value."""
        import torch
        import torch.nn.functional as tF
        M, D, F = self.cfg["M"], self.cfg["D"], self.cfg["F"]
        X, Wu, bu = g["X"].view(torch.bfloat16), g["W_up"].view(torch.bfloat16), g["b_up"].view(torch.bfloat16)
        Wd, bd = g["W_down"].view(torch.bfloat16), g["b_down"].view(torch.bfloat16)
        c = {"P": torch.empty((M, F), dtype=torch.bfloat16, device=dev),
             "H": torch.empty((M, F), dtype=torch.bfloat16, device=dev),
             "Y": torch.empty((M, D), dtype=torch.bfloat16, device=dev)}
        return [("cublas_up_gemm_bias", "TFLOP/s", 2.0 * M * D * F, lambda: torch.addmm(bu, X, Wu.t(), out=c["P"])),
                ("torch_gelu_tanh", "GB/s", 2.0 * M * F * 2,
                 lambda: c["H"].copy_(tF.gelu(c["P"], approximate="tanh"))),
                ("cublas_down_gemm_bias", "TFLOP/s", 2.0 * M * F * D,
                 lambda: torch.addmm(bd, c["H"], Wd.t(), out=c["Y"]))]

    def one_shot(self, tp, gi, dev):
        """The public one-shot call on device inputs `gi`; returns the output tensor."""
        import torch
        M, D, F, T = self.cfg["M"], self.cfg["D"], self.cfg["F"], self.cfg["T"]
        if not hasattr(self, "_ws"):
            self._ws = torch.empty(tp.tp_mlp_workspace_bytes(M, D, F, T), dtype=torch.uint8, device=dev)
            self._y = torch.empty((M, D), dtype=torch.int16, device=dev)
        tp._check(tp.tp_mlp_pair(gi["X"], M, D, F, gi["W_up"], gi["b_up"], gi["W_down"], gi["b_down"], T, self._y,
                                 self._ws, self._ws.numel()), "tp_mlp_pair")
        return self._y

    e2e_call = "tp_mlp_pair with X, W_up, b_up, W_down, b_down copied from pinned host memory and Y copied back"

    def prepared(self, tp, g, dev):
        """The prepared layer a serving loop runs: the shards made once (tp_mlp_prepare), each step's input
        is the tokens X only.  Returns (per-step input keys, step function, description)."""
        import torch
        c = self.cfg
        self._pair = tp.MlpPair(g["W_up"], g["b_up"], g["W_down"], g["b_down"], c["T"])
        self._yp = [torch.empty((c["M"], c["D"]), dtype=torch.int16, device=dev) for _ in range(2)]
        return ["X"], lambda gi, b: self._pair(gi["X"], Y=self._yp[b]), (
            "MlpPair: tp_mlp_prepare once, tp_mlp_run every step with X copied from pinned host memory and Y "
            "copied back")

    def oracle_run(self, d, rows):
        """Runs the oracle on the first `rows` tokens; returns (seconds, algorithmic work done)."""
        import oracle as o
        import synthetic as syn
        c = self.cfg
        f = _f64(d, ["W_up", "b_up", "W_down", "b_down"])
        X = syn.bf16_bits_to_f64(d["X"][:rows])
        t0 = time.perf_counter()
        o.mlp_sharded_summed(X, f["W_up"], f["b_up"], f["W_down"], f["b_down"], c["T"])
        return time.perf_counter() - t0, 4.0 * rows * c["D"] * c["F"]

    oracle_fn = "mlp_sharded_summed"

    def config(self, world):
        c = self.cfg
        return {"workload": (f"flux_mlp: TP MLP pair (colwise FFN-in + GELU(tanh), rowwise FFN-out with the "
                             f"cross-shard sum fused), all tp_degree shards on one GPU; M={c['M']} tokens "
                             f"(4096 image + 512 text), D={c['D']}, F={c['F']}"),
                "M": c["M"], "D": c["D"], "F": c["F"], "tp_degree": c["T"],
                "global_batch_tokens": c["M"] * world}


def _no_prepared_form(self, tp, g, dev):
    """Workloads whose public call has no load-once form: end to end is the one-shot call."""
    return None


class SweepWorkload(MlpWorkload):
    """flux_mlp_sweep: the flux_mlp pair at every tp_degree in {1, 2, 4, 8} with
    the same seeded weights and tokens, one kernel set per degree in each step
    (so the degrees share the box, the clocks and the timed region)."""
    key = "flux_mlp_sweep"
    metric = "TP MLP-pair bf16 TFLOP/s per tp_degree on 1 B200"

    def __init__(self, cfg=None):
        import synthetic as syn
        self.cfg = dict(cfg or syn.CONFIGS["flux_mlp_sweep"])
        self.degrees = tuple(self.cfg["T"])

    def work(self):
        c = self.cfg
        return 4.0 * c["M"] * c["D"] * c["F"] * len(self.degrees)

    def kernels(self, tp, g, dev):
        ks, self.bufs = [], {}
        for T in self.degrees:
            sub = MlpWorkload(dict(self.cfg, T=T))
            ks += [Kernel(f"T{T}_{k.name}", k.unit, k.work, k.fn, k.load, group=T) for k in sub.kernels(tp, g, dev)]
            self.bufs.update({f"T{T}_{n}": b for n, b in sub.bufs.items()})
        return ks

    def one_shot(self, tp, gi, dev):
        """The public one-shot call at every degree in turn; returns the last output."""
        import torch
        M, D, F = self.cfg["M"], self.cfg["D"], self.cfg["F"]
        if not hasattr(self, "_ws"):
            self._ws = torch.empty(max(tp.tp_mlp_workspace_bytes(M, D, F, T) for T in self.degrees),
                                   dtype=torch.uint8, device=dev)
            self._y = torch.empty((M, D), dtype=torch.int16, device=dev)
        for T in self.degrees:
            tp._check(tp.tp_mlp_pair(gi["X"], M, D, F, gi["W_up"], gi["b_up"], gi["W_down"], gi["b_down"], T,
                                     self._y, self._ws, self._ws.numel()), f"tp_mlp_pair T={T}")
        return self._y

    e2e_call = ("tp_mlp_pair at tp_degree 1, 2, 4 and 8 in turn, X and the weights copied from pinned host memory "
                "once per step and the last Y copied back")

    def prepared(self, tp, g, dev):
        import torch
        c = self.cfg
        self._pairs = [tp.MlpPair(g["W_up"], g["b_up"], g["W_down"], g["b_down"], T) for T in self.degrees]
        self._yp = [[torch.empty((c["M"], c["D"]), dtype=torch.int16, device=dev) for _ in self.degrees]
                    for _ in range(2)]
        return ["X"], lambda gi, b: tuple(p(gi["X"], Y=y) for p, y in zip(self._pairs, self._yp[b])), (
            "MlpPair at tp_degree 1, 2, 4 and 8 (prepared once), each run every step on X copied from pinned host "
            "memory, all four Y copied back")

    def oracle_run(self, d, rows):
        import oracle as o
        import synthetic as syn
        c = self.cfg
        f = _f64(d, ["W_up", "b_up", "W_down", "b_down"])
        X = syn.bf16_bits_to_f64(d["X"][:rows])
        t0 = time.perf_counter()
        for T in self.degrees:
            o.mlp_sharded_summed(X, f["W_up"], f["b_up"], f["W_down"], f["b_down"], T)
        return time.perf_counter() - t0, 4.0 * rows * c["D"] * c["F"] * len(self.degrees)

    oracle_fn = "mlp_sharded_summed at every degree"

    def config(self, world):
        c = self.cfg
        return {"workload": (f"flux_mlp_sweep: the flux_mlp TP MLP pair at tp_degree {list(self.degrees)}, same "
                             f"seeded weights and tokens for every degree; M={c['M']}, D={c['D']}, F={c['F']}"),
                "M": c["M"], "D": c["D"], "F": c["F"], "tp_degree": list(self.degrees),
                "global_batch_tokens": c["M"] * world}


class AttnWorkload(MlpWorkload):
    """flux_attn: the attention block, a1 (QKV head split, W_o rowwise) and a5..a7."""
    key = "flux_attn"
    metric = "TP attention-block TFLOP/s (QKV fp16, bf16 weights) on 1 B200"

    def __init__(self, cfg=None):
        import synthetic as syn
        self.cfg = cfg or syn.CONFIGS["flux_attn"]

    def host_inputs(self, rank):
        import synthetic as syn
        c = self.cfg
        d = syn.attn_inputs(c["M"], c["D"], c["seed"])
        if rank:
            d["X"] = syn.normal_bf16((c["M"], c["D"]), 1.0, seed=c["seed"] + 1000 * rank, tid=syn.TID["X"])
        return d

    def work(self):
        M, D = self.cfg["M"], self.cfg["D"]
        return 2.0 * M * D * 3 * D + 4.0 * M * M * D + 2.0 * M * D * D

    def attn_kernels(self, tp, g, dev, X, M, D, H, T, prefix=""):
        import torch
        Ds = D // T
        b = {"w_qkv": torch.empty((T, 3 * Ds, D), dtype=torch.int16, device=dev),
             "w_o": torch.empty((T, D, Ds), dtype=torch.int16, device=dev),
             "QKV": torch.empty((T, M, 3 * Ds), dtype=torch.int16, device=dev),
             "O": torch.empty((T, M, Ds), dtype=torch.int16, device=dev),
             "A": torch.empty((M, D), dtype=torch.int16, device=dev)}
        ck = tp._check

        # the head split of W_qkv is packed colwise with blocks [1, 1, 1]; with W_o: one launch
        jobs = [(g["W_qkv"], 3 * D, D, tp.TP_COLWISE, b["w_qkv"], [1, 1, 1]),
                (g["W_o"], D, D, tp.TP_ROWWISE, b["w_o"])]
        ks = [
            Kernel(prefix + "slice_weights", "GB/s", 2.0 * 4 * D * D * 2,
                   lambda: ck(tp.tp_shard_weights_batch(jobs, T), "slice W_qkv, W_o"), load=True),
            Kernel(prefix + "qkv_gemm", "TFLOP/s", 2.0 * M * D * 3 * D,
                   lambda: ck(tp.tp_colwise_linear(X, M, D, b["w_qkv"], None, 3 * Ds, T, 0, tp.TP_OUT_F16,
                                                   b["QKV"]), "qkv")),
            Kernel(prefix + "sdpa", "TFLOP/s", 4.0 * M * M * D,
                   lambda: ck(tp.tp_sdpa_shards(b["QKV"], M, H, T, b["O"]), "sdpa")),
            Kernel(prefix + "out_gemm", "TFLOP/s", 2.0 * M * D * D,
                   lambda: ck(tp.tp_rowwise_linear_sum(b["O"], M, Ds, b["w_o"], D, None, T, b["A"]), "out")),
        ]
        return ks, b

    def kernels(self, tp, g, dev):
        c = self.cfg
        ks, self.bufs = self.attn_kernels(tp, g, dev, g["X"], c["M"], c["D"], c["H"], c["T"])
        return ks

    def one_shot(self, tp, gi, dev):
        import torch
        c = self.cfg
        M, D, H, T = c["M"], c["D"], c["H"], c["T"]
        if not hasattr(self, "_ws"):
            self._ws = torch.empty(tp.tp_attn_workspace_bytes(M, D, H, T), dtype=torch.uint8, device=dev)
            self._y = torch.empty((M, D), dtype=torch.int16, device=dev)
        tp._check(tp.tp_attn_block(gi["X"], M, D, gi["W_qkv"], gi["W_o"], H, T, self._y, self._ws,
                                   self._ws.numel()), "tp_attn_block")
        return self._y

    e2e_call = "tp_attn_block with X, W_qkv, W_o copied from pinned host memory and Y copied back"

    def prepared(self, tp, g, dev):
        import torch
        c = self.cfg
        self._blk = tp.AttnBlock(g["W_qkv"], g["W_o"], c["H"], c["T"])
        self._yp = [torch.empty((c["M"], c["D"]), dtype=torch.int16, device=dev) for _ in range(2)]
        return ["X"], lambda gi, b: self._blk(gi["X"], Y=self._yp[b]), (
            "AttnBlock: tp_attn_prepare once, tp_attn_run every step with X copied from pinned host memory and Y "
            "copied back")

    def oracle_run(self, d, rows):
        import oracle as o
        c = self.cfg
        M, D, H, T = c["M"], c["D"], c["H"], c["T"]
        f = _f64(d, ["X", "W_qkv", "W_o"])
        t0 = time.perf_counter()
        o.attn_rows(f["X"], f["W_qkv"], f["W_o"], H, list(range(rows)), tp_degree=T)
        # work actually done: K and V for every token, Q / attention / out-projection for `rows` tokens
        done = 2.0 * M * D * 2 * D + 2.0 * rows * D * D + 4.0 * rows * M * D + 2.0 * rows * D * D
        return time.perf_counter() - t0, done

    oracle_fn = "attn_rows"

    def config(self, world):
        c = self.cfg
        return {"workload": (f"flux_attn: TP attention block (head-split QKV colwise, per-shard SDPA, rowwise "
                             f"out-projection with the cross-shard sum fused); M={c['M']}, D={c['D']}, "
                             f"{c['H']} heads x 128"),
                "M": c["M"], "D": c["D"], "heads": c["H"], "tp_degree": c["T"],
                "global_batch_tokens": c["M"] * world}


class JointAttnWorkload(AttnWorkload):
    """flux_joint_attn: dual-stream joint attention (both streams' weights
    sliced in one launch, head-split QKV per stream, one SDPA over
    4096 + 512 tokens, per-stream rowwise out-projections)."""
    key = "flux_joint_attn"
    metric = "TP dual-stream joint-attention TFLOP/s (QKV fp16, bf16 weights) on 1 B200"

    def __init__(self, cfg=None):
        import synthetic as syn
        self.cfg = dict(cfg or syn.CONFIGS["flux_joint_attn"])
        self.cfg["M"] = self.cfg["M_img"] + self.cfg["M_txt"]  # joint tokens (the oracle legs sample these)

    def host_inputs(self, rank):
        import synthetic as syn
        c = self.cfg
        d = syn.joint_attn_inputs(c["M_img"], c["M_txt"], c["D"], c["seed"])
        if rank:
            d["X_img"] = syn.normal_bf16((c["M_img"], c["D"]), 1.0, c["seed"] + 1000 * rank, syn.TID["X"])
            d["X_txt"] = syn.normal_bf16((c["M_txt"], c["D"]), 1.0, c["seed"] + 1000 * rank, syn.TID["X_txt"])
        return d

    def work(self):
        Mi, Mt, D = self.cfg["M_img"], self.cfg["M_txt"], self.cfg["D"]
        M = Mi + Mt
        return 2.0 * M * D * 3 * D + 4.0 * M * M * D + 2.0 * M * D * D

    def kernels(self, tp, g, dev):
        import torch
        c = self.cfg
        Mi, Mt, D, H, T = c["M_img"], c["M_txt"], c["D"], c["H"], c["T"]
        M, Ds = Mi + Mt, D // T
        b = {"wq_img": torch.empty((T, 3 * Ds, D), dtype=torch.int16, device=dev),
             "wq_txt": torch.empty((T, 3 * Ds, D), dtype=torch.int16, device=dev),
             "wo_img": torch.empty((T, D, Ds), dtype=torch.int16, device=dev),
             "wo_txt": torch.empty((T, D, Ds), dtype=torch.int16, device=dev),
             "QKV": torch.empty((T, M, 3 * Ds), dtype=torch.int16, device=dev),
             "O": torch.empty((T, M, Ds), dtype=torch.int16, device=dev),
             "Y_img": torch.empty((Mi, D), dtype=torch.int16, device=dev),
             "Y_txt": torch.empty((Mt, D), dtype=torch.int16, device=dev)}
        self.bufs = b
        ck = tp._check
        qkv_txt = b["QKV"].view(T, M * 3 * Ds)[:, Mi * 3 * Ds:]  # rows [Mi, M) of every shard's block
        o_txt = b["O"].view(T, M * Ds)[:, Mi * Ds:]
        jobs = [(g["W_qkv_img"], 3 * D, D, tp.TP_COLWISE, b["wq_img"], [1, 1, 1]),
                (g["W_qkv_txt"], 3 * D, D, tp.TP_COLWISE, b["wq_txt"], [1, 1, 1]),
                (g["W_o_img"], D, D, tp.TP_ROWWISE, b["wo_img"]), (g["W_o_txt"], D, D, tp.TP_ROWWISE, b["wo_txt"])]
        # The step: one call of the prepared layer (tp_joint_attn_run), which
        # runs the two streams' projections side by side.  The same kernels
        # are then timed one at a time through the step-level calls.
        self._blk_step = tp.JointAttnBlock(g["W_qkv_img"], g["W_qkv_txt"], g["W_o_img"], g["W_o_txt"], H, T)
        nb = tp.tp_joint_attn_run_workspace_bytes(Mi, Mt, D, H, T)
        b["ws"] = torch.empty(nb, dtype=torch.uint8, device=dev)
        b["Yj_img"] = torch.empty((Mi, D), dtype=torch.int16, device=dev)
        b["Yj_txt"] = torch.empty((Mt, D), dtype=torch.int16, device=dev)
        return [
            Kernel("slice_weights", "GB/s", 2.0 * 8 * D * D * 2,
                   lambda: ck(tp.tp_shard_weights_batch(jobs, T), "slice both streams' W_qkv, W_o"), load=True),
            Kernel("joint_layer", "TFLOP/s", self.work(),
                   lambda: ck(tp.tp_joint_attn_run(self._blk_step.handle, g["X_img"], Mi, g["X_txt"], Mt, b["Yj_img"],
                                                   b["Yj_txt"], b["ws"], nb), "tp_joint_attn_run"),
                   composite=True),
            Kernel("qkv_gemm_img", "TFLOP/s", 2.0 * Mi * D * 3 * D,
                   lambda: ck(tp.tp_colwise_linear_rows(g["X_img"], Mi, D, b["wq_img"], None, 3 * Ds, T, 0,
                                                        tp.TP_OUT_F16, b["QKV"], M), "qkv img"), breakdown=True),
            Kernel("qkv_gemm_txt", "TFLOP/s", 2.0 * Mt * D * 3 * D,
                   lambda: ck(tp.tp_colwise_linear_rows(g["X_txt"], Mt, D, b["wq_txt"], None, 3 * Ds, T, 0,
                                                        tp.TP_OUT_F16, qkv_txt.data_ptr(), M), "qkv txt"),
                   breakdown=True),
            Kernel("sdpa", "TFLOP/s", 4.0 * M * M * D,
                   lambda: ck(tp.tp_sdpa_shards(b["QKV"], M, H, T, b["O"]), "sdpa"), breakdown=True),
            Kernel("out_gemm_img", "TFLOP/s", 2.0 * Mi * D * D,
                   lambda: ck(tp.tp_rowwise_linear_sum_rows(b["O"], Mi, Ds, M, b["wo_img"], D, None, T, b["Y_img"]),
                              "out img"), breakdown=True),
            Kernel("out_gemm_txt", "TFLOP/s", 2.0 * Mt * D * D,
                   lambda: ck(tp.tp_rowwise_linear_sum_rows(o_txt.data_ptr(), Mt, Ds, M, b["wo_txt"], D, None, T,
                                                            b["Y_txt"]), "out txt"), breakdown=True),
        ]

    def one_shot(self, tp, gi, dev):
        import torch
        c = self.cfg
        Mi, Mt, D, H, T = c["M_img"], c["M_txt"], c["D"], c["H"], c["T"]
        if not hasattr(self, "_ws"):
            self._ws = torch.empty(tp.tp_joint_attn_workspace_bytes(Mi, Mt, D, H, T), dtype=torch.uint8,
                                   device=dev)
            self._y = torch.empty((Mi + Mt, D), dtype=torch.int16, device=dev)
        tp._check(tp.tp_joint_attn_block(gi["X_img"], Mi, gi["X_txt"], Mt, D, gi["W_qkv_img"], gi["W_qkv_txt"],
                                         gi["W_o_img"], gi["W_o_txt"], H, T, self._y, self._y[Mi:], self._ws,
                                         self._ws.numel()), "tp_joint_attn_block")
        return self._y

    e2e_call = ("tp_joint_attn_block with both streams' X and weights copied from pinned host memory and "
                "Y_img, Y_txt copied back")

    def prepared(self, tp, g, dev):
        c = self.cfg
        self._blk = tp.JointAttnBlock(g["W_qkv_img"], g["W_qkv_txt"], g["W_o_img"], g["W_o_txt"], c["H"], c["T"])
        return ["X_img", "X_txt"], lambda gi, b: self._blk(gi["X_img"], gi["X_txt"]), (
            "JointAttnBlock: tp_joint_attn_prepare once, tp_joint_attn_run every step with both streams' X copied "
            "from pinned host memory and Y_img, Y_txt copied back")

    def oracle_run(self, d, rows):
        import oracle as o
        c = self.cfg
        Mi, Mt, D, H, T = c["M_img"], c["M_txt"], c["D"], c["H"], c["T"]
        M = Mi + Mt
        f = _f64(d, ["X_img", "X_txt", "W_qkv_img", "W_qkv_txt", "W_o_img", "W_o_txt"])
        ri = list(range(min(rows, Mi)))
        rt = list(range(max(0, rows - Mi)))
        t0 = time.perf_counter()
        o.joint_attn_rows(f["X_img"], f["X_txt"], f["W_qkv_img"], f["W_qkv_txt"], f["W_o_img"], f["W_o_txt"], H,
                          ri, rt, tp_degree=T)
        n = len(ri) + len(rt)
        done = 2.0 * M * D * 2 * D + 2.0 * n * D * D + 4.0 * n * M * D + 2.0 * n * D * D
        return time.perf_counter() - t0, done

    oracle_fn = "joint_attn_rows"

    def config(self, world):
        c = self.cfg
        return {"workload": (f"flux_joint_attn: TP dual-stream joint attention (image and text streams' head-split "
                             f"QKV colwise, one per-shard SDPA over both streams' tokens, per-stream rowwise "
                             f"out-projections with the sum fused); M_img={c['M_img']}, M_txt={c['M_txt']}, "
                             f"D={c['D']}, {c['H']} heads x 128"),
                "M_img": c["M_img"], "M_txt": c["M_txt"], "D": c["D"], "heads": c["H"], "tp_degree": c["T"],
                "global_batch_tokens": (c["M_img"] + c["M_txt"]) * world}


class RingAttnWorkload(AttnWorkload):
    """flux_ring_attn: Ring attention ("Context parallelism" page) over the
    flux_attn tokens, R = 4 ranks emulated on one GPU.  Q/K/V (24 heads x 128,
    fp16, the projections a flux_attn block makes) are split into R token
    blocks.  Step s: every rank r attends its queries to the key/value block
    it holds then, rank (r - s) mod R's -- one tp_sdpa_block_stats launch over
    all ranks, the blocks laid out twice so that the rotation is a pointer
    offset (on R GPUs it is the NCCL send/recv of the block) -- and a final
    tp_attn_merge per step combines the R results.  Work: the SDPA's 4 M^2 D."""
    prepared = _no_prepared_form
    key = "flux_ring_attn"
    metric = "Ring-attention (context parallel, 4 ranks on 1 GPU) TFLOP/s on 1 B200"
    R = 4

    def host_inputs(self, rank):
        import synthetic as syn
        c = self.cfg
        return {"QKV": syn.normal_f16((c["M"], 3 * c["D"]), 1.0, seed=c["seed"] + rank, tid=420)}

    def work(self):
        M, D = self.cfg["M"], self.cfg["D"]
        return 4.0 * M * M * D

    def kernels(self, tp, g, dev):
        import torch
        c = self.cfg
        M, D, H, R = c["M"], c["D"], c["H"], self.R
        Ms = M // R
        qkv = g["QKV"].view(R, Ms, 3 * D)
        ring = torch.cat([qkv, qkv]).contiguous()  # blocks 0..R-1 twice: step s starts at block R - s
        b = {"ring": ring, "O": torch.empty((R, R, Ms, D), dtype=torch.float16, device=dev),
             "L": torch.empty((R, R, H, Ms), dtype=torch.float32, device=dev),
             "Y": torch.empty((R, Ms, D), dtype=torch.int16, device=dev)}
        self.bufs = b
        ck = tp._check
        blk = Ms * 3 * D  # elements per token block
        ks = []
        for st in range(R):
            ks.append(Kernel(f"ring_step{st}", "TFLOP/s", 4.0 * M * Ms * D,
                             lambda st=st: ck(tp.tp_sdpa_block_stats(qkv, Ms, ring.data_ptr() + 2 * (R - st) * blk,
                                                                     Ms, H * R, R, b["O"][st], b["L"][st]),
                                              f"ring step {st}")))
        ks.append(Kernel("merge", "GB/s", R * (M * D * 2 + H * M * 4) + M * D * 2,
                         lambda: ck(tp.tp_attn_merge(b["O"], b["L"], R, Ms, H * R, R, b["Y"]), "merge")))
        return ks

    def one_shot(self, tp, gi, dev):
        """Every step's kernels on the staged inputs `gi` (buffers from torch's caching allocator)."""
        for k in self.kernels(tp, gi, dev):
            k.fn()
        return self.bufs["Y"]

    e2e_call = "tp_sdpa_block_stats per ring step and tp_attn_merge, Q/K/V copied from pinned host memory, O back"

    def oracle_run(self, d, rows):
        import oracle as o
        import synthetic as syn
        c = self.cfg
        M, D, H = c["M"], c["D"], c["H"]
        q = syn.f16_bits_to_f64(d["QKV"])
        t0 = time.perf_counter()
        for h in range(H):
            o.sdpa(q[:rows, h * 128:(h + 1) * 128], q[:, D + h * 128:D + (h + 1) * 128],
                   q[:, 2 * D + h * 128:2 * D + (h + 1) * 128])
        return time.perf_counter() - t0, 4.0 * rows * M * D

    oracle_fn = "sdpa over all keys (the result Ring attention must reach)"

    def config(self, world):
        c = self.cfg
        return {"workload": (f"flux_ring_attn: Ring attention over {c['M']} tokens, {self.R} ranks emulated on one "
                             f"GPU, {c['H']} heads x 128 (fp16 Q/K/V)"), "M": c["M"], "D": c["D"], "heads": c["H"],
                "ring_degree": self.R, "global_batch_tokens": c["M"] * world}


class UlyssesAttnWorkload(RingAttnWorkload):
    """flux_ulysses_attn: Ulysses attention ("Context parallelism" page) over
    the flux_attn tokens, U = 4 ranks emulated on one GPU.  Each rank packs
    its tokens' Q/K/V by destination head group (packed rowwise slicing,
    blocks [1, 1, 1]; all ranks in one launch), the all-to-all moves the
    blocks (device copies here, timed as their own entry; NCCL on U GPUs),
    each rank attends all M tokens of its H/U heads (one launch for all ranks:
    the ranks are the SDPA's shards), the reverse all-to-all brings the rows
    home and each rank puts its head groups back in place
    (tp_unshard_rowwise_all).  Work: the SDPA's 4 M^2 D."""
    key = "flux_ulysses_attn"
    metric = "Ulysses-attention (context parallel, 4 ranks on 1 GPU) TFLOP/s on 1 B200"
    R = 4

    def kernels(self, tp, g, dev):
        import torch
        c = self.cfg
        M, D, H, U = c["M"], c["D"], c["H"], self.R
        Ms, C = M // U, 3 * D
        qkv = g["QKV"].view(U, Ms, C)
        b = {"send": torch.empty((U, U, Ms, C // U), dtype=torch.int16, device=dev),   # [src][dst]
             "recv": torch.empty((U, U, Ms, C // U), dtype=torch.int16, device=dev),   # [dst][src] = [dst][M][..]
             "O": torch.empty((U, M, D // U), dtype=torch.int16, device=dev),           # [rank = shard][M][(H/U) 128]
             "back": torch.empty((U, U, Ms, D // U), dtype=torch.int16, device=dev),   # [dst][src]
             "Y": torch.empty((U, Ms, D), dtype=torch.int16, device=dev)}
        self.bufs = b
        ck = tp._check
        jobs = [(qkv[s], Ms, C, tp.TP_ROWWISE, b["send"][s], [1, 1, 1]) for s in range(U)]

        def a2a(dst, src):  # the all-to-all: block [i][j] of src lands at [j][i] of dst
            dst.copy_(src.transpose(0, 1))

        return [
            Kernel("pack", "GB/s", 2.0 * M * C * 2, lambda: ck(tp.tp_shard_weights_batch(jobs, U), "pack")),
            Kernel("alltoall_emulated", "GB/s", 2.0 * M * C * 2, lambda: a2a(b["recv"], b["send"]), exchange=True),
            Kernel("sdpa", "TFLOP/s", 4.0 * M * M * D,
                   lambda: ck(tp.tp_sdpa_shards(b["recv"], M, H, U, b["O"]), "sdpa")),
            Kernel("alltoall_back_emulated", "GB/s", 2.0 * M * D * 2,
                   lambda: a2a(b["back"], b["O"].view(U, U, Ms, D // U)), exchange=True),
            Kernel("unpack", "GB/s", 2.0 * M * D * 2,
                   lambda: [ck(tp.tp_unshard_rowwise_all(b["back"][s], Ms, D, U, b["Y"][s]), "unpack")
                            for s in range(U)]),
        ]

    e2e_call = ("pack, all-to-all (device copies), tp_sdpa_shards, all-to-all back, tp_unshard_rowwise_all; Q/K/V "
                "copied from pinned host memory, O back")

    def config(self, world):
        d = RingAttnWorkload.config(self, world)
        d["workload"] = d["workload"].replace("flux_ring_attn: Ring", "flux_ulysses_attn: Ulysses")
        d["ulysses_degree"] = d.pop("ring_degree")
        return d


class BlockWorkload(AttnWorkload):
    """wide_block: attention then MLP pair at tp_degree 8 (every row a1..a7)."""
    key = "wide_block"
    metric = "TP DiT-block (attention + MLP pair) TFLOP/s on 1 B200"

    def __init__(self, cfg=None):
        import synthetic as syn
        self.cfg = cfg or syn.CONFIGS["wide_block"]

    def host_inputs(self, rank):
        import synthetic as syn
        c = self.cfg
        d = syn.block_inputs(c["M"], c["D"], c["F"], c["seed"])
        if rank:
            d["X"] = syn.normal_bf16((c["M"], c["D"]), 1.0, seed=c["seed"] + 1000 * rank, tid=syn.TID["X"])
        return d

    def work(self):
        c = self.cfg
        return AttnWorkload.work(self) + 4.0 * c["M"] * c["D"] * c["F"]

    def kernels(self, tp, g, dev):
        c = self.cfg
        M, D, H, F, T = c["M"], c["D"], c["H"], c["F"], c["T"]
        ks, b = self.attn_kernels(tp, g, dev, g["X"], M, D, H, T, prefix="attn_")
        mlp = MlpWorkload(dict(M=M, D=D, F=F, T=T, seed=c["seed"]))
        g2 = dict(g)
        g2["X"] = b["A"]
        ks += [Kernel("mlp_" + k.name, k.unit, k.work, k.fn, k.load) for k in mlp.kernels(tp, g2, dev)]
        self.bufs = {**b, **mlp.bufs}
        return ks

    def one_shot(self, tp, gi, dev):
        import torch
        c = self.cfg
        M, D, H, F, T = c["M"], c["D"], c["H"], c["F"], c["T"]
        if not hasattr(self, "_ws"):
            self._ws = torch.empty(max(tp.tp_attn_workspace_bytes(M, D, H, T), tp.tp_mlp_workspace_bytes(M, D, F, T)),
                                   dtype=torch.uint8, device=dev)
            self._a = torch.empty((M, D), dtype=torch.int16, device=dev)
            self._y = torch.empty((M, D), dtype=torch.int16, device=dev)
        tp._check(tp.tp_attn_block(gi["X"], M, D, gi["W_qkv"], gi["W_o"], H, T, self._a, self._ws,
                                   self._ws.numel()), "tp_attn_block")
        tp._check(tp.tp_mlp_pair(self._a, M, D, F, gi["W_up"], gi["b_up"], gi["W_down"], gi["b_down"], T, self._y,
                                 self._ws, self._ws.numel()), "tp_mlp_pair")
        return self._y

    e2e_call = ("tp_attn_block then tp_mlp_pair with X and all weights copied from pinned host memory and Y "
                "copied back")

    def prepared(self, tp, g, dev):
        import torch
        c = self.cfg
        self._blk = tp.AttnBlock(g["W_qkv"], g["W_o"], c["H"], c["T"])
        self._pair = tp.MlpPair(g["W_up"], g["b_up"], g["W_down"], g["b_down"], c["T"])
        self._ap = torch.empty((c["M"], c["D"]), dtype=torch.int16, device=dev)
        self._yp = [torch.empty((c["M"], c["D"]), dtype=torch.int16, device=dev) for _ in range(2)]
        return ["X"], lambda gi, b: self._pair(self._blk(gi["X"], Y=self._ap), Y=self._yp[b]), (
            "AttnBlock then MlpPair (prepared once), run every step on X copied from pinned host memory, Y copied "
            "back")

    def oracle_run(self, d, rows):
        import oracle as o
        c = self.cfg
        M, D, H, F, T = c["M"], c["D"], c["H"], c["F"], c["T"]
        f = _f64(d, ["X", "W_qkv", "W_o", "W_up", "b_up", "W_down", "b_down"])
        t0 = time.perf_counter()
        o.block_rows(f["X"], f["W_qkv"], f["W_o"], H, f["W_up"], f["b_up"], f["W_down"], f["b_down"],
                     list(range(rows)), tp_degree=T)
        done = (2.0 * M * D * 2 * D + 2.0 * rows * D * D + 4.0 * rows * M * D + 2.0 * rows * D * D
                + 4.0 * rows * D * F)
        return time.perf_counter() - t0, done

    oracle_fn = "block_rows"

    def config(self, world):
        c = self.cfg
        return {"workload": (f"wide_block: attention block then MLP pair, tp_degree {c['T']}; M={c['M']}, "
                             f"D={c['D']}, {c['H']} heads x 128, F={c['F']}"),
                "M": c["M"], "D": c["D"], "heads": c["H"], "F": c["F"], "tp_degree": c["T"],
                "global_batch_tokens": c["M"] * world}


class ReduceWorkload(MlpWorkload):
    """flux_reduce: the standalone partial-sum reduction (a8) on flux_mlp-sized partials."""
    prepared = _no_prepared_form
    key = "flux_reduce"
    metric = "TP partial-sum reduction GB/s on 1 B200"
    unit = "GB/s"

    def __init__(self, cfg=None):
        import synthetic as syn
        c = syn.CONFIGS["flux_mlp"]
        self.cfg = cfg or dict(M=c["M"], N=c["D"], T=c["T"], seed=c["seed"])

    def host_inputs(self, rank):
        import numpy as np
        import synthetic as syn
        c = self.cfg
        parts = syn.bf16_bits_to_f32(syn.normal_bf16((c["T"], c["M"], c["N"]), 1.0, seed=c["seed"] + rank,
                                                     tid=200))
        return {"parts": np.ascontiguousarray(parts), "bias": syn.normal_bf16((c["N"],), 0.02, c["seed"], 202)}

    def work(self):
        c = self.cfg
        return 4.0 * c["T"] * c["M"] * c["N"] + 2.0 * c["M"] * c["N"] + 2.0 * c["N"]

    def kernels(self, tp, g, dev):
        import torch
        c = self.cfg
        self.bufs = {"Y": torch.empty((c["M"], c["N"]), dtype=torch.int16, device=dev)}
        return [Kernel("reduce", "GB/s", self.work(),
                       lambda: tp._check(tp.tp_reduce_partials(g["parts"], c["M"], c["N"], c["T"], g["bias"],
                                                               self.bufs["Y"]), "reduce"))]

    def one_shot(self, tp, gi, dev):
        c = self.cfg
        tp._check(tp.tp_reduce_partials(gi["parts"], c["M"], c["N"], c["T"], gi["bias"], self.bufs["Y"]), "reduce")
        return self.bufs["Y"]

    e2e_call = "tp_reduce_partials with the fp32 partials copied from pinned host memory and Y copied back"

    def oracle_run(self, d, rows):
        import numpy as np
        import oracle as o
        import synthetic as syn
        c = self.cfg
        parts = [d["parts"][r][:rows].astype(np.float64) for r in range(c["T"])]
        t0 = time.perf_counter()
        o.reduce_partials(parts, syn.bf16_bits_to_f64(d["bias"]))
        return time.perf_counter() - t0, rows * (4.0 * c["T"] * c["N"] + 2.0 * c["N"])

    oracle_fn = "reduce_partials"

    def config(self, world):
        c = self.cfg
        return {"workload": f"flux_reduce: Y = bf16(sum of {c['T']} fp32 partials + bias), {c['M']} x {c['N']}",
                "M": c["M"], "N": c["N"], "tp_degree": c["T"], "global_batch_tokens": c["M"] * world}


class SwigluWorkload(MlpWorkload):
    """flux_swiglu: the SwiGLU pair with gate and up packed (blocks [1, 1]):
    packed colwise slicing of W_in and b_in with W_out's rowwise slicing in
    one launch, the SwiGLU colwise GEMM, the rowwise GEMM."""
    key = "flux_swiglu"
    metric = "TP SwiGLU MLP-pair bf16 TFLOP/s on 1 B200"

    def __init__(self, cfg=None):
        import synthetic as syn
        self.cfg = cfg or syn.CONFIGS["flux_swiglu"]

    def host_inputs(self, rank):
        import synthetic as syn
        c = self.cfg
        d = syn.swiglu_inputs(c["M"], c["D"], c["F"], c["seed"])
        if rank:
            d["X"] = syn.normal_bf16((c["M"], c["D"]), 1.0, seed=c["seed"] + 1000 * rank, tid=syn.TID["X"])
        return d

    def work(self):
        c = self.cfg
        return 6.0 * c["M"] * c["D"] * c["F"]  # 2 M D (2F) for gate+up, 2 M F D for the out-projection

    def kernels(self, tp, g, dev):
        import torch
        M, D, F, T = self.cfg["M"], self.cfg["D"], self.cfg["F"], self.cfg["T"]
        Fs = F // T
        b = {"w_in": torch.empty((T, 2 * Fs, D), dtype=torch.int16, device=dev),
             "b_in": torch.empty((T, 2 * Fs), dtype=torch.int16, device=dev),
             "w_out": torch.empty((T, D, Fs), dtype=torch.int16, device=dev),
             "H": torch.empty((T, M, Fs), dtype=torch.int16, device=dev),
             "Y": torch.empty((M, D), dtype=torch.int16, device=dev)}
        ck = tp._check
        self.bufs = b
        jobs = [(g["W_in"], 2 * F, D, tp.TP_COLWISE, b["w_in"], [1, 1]),
                (g["W_out"], D, F, tp.TP_ROWWISE, b["w_out"]),
                (g["b_in"], 1, 2 * F, tp.TP_ROWWISE, b["b_in"], [1, 1])]
        return [
            Kernel("slice_weights", "GB/s", 2.0 * (2 * F * D + D * F + 2 * F) * 2,
                   lambda: ck(tp.tp_shard_weights_batch(jobs, T), "slice W_in (packed), W_out, b_in (packed)"),
                   load=True),
            Kernel("colwise_swiglu", "TFLOP/s", 2.0 * M * D * 2 * F,
                   lambda: ck(tp.tp_colwise_swiglu(g["X"], M, D, b["w_in"], b["b_in"], Fs, T, b["H"]),
                              "colwise swiglu")),
            Kernel("rowwise_gemm", "TFLOP/s", 2.0 * M * F * D,
                   lambda: ck(tp.tp_rowwise_linear_sum(b["H"], M, Fs, b["w_out"], D, g["b_out"], T, b["Y"]),
                              "rowwise")),
        ]

    def one_shot(self, tp, gi, dev):
        import torch
        M, D, F, T = self.cfg["M"], self.cfg["D"], self.cfg["F"], self.cfg["T"]
        if not hasattr(self, "_ws"):
            self._ws = torch.empty(tp.tp_swiglu_workspace_bytes(M, D, F, T), dtype=torch.uint8, device=dev)
            self._y = torch.empty((M, D), dtype=torch.int16, device=dev)
        tp._check(tp.tp_swiglu_mlp_pair(gi["X"], M, D, F, gi["W_in"], gi["b_in"], gi["W_out"], gi["b_out"], T,
                                        self._y, self._ws, self._ws.numel()), "tp_swiglu_mlp_pair")
        return self._y

    e2e_call = "tp_swiglu_mlp_pair with X, W_in, b_in, W_out, b_out copied from pinned host memory and Y copied back"

    def prepared(self, tp, g, dev):
        import torch
        c = self.cfg
        self._pair = tp.MlpPair(g["W_in"], g["b_in"], g["W_out"], g["b_out"], c["T"], activation="swiglu")
        self._yp = [torch.empty((c["M"], c["D"]), dtype=torch.int16, device=dev) for _ in range(2)]
        return ["X"], lambda gi, b: self._pair(gi["X"], Y=self._yp[b]), (
            "MlpPair(activation='swiglu'): tp_swiglu_prepare once, tp_mlp_run every step with X copied from "
            "pinned host memory and Y copied back")

    def oracle_run(self, d, rows):
        import oracle as o
        import synthetic as syn
        c = self.cfg
        f = _f64(d, ["W_in", "b_in", "W_out", "b_out"])
        X = syn.bf16_bits_to_f64(d["X"][:rows])
        t0 = time.perf_counter()
        o.swiglu_sharded_summed(X, f["W_in"], f["b_in"], f["W_out"], f["b_out"], c["T"])
        return time.perf_counter() - t0, 6.0 * rows * c["D"] * c["F"]

    oracle_fn = "swiglu_sharded_summed"

    def config(self, world):
        c = self.cfg
        return {"workload": (f"flux_swiglu: TP SwiGLU pair (gate/up packed colwise with blocks [1, 1], "
                             f"silu(gate) * up fused in the colwise epilogue, rowwise out-projection with the "
                             f"cross-shard sum fused); M={c['M']}, D={c['D']}, F={c['F']} (mlp_ratio 3)"),
                "M": c["M"], "D": c["D"], "F": c["F"], "tp_degree": c["T"],
                "global_batch_tokens": c["M"] * world}


class SplitInputWorkload(MlpWorkload):
    """flux_split_input: rowwise_split_input, the replicated input sliced by TMA
    coordinates inside the rowwise GEMM (FFN-out sized)."""
    prepared = _no_prepared_form
    key = "flux_split_input"
    metric = "TP rowwise_split_input bf16 TFLOP/s on 1 B200"

    def __init__(self, cfg=None):
        import synthetic as syn
        c = syn.CONFIGS["flux_mlp"]
        self.cfg = cfg or dict(M=c["M"], K=c["F"], N=c["D"], T=c["T"], seed=5)

    def host_inputs(self, rank):
        import numpy as np
        import synthetic as syn
        c = self.cfg
        return {"X": syn.normal_bf16((c["M"], c["K"]), 1.0, c["seed"] + 1000 * rank, syn.TID["X"]),
                "W": syn.normal_bf16((c["N"], c["K"]), 1.0 / np.sqrt(c["K"]), c["seed"], syn.TID["W_down"]),
                "b": syn.normal_bf16((c["N"],), 0.02, c["seed"], syn.TID["b_down"])}

    def work(self):
        c = self.cfg
        return 2.0 * c["M"] * c["K"] * c["N"]

    def kernels(self, tp, g, dev):
        import torch
        M, K, N, T = self.cfg["M"], self.cfg["K"], self.cfg["N"], self.cfg["T"]
        b = {"w": torch.empty((T, N, K // T), dtype=torch.int16, device=dev),
             "Y": torch.empty((M, N), dtype=torch.int16, device=dev)}
        ck = tp._check
        self.bufs = b
        return [
            Kernel("slice_w", "GB/s", 2.0 * N * K * 2,
                   lambda: ck(tp.tp_shard_weight_all(g["W"], N, K, tp.TP_ROWWISE_SPLIT_INPUT, T, b["w"]),
                              "slice W"), load=True),
            Kernel("split_input_gemm", "TFLOP/s", self.work(),
                   lambda: ck(tp.tp_rowwise_split_input_linear(g["X"], M, K, b["w"], N, g["b"], T, b["Y"]),
                              "split input")),
        ]

    def one_shot(self, tp, gi, dev):
        M, K, N, T = self.cfg["M"], self.cfg["K"], self.cfg["N"], self.cfg["T"]
        ck = tp._check
        ck(tp.tp_shard_weight_all(gi["W"], N, K, tp.TP_ROWWISE_SPLIT_INPUT, T, self.bufs["w"]), "slice W")
        ck(tp.tp_rowwise_split_input_linear(gi["X"], M, K, self.bufs["w"], N, gi["b"], T, self.bufs["Y"]),
           "split input")
        return self.bufs["Y"]

    e2e_call = ("tp_shard_weight_all + tp_rowwise_split_input_linear with X, W, b copied from pinned host memory "
                "and Y copied back")

    def oracle_run(self, d, rows):
        import oracle as o
        import synthetic as syn
        c = self.cfg
        W = syn.bf16_bits_to_f64(d["W"])
        b = syn.bf16_bits_to_f64(d["b"])
        X = syn.bf16_bits_to_f64(d["X"][:rows])
        t0 = time.perf_counter()
        o.rowwise_split_input(X, W, b, c["T"])
        return time.perf_counter() - t0, 2.0 * rows * c["K"] * c["N"]

    oracle_fn = "rowwise_split_input"

    def config(self, world):
        c = self.cfg
        return {"workload": (f"flux_split_input: rowwise_split_input (replicated input, each shard reads its "
                             f"K/T columns in place), M={c['M']}, K={c['K']}, N={c['N']}"),
                "M": c["M"], "K": c["K"], "N": c["N"], "tp_degree": c["T"], "global_batch_tokens": c["M"] * world}


WORKLOADS = {w.key: w for w in (MlpWorkload, SweepWorkload, AttnWorkload, BlockWorkload, ReduceWorkload,
                                SwigluWorkload, SplitInputWorkload, JointAttnWorkload, RingAttnWorkload,
                                UlyssesAttnWorkload)}


def workload_cfg():
    """The default workload's configuration."""
    return MlpWorkload().cfg


def _scale(unit):
    return 1e12 if unit == "TFLOP/s" else 1e9


# --------------------------------------------------------------------------- CPU oracle legs
def _rows_for(wl, d, seconds: float) -> int:
    """Token rows of the workload the oracle processes in about `seconds`: the
    per-row cost and the fixed cost (slicing, K/V of every token) from two
    probe sizes."""
    M = wl.cfg["M"]
    wl.oracle_run(d, 8)  # warm
    t1, _ = wl.oracle_run(d, 16)
    t2, _ = wl.oracle_run(d, 64)
    per_row = max((t2 - t1) / 48.0, 1e-7)
    fixed = max(t1 - 16 * per_row, 0.0)
    return int(min(M, max(16, (seconds - fixed) / per_row)))


def cpu_baseline(wl, d, budget_s: float = 15.0):
    """The oracle as it stands, on a bounded sample of the workload's token rows."""
    M = wl.cfg["M"]
    rows = _rows_for(wl, d, budget_s)
    if wl.key in ("flux_attn", "wide_block", "flux_joint_attn"):
        rows = min(rows, 256)  # the K/V projection of every token dominates; more rows add little
    t, done = wl.oracle_run(d, rows)
    return {"value": done / t / _scale(wl.unit), "unit": wl.unit, "cores": oracle_threads(), "kind": "oracle",
            "sample": f"{rows} of {M} token rows of the workload through the fp64 oracle ({wl.oracle_fn}, "
                      f"tp_degree {wl.cfg['T']}), {t:.1f} s; value = work the oracle performed / time"}


def run_reference(args, wl, rank, world):
    if rank != 0:
        return None  # rank 0 alone runs the CPU reference
    d = wl.host_inputs(0)
    M = wl.cfg["M"]
    per_step = max(0.2, min(5.0, 120.0 / max(1, args.steps + args.warmup)))
    rows = _rows_for(wl, d, per_step)
    for _ in range(args.warmup):
        wl.oracle_run(d, rows)
    res = [wl.oracle_run(d, rows) for _ in range(args.steps)]
    total = sum(r[0] for r in res)
    value = sum(r[1] for r in res) / total / _scale(wl.unit)
    sample = (f"{rows} of {M} token rows per step through the fp64 oracle ({wl.oracle_fn}, "
              f"tp_degree {wl.cfg['T']}) on host cores")
    return {
        "impl": "reference", "metric": wl.metric, "value": value, "unit": wl.unit, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": config_dict(wl, world),
        "cpu_baseline": {"value": value, "unit": wl.unit, "cores": oracle_threads(), "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": wl.unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def config_dict(wl, world):
    d = wl.config(world)
    d["l2"] = ("not flushed: inputs larger than L2 (the step reads more than 126 MB of inputs and moves "
               "several times that)")
    d["parallelism"] = "single GPU" if world == 1 else f"{world} independent replicas (one per GPU)"
    return d


# --------------------------------------------------------------------------- GPU leg
def run_ours(args, wl, rank, local_rank, world, light=False):
    import numpy as np
    import torch

    import tensor_transformer_layers_b200 as tp

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    d = wl.host_inputs(rank)

    def pin(v):
        a = np.ascontiguousarray(v)
        t = torch.from_numpy(a.view(np.int16) if a.dtype == np.uint16 else a)
        return t.pin_memory()

    host = {k: pin(v) for k, v in d.items()}
    g = {k: v.to(dev) for k, v in host.items()}
    input_bytes = sum(v.numel() * v.element_size() for v in g.values())
    # Inputs larger than L2 need no flush between steps; smaller ones get one.
    flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev) if input_bytes <= L2_BYTES else None
    kernels = wl.kernels(tp, g, dev)
    names = [k.name for k in kernels]
    nk = len(kernels)

    def step(ev):
        ev[0].record()
        for j, k in enumerate(kernels):
            k.fn()
            ev[j + 1].record()

    def new_events():
        return [torch.cuda.Event(enable_timing=True) for _ in range(nk + 1)]

    for _ in range(args.warmup):
        if flush is not None:
            flush.zero_()
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
        if flush is not None:
            flush.zero_()  # outside the step's events
        step(evs[i])
    torch.cuda.synchronize()
    t_wall = time.perf_counter() - t_wall0
    clocks = sampler.stop()
    launches = tp.tp_kernel_launches() - launches0
    barrier()
    assert tp.tp_check_device_error() == 0

    per_kernel = {n: [] for n in names}
    step_ms, one_shot_ms, exch_ms = [], [], []
    for ev in evs:
        for j, n in enumerate(names):
            per_kernel[n].append(ev[j].elapsed_time(ev[j + 1]))
        # the step: the per-step kernels of the prepared layer; load-time slicing is timed beside it
        step_ms.append(sum(per_kernel[k.name][-1] for k in kernels if not (k.load or k.exchange or k.breakdown)))
        exch_ms.append(sum(per_kernel[k.name][-1] for k in kernels if k.exchange))
        one_shot_ms.append(sum(per_kernel[k.name][-1] for k in kernels if not (k.exchange or k.breakdown)))
    local_s = sum(step_ms) / 1e3
    max_s = max_over_ranks(local_s)
    max_one_shot_s = max_over_ranks(sum(one_shot_ms) / 1e3)
    scale = _scale(wl.unit)
    value = wl.work() * world * args.steps / max_s / scale
    one_shot_value = wl.work() * world * args.steps / max_one_shot_s / scale

    peaks, peak_src = load_peaks()
    tc_peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    hbm_peak = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    tot = sum(statistics.mean(v) for v in per_kernel.values())
    kinfo = {}
    for k in kernels:
        ms = statistics.mean(per_kernel[k.name])
        ach = k.work / (ms / 1e3) / _scale(k.unit)
        pk = tc_peak if k.unit == "TFLOP/s" else hbm_peak
        kinfo[k.name] = {"ms": round(ms, 5), "share": round(ms / tot, 4), "achieved": round(ach, 1),
                         "unit": k.unit, "frac": round(ach / pk, 4)}
    for k in kernels:
        if k.load:
            kinfo[k.name]["load_time"] = True
        if k.exchange:
            kinfo[k.name]["emulated_exchange"] = True
        if k.breakdown:
            kinfo[k.name]["breakdown"] = True
        if k.composite:
            kinfo[k.name]["composite"] = True
    # Attention's second bound: the exponentials (Mq * Mk * heads = FLOP / (4 * head dim 128)) against the MUFU
    # rate, 16 ex2 per clock per SM (the CUDA programming guide's arithmetic-throughput table).
    sm_count = torch.cuda.get_device_properties(dev).multi_processor_count
    mufu_peak = 16.0 * sm_count * float(clocks.get("sm_max_mhz") or 1965) * 1e6
    for k in kernels:
        if k.unit == "TFLOP/s" and ("sdpa" in k.name or k.name.startswith("ring_step")):
            rate = k.work / (4.0 * 128) / (kinfo[k.name]["ms"] / 1e3)
            kinfo[k.name]["exp_per_s"] = float(f"{rate:.4g}")
            kinfo[k.name]["exp_frac_of_mufu"] = round(rate / mufu_peak, 4)
    dom = max((k for k in kernels if not (k.load or k.exchange or k.composite)), key=lambda k: kinfo[k.name]["ms"])
    src = "MEASURED_PEAKS.json" if peak_src == "measured" else "the recipe's fallback"
    roofline = {"kernel": dom.name, "bound": "tensor" if dom.unit == "TFLOP/s" else "hbm",
                "achieved": kinfo[dom.name]["achieved"], "peak": tc_peak if dom.unit == "TFLOP/s" else hbm_peak,
                "unit": dom.unit, "frac": kinfo[dom.name]["frac"], "traffic": recorded_traffic(dom.name, wl.key),
                "peak_source": f"{peak_src}: {'bf16 burst' if dom.unit == 'TFLOP/s' else 'HBM copy'} from {src}",
                "algorithmic_work_per_launch": dom.work}
    if "exp_frac_of_mufu" in kinfo[dom.name]:
        roofline["mufu"] = {"exp_per_s": kinfo[dom.name]["exp_per_s"], "peak_exp_per_s": float(f"{mufu_peak:.4g}"),
                            "frac": kinfo[dom.name]["exp_frac_of_mufu"],
                            "peak_basis": f"16 ex2 per clock per SM x {sm_count} SMs x max SM clock"}

    # ---- end to end through the public API, every step's inputs copied in from pinned host memory and its
    # result copied back, as a serving loop runs it: step i+1's inputs are staged (second device buffer, own
    # stream) while step i computes, and the result's copy back runs on a third stream.  Every copy of every
    # step is inside the timed region.  The headline form is the prepared layer (weights sharded once, the
    # tokens are a step's input); the one-shot call (weights copied and sliced every step) is reported beside it.
    s_h2d, s_cmp, s_d2h = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)

    def e2e_measure(keys, fn, call, single_output):
        gis = [{k: torch.empty_like(host[k], device=dev) for k in keys} for _ in range(2)]
        y0 = fn(g if keys == list(host) else {k: g[k] for k in keys}, 0)
        ys = y0 if isinstance(y0, tuple) else (y0,)
        y_host = [torch.empty(y.shape, dtype=y.dtype).pin_memory() for y in ys]
        h2d = sum(host[k].numel() * host[k].element_size() for k in keys)
        d2h = sum(y.numel() * y.element_size() for y in y_host)

        def run(n, start_ev):
            for st in (s_h2d, s_cmp, s_d2h):
                st.wait_event(start_ev)
            used = [None, None]
            d2h_done = [None, None]
            for i in range(n):
                b = i & 1
                if used[b] is not None:
                    s_h2d.wait_event(used[b])  # step i-2 no longer reads this staging buffer
                with torch.cuda.stream(s_h2d):
                    for k in keys:
                        gis[b][k].copy_(host[k], non_blocking=True)
                    staged = torch.cuda.Event()
                    staged.record(s_h2d)
                s_cmp.wait_event(staged)
                if d2h_done[b] is not None:
                    s_cmp.wait_event(d2h_done[b])  # step i-2's result has left output buffer b
                if single_output and d2h_done[b ^ 1] is not None:
                    s_cmp.wait_event(d2h_done[b ^ 1])  # one output buffer: step i-1's result has left it
                with torch.cuda.stream(s_cmp):
                    y = fn(gis[b], b)
                    used[b] = torch.cuda.Event()
                    used[b].record(s_cmp)
                s_d2h.wait_event(used[b])
                with torch.cuda.stream(s_d2h):
                    for yh, yd in zip(y_host, y if isinstance(y, tuple) else (y,)):
                        yh.copy_(yd, non_blocking=True)
                    d2h_done[b] = torch.cuda.Event()
                    d2h_done[b].record(s_d2h)
            cur = torch.cuda.current_stream(dev)
            cur.wait_stream(s_h2d)
            cur.wait_stream(s_cmp)
            cur.wait_stream(s_d2h)

        def copies_only(n, start_ev):  # the same copies with no compute: the host link's own time
            for st in (s_h2d, s_d2h):
                st.wait_event(start_ev)
            for i in range(n):
                with torch.cuda.stream(s_h2d):
                    for k in keys:
                        gis[i & 1][k].copy_(host[k], non_blocking=True)
                with torch.cuda.stream(s_d2h):
                    for yh, yd in zip(y_host, ys):
                        yh.copy_(yd, non_blocking=True)
            cur = torch.cuda.current_stream(dev)
            cur.wait_stream(s_h2d)
            cur.wait_stream(s_d2h)

        def timed(fn):
            w0 = torch.cuda.Event()
            w0.record()
            fn(max(1, args.warmup), w0)
            torch.cuda.synchronize()
            barrier()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn(args.steps, e0)
            e1.record()
            torch.cuda.synchronize()
            t = max_over_ranks(e0.elapsed_time(e1) / 1e3)
            barrier()
            return t

        e2e_s = timed(run)
        copy_s = timed(copies_only)
        return {"value": wl.work() * world * args.steps / e2e_s / scale, "unit": wl.unit, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "call": call,
                "copy_only_ms_per_step": round(1e3 * copy_s / args.steps, 4),
                "frac_of_copy_bound": round(copy_s / e2e_s, 3),
                "pipelining": ("two device staging buffers" + ("" if single_output else " and two output buffers") +
                               ": step i+1's host-to-device copies overlap step i's compute; device-to-host "
                               "copies on a third stream; all copies inside the timed region")}

    # ---- context row: the same layer through torch / cuBLAS on the same inputs, timed the same way (not the
    # library, not in value)
    context = None
    if not light and getattr(args, "context_torch", False) and has_context_row(wl):
        ctx = wl.context(g, dev)
        for _ in range(max(3, args.warmup)):
            for _, _, _, fn in ctx:
                fn()
        torch.cuda.synchronize()
        cev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(ctx) + 1)] for _ in range(args.steps)]
        for i in range(args.steps):
            cev[i][0].record()
            for j, (_, _, _, fn) in enumerate(ctx):
                fn()
                cev[i][j + 1].record()
        torch.cuda.synchronize()
        context = {"note": "torch / cuBLAS on the same shapes and inputs, timed like the kernels above; outside "
                           "the library and the value"}
        for j, (name, unit, work, _) in enumerate(ctx):
            ms = statistics.mean(cev[i][j].elapsed_time(cev[i][j + 1]) for i in range(args.steps))
            context[name] = {"ms": round(ms, 5), "unit": unit, "achieved": round(work / (ms / 1e3) / (1e12 if unit == "TFLOP/s" else 1e9), 1)}
        tot = sum(context[n]["ms"] for n, _, _, _ in ctx)
        context["step_ms"] = round(tot, 5)
        context["value"] = round(wl.work() / (tot / 1e3) / 1e12, 1)

    if light:  # a secondary configuration of the default run: kernels and step only, no e2e legs
        one_shot_e2e, prep, e2e = None, None, None
    else:
        one_shot_e2e = e2e_measure(list(host), lambda gi, b: wl.one_shot(tp, gi, dev), wl.e2e_call, True)
        prep = wl.prepared(tp, g, dev)
        e2e = e2e_measure(prep[0], prep[1], prep[2], False) if prep is not None else one_shot_e2e

    out = {
        "metric": wl.metric, "value": value, "unit": wl.unit, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1e3 * max_s / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded)",
        "config": config_dict(wl, world),
    }
    if flush is not None:
        out["config"]["l2"] = (f"flushed before every step ({2 * L2_BYTES >> 20} MiB write, outside the step's "
                               f"events): the inputs ({input_bytes >> 20} MiB) fit in L2")
    out["median_ms_per_step"] = statistics.median(step_ms)
    if any(k.exchange for k in kernels):
        out["value_with_emulated_exchange"] = wl.work() * world * args.steps / max_over_ranks(
            (sum(step_ms) + sum(exch_ms)) / 1e3) / scale
        out["exchange"] = ("the ranks share one GPU, so the all-to-all between them is device copies, timed as "
                           "their own entries and left out of 'value' (on several GPUs it is NCCL's)")
    if any(k.load for k in kernels):
        out["step"] = ("the prepared layer's per-step kernels (shards sliced at load time, as each rank does when "
                       "the model is loaded); the load-time slicing runs in the same loop, outside the step, and "
                       "has its own entry in 'kernels'")
        out["one_shot_value"] = one_shot_value
        out["one_shot_ms_per_step"] = 1e3 * max_one_shot_s / args.steps
    if wl.unit == "TFLOP/s":
        out["frac_of_nominal_dense_bf16"] = round(value / world / 2250.0, 4)
        out["frac_of_measured_bf16"] = round(value / world / tc_peak, 4)
    groups = sorted({k.group for k in kernels if k.group is not None})
    if groups:
        per_group = {}
        for gk in groups:
            ks_g = [k for k in kernels if k.group == gk]
            ms_step = sum(kinfo[k.name]["ms"] for k in ks_g if not k.load)
            ms_all = sum(kinfo[k.name]["ms"] for k in ks_g)
            w_g = sum(k.work for k in ks_g if not k.load and k.unit == wl.unit)
            per_group[str(gk)] = {"ms": round(ms_step, 5), "value": round(w_g / (ms_step / 1e3) / scale, 1),
                                  "one_shot_ms": round(ms_all, 5),
                                  "one_shot_value": round(w_g / (ms_all / 1e3) / scale, 1),
                                  "frac_of_nominal_dense_bf16": round(w_g / (ms_step / 1e3) / scale / 2250.0, 4)}
        out["per_degree"] = per_group
    if prep is not None:
        out["e2e_one_shot"] = one_shot_e2e
    if context is not None:
        out["context_torch"] = context
    out.update({"roofline": roofline, "kernels": kinfo, "clocks": clocks, "e2e": e2e,
                "gpu_launches": int(launches), "wall_s_timed_region": round(t_wall, 4), "cpu_baseline": None})
    if rank == 0 and world == 1 and not args.no_cpu_baseline and not light:
        out["cpu_baseline"] = cpu_baseline(wl, d)
    return out


# The other configurations, timed after the headline line's own measurement in
# a default one-GPU run (same process, same box), each with a short loop:
# (workload, steps, warmup).
OTHER_CONFIGS = [("flux_attn", 10, 3), ("flux_mlp_sweep", 5, 3), ("wide_block", 3, 3), ("flux_reduce", 20, 3),
                 ("flux_swiglu", 10, 3), ("flux_split_input", 10, 3), ("flux_joint_attn", 10, 3),
                 ("flux_ring_attn", 10, 3), ("flux_ulysses_attn", 10, 3)]


def other_configs(args, rank, local_rank):
    """Compact lines for the other configurations and rows (attention block,
    tp_degree sweep, wide block, standalone reduction, SwiGLU pair,
    rowwise_split_input, joint attention, Ring and Ulysses attention): value,
    step time, the dominant kernel's roofline fraction and every kernel's
    rate.  A failure is reported in its entry and does not stop the headline
    line."""
    res = {}
    for key, steps, warmup in OTHER_CONFIGS:
        a = argparse.Namespace(**vars(args))
        a.steps, a.warmup, a.no_cpu_baseline = steps, warmup, True
        try:
            o = run_ours(a, WORKLOADS[key](), rank, local_rank, 1, light=True)
        except Exception as e:  # noqa: BLE001 - recorded in the line, the headline stands
            res[key] = {"error": f"{type(e).__name__}: {e}"}
            continue
        r = o["roofline"]
        res[key] = {"config": o["config"]["workload"], "value": round(o["value"], 1), "unit": o["unit"],
                    "steps": steps, "warmup": warmup, "ms_per_step": round(o["ms_per_step"], 5),
                    "roofline": {"kernel": r["kernel"], "achieved": r["achieved"], "peak": r["peak"],
                                 "unit": r["unit"], "frac": r["frac"]},
                    "kernels": {n: {"achieved": k["achieved"], "unit": k["unit"], "frac": k["frac"],
                                    **({"exp_frac_of_mufu": k["exp_frac_of_mufu"]} if "exp_frac_of_mufu" in k else {})}
                                for n, k in o["kernels"].items()},
                    "clocks": o["clocks"], "gpu_launches": o["gpu_launches"]}
        if "mufu" in r:
            res[key]["roofline"]["mufu_frac"] = r["mufu"]["frac"]
        for extra in ("per_degree", "frac_of_nominal_dense_bf16", "value_with_emulated_exchange"):
            if extra in o:
                res[key][extra] = o[extra]
    return res


def run_tp(args, wl, rank, local_rank, world):
    """--mode tp: tensor parallelism across processes.  tp_degree = world size;
    rank r holds only its own shards (cut once, as sharded loading would) and
    every step runs its partial (tp_*_rank_partial), ONE NCCL AllReduce(sum)
    of the fp32 [M x D] partial, and the finish (bias once, one bf16 rounding,
    tp_reduce_partials).  The layer's total work is fixed, so scaling is
    "strong"; X is replicated (every rank gets the same tokens)."""
    import numpy as np
    import torch
    import torch.distributed as dist

    import tensor_transformer_layers_b200 as tp
    from tensor_transformer_layers_b200.dist import AttnRank, MlpRank

    if wl.key not in ("flux_mlp", "flux_attn"):
        raise SystemExit("--mode tp runs the flux_mlp or flux_attn workload")
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    T = world
    d = wl.host_inputs(0)
    host = {k: torch.from_numpy(np.ascontiguousarray(v).view(np.int16)).pin_memory() for k, v in d.items()}
    g = {k: v.to(dev) for k, v in host.items()}
    c = wl.cfg
    M, D = c["M"], c["D"]
    if wl.key == "flux_mlp":
        obj = MlpRank(g["W_up"], g["b_up"], g["W_down"], g["b_down"], T, rank)
    else:
        obj = AttnRank(g["W_qkv"], g["W_o"], c["H"], T, rank)
    part = torch.empty((M, D), dtype=torch.float32, device=dev)
    Y = torch.empty((M, D), dtype=torch.int16, device=dev)
    grouped = dist.is_available() and dist.is_initialized()

    def step(ev, X):
        ev[0].record()
        obj.partial(X, out=part)
        ev[1].record()
        if grouped:
            dist.all_reduce(part, op=dist.ReduceOp.SUM)
        ev[2].record()
        obj.finish(part, out=Y)
        ev[3].record()

    new_events = lambda: [torch.cuda.Event(enable_timing=True) for _ in range(4)]  # noqa: E731
    for _ in range(args.warmup):
        step(new_events(), g["X"])
    torch.cuda.synchronize()
    sampler = ClockSampler(local_rank)
    evs = [new_events() for _ in range(args.steps)]
    barrier()
    torch.cuda.synchronize()
    launches0 = tp.tp_kernel_launches()
    sampler.start()
    for i in range(args.steps):
        step(evs[i], g["X"])
    torch.cuda.synchronize()
    clocks = sampler.stop()
    launches = tp.tp_kernel_launches() - launches0
    barrier()
    assert tp.tp_check_device_error() == 0
    parts_ms = [[ev[j].elapsed_time(ev[j + 1]) for ev in evs] for j in range(3)]
    local_s = sum(ev[0].elapsed_time(ev[3]) for ev in evs) / 1e3
    max_s = max_over_ranks(local_s)
    value = wl.work() * args.steps / max_s / 1e12

    peaks, peak_src = load_peaks()
    tc_peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    hbm_peak = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    ar_bytes = 2.0 * (T - 1) / T * M * D * 4  # ring AllReduce bus bytes of the fp32 partial
    fin_bytes = M * D * 4 + M * D * 2 + D * 2
    ms = [statistics.mean(x) for x in parts_ms]
    tot = sum(ms)
    kinfo = {
        "rank_partial": {"ms": round(ms[0], 5), "share": round(ms[0] / tot, 4), "unit": "TFLOP/s",
                         "achieved": round(wl.work() / T / (ms[0] / 1e3) / 1e12, 1)},
        "allreduce": {"ms": round(ms[1], 5), "share": round(ms[1] / tot, 4), "unit": "GB/s",
                      "achieved": round(ar_bytes / (ms[1] / 1e3) / 1e9, 1) if ms[1] > 0 and T > 1 else None,
                      "bytes": ar_bytes, "note": "NCCL AllReduce(sum) of the fp32 partial; bus bytes 2(T-1)/T x"},
        "finish": {"ms": round(ms[2], 5), "share": round(ms[2] / tot, 4), "unit": "GB/s",
                   "achieved": round(fin_bytes / (ms[2] / 1e3) / 1e9, 1)},
    }
    kinfo["rank_partial"]["frac"] = round(kinfo["rank_partial"]["achieved"] / tc_peak, 4)
    kinfo["finish"]["frac"] = round(kinfo["finish"]["achieved"] / hbm_peak, 4)
    # end to end: X copied in from pinned host memory and Y copied back every step
    y_host = torch.empty((M, D), dtype=torch.int16).pin_memory()
    x_dev = torch.empty_like(g["X"])
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        x_dev.copy_(host["X"], non_blocking=True)
        step(new_events(), x_dev)
        y_host.copy_(Y, non_blocking=True)
    e1.record()
    torch.cuda.synchronize()
    e2e_s = max_over_ranks(e0.elapsed_time(e1) / 1e3)
    barrier()
    cfg = config_dict(wl, world)
    cfg["tp_degree"] = T
    cfg["global_batch_tokens"] = M
    cfg["parallelism"] = (f"tp{T}: tensor parallelism across {T} process(es), one shard per rank, one NCCL "
                          f"AllReduce(sum) of the fp32 [M x D] partial per layer, bias once after the sum")
    return {
        "metric": wl.metric, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1e3 * max_s / args.steps, "higher_is_better": True,
        "scaling": "strong", "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded)", "config": cfg,
        "roofline": {"kernel": "rank_partial", "bound": "tensor", "achieved": kinfo["rank_partial"]["achieved"],
                     "peak": tc_peak, "unit": "TFLOP/s", "frac": kinfo["rank_partial"]["frac"], "traffic": None,
                     "peak_source": f"{peak_src}: bf16 burst"},
        "kernels": kinfo, "clocks": clocks,
        "e2e": {"value": wl.work() * args.steps / e2e_s / 1e12, "unit": "TFLOP/s",
                "h2d_bytes_per_step": host["X"].numel() * 2, "d2h_bytes_per_step": M * D * 2,
                "call": "rank partial + all_reduce + finish with X copied from pinned host memory, Y copied back"},
        "gpu_launches": int(launches), "cpu_baseline": None,
    }


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="flux_mlp",
                    help="flux_mlp (default: the headline line); the others time the remaining rows")
    ap.add_argument("--no-cpu-baseline", action="store_true",
                    help="leave out the CPU oracle leg (cpu_baseline is then null)")
    ap.add_argument("--headline-only", action="store_true",
                    help="leave out the other configurations that a default one-GPU run times after the "
                         "headline (other_configs)")
    ap.add_argument("--context-torch", action="store_true",
                    help="also time the same MLP pair through torch / cuBLAS (context_torch: a context row outside "
                         "the library and the value; flux_mlp only)")
    ap.add_argument("--mode", choices=["replicas", "tp"], default="replicas",
                    help="replicas (default): every GPU runs the whole layer (all tp_degree shards) on its own "
                         "tokens; tp: tensor parallelism across the processes, one shard per rank, one NCCL "
                         "AllReduce per layer (flux_mlp / flux_attn)")
    args = ap.parse_args(argv)
    rank, local_rank, world = dist_env()
    wl = WORKLOADS[args.workload]()

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
            out = run_reference(args, wl, rank, world)
        elif args.mode == "tp":
            out = run_tp(args, wl, rank, local_rank, world)
        else:
            out = run_ours(args, wl, rank, local_rank, world)
            if world == 1 and args.workload == "flux_mlp" and not args.headline_only:
                out["other_configs"] = other_configs(args, rank, local_rank)
        if rank == 0 and out is not None:
            print(json.dumps(out), flush=True)
    finally:
        if world > 1 and args.impl == "ours":
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
