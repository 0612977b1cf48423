"""Benchmark of the tensor-parallel Transformer layer forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--shards N] [--no-cpu-baseline]

A step is one forward pass of the whole hot path over one batch: the
pre-LN layer (LN1 -> QKV column-parallel -> local attention -> W_O
row-parallel -> partial sum + residual + LN2 -> MLP column-parallel +
GeLU -> row-parallel -> partial sum + residual) on 2 x 2048 tokens, h 4096,
32 heads x 128, FFN 16384, N = 8 shards, through tp_layer_forward. Inputs
are seeded synthetic bf16 (see tensor_transformer_layer_linear_b200/synth.py)
and already resident in HBM when timing starts; the per-step working set
(weights 402 MB, partials 537 MB) is far larger than the 126 MB L2, so no
flush is needed between steps.

Printed (rank 0, one JSON line): whole-job TFLOP/s of algorithmic work,
the dominant kernel's roofline (from CUDA events around every launch in
the timed region), the partial-sum reduction's HBM bandwidth, an end-to-end
figure through the C ABI with host buffers, the fp64 oracle timed on the
host cores on a bounded sample, SM clocks sampled during the timed region,
and the number of library kernel launches.

With --gpus N > 1 (launched under torch.distributed.run) every rank runs the
same single-GPU step on its own batch (independent replicas, no data-path
collective; weak scaling); time is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from tensor_transformer_layer_linear_b200 import synth  # noqa: E402

DEFAULT_WORKLOAD = "layer_2x2048_h4096_32x128_f16384_n8"
METRIC = "TP-layer fwd TFLOP/s & % BF16 peak (1 B200); partial-reduce GB/s & % HBM"
L2_BYTES = 126 * 1024 * 1024

# DRAM bytes per launch (dram__bytes_read.sum + dram__bytes_write.sum) from the
# committed ncu captures, keyed by (workload, kernel). None
# until a capture of the current kernel exists.
NCU_TRAFFIC = {
    # ncu capture of one layer step: dram__bytes_read.sum + dram__bytes_write.sum per launch;
    # QKV 244.1 MB and MLP-up 316.2 MB -> mean per launch
    (DEFAULT_WORKLOAD, "gemm_column_parallel"): 280.2e6,
    # W_O 540.5 MB and MLP-down 765.1 MB -> mean per launch
    (DEFAULT_WORKLOAD, "gemm_row_parallel"): 652.8e6,
    # persistent attention (three S buffers): 134.1 MB read + 14.2 MB written
    (DEFAULT_WORKLOAD, "attention"): 148.3e6,
    # the reductions and LN1 (profiles/reduce_partials_ncu.md): read + write per launch
    (DEFAULT_WORKLOAD, "reduce_partials"): 574.0e6,
    (DEFAULT_WORKLOAD, "reduce_partials_layernorm"): 591.8e6,
    (DEFAULT_WORKLOAD, "layernorm"): 34.0e6,
    # layer backward: the streamed LN-backward reduction (604.0 MB read + 13.8 MB written)
    (DEFAULT_WORKLOAD, "reduce_partials_layernorm_backward"): 617.8e6,
}


def peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(hbm=float(d["hbm_gbs"]), bf16=float(d["bf16_tflops"]),
                    bf16_sustained=float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                    source="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sustained=1400.0, source="fallback")


# --------------------------------------------------------------------------
# algorithmic work per step (what the method must compute, not what runs)
# --------------------------------------------------------------------------

def work(cfg: dict) -> dict:
    """Per-step algorithmic work by kernel name (as the launch trace names
    the kernels): FLOPs of the contractions, bytes of the HBM-bound kernels
    (per-step totals), and the bytes of one launch of each HBM-bound kernel."""
    M = cfg["batch"] * cfg["seq"]
    h = cfg["h"]
    n = cfg["n_shards"]
    kind = cfg["kind"]
    fl = {"gemm_column_parallel": 0.0, "gemm_row_parallel": 0.0, "attention": 0.0}
    by, launch = {}, {}
    partial_read = n * M * h * 4
    act = M * h * 2

    def hbm(name, nbytes):
        by[name] = by.get(name, 0) + nbytes
        launch[name] = nbytes

    def row_block(K, res, ln_after=False):
        """A block's output projection (K = its per-shard inner size) and its
        one reduction of the N partials (+ bias, + residual when res, + LN
        when ln_after)."""
        fl["gemm_row_parallel"] += 2.0 * M * (K * n) * h
        if ln_after:
            hbm("reduce_partials_layernorm", partial_read + act + 3 * h * 2 + 2 * act)
        else:
            hbm("reduce_partials", partial_read + (act if res else 0) + h * 2 + act)

    if cfg.get("backward"):
        # algorithmic backward work (recomputed forward products are extra):
        # MLP dH, dX, dA, dB; attention block dO, dX, dW_QKV, dW_O and the
        # head gradients dV, dP, dK, dQ (twice the forward attention)
        F = cfg.get("ffn", 0)
        gb, ab = 0.0, 0.0
        att = 0.0
        if kind in ("attn", "layer", "attn_gqa"):
            d = h // cfg["n_heads"]
            att = 4.0 * cfg["seq"] ** 2 * d * cfg["n_heads"] * cfg["batch"] / (
                2 if cfg.get("causal", True) else 1)
        if kind in ("mlp", "layer"):
            gb += 8.0 * M * h * F
        if kind in ("attn", "layer"):
            gb += 16.0 * M * h * h
            ab = 2.0 * att
        if kind == "attn_gqa":
            qkv = (cfg["n_heads"] + 2 * cfg["n_kv_heads"]) * (h // cfg["n_heads"])
            gb += 4.0 * M * h * h + 4.0 * M * qkv * h   # dO, dW_O; dX, dW_QKV
            ab = 2.0 * att
        fl = {"gemm_backward": gb, "attention_backward": ab}
        if kind == "layer":
            # one LN-backward reduction per block (the MLP's through LN2, the
            # attention block's through LN1), each of the same size
            for _ in range(2):
                hbm("reduce_partials_layernorm_backward", n * M * h * 4 + 3 * M * h * 2 + h * 2)
        else:
            hbm("reduce_partials", partial_read + (act if cfg.get("residual") else 0) + act)
        return dict(flops=fl, bytes=by, launch_bytes=launch, total_flops=sum(fl.values()))
    if kind == "layer":
        hbm("layernorm", act + 2 * h * 2 + act)                      # LN1
    if kind in ("attn", "layer"):
        fl["gemm_column_parallel"] += 2.0 * M * h * 3 * h
    if kind == "attn_gqa":
        d = h // cfg["n_heads"]
        fl["gemm_column_parallel"] += 2.0 * M * h * (cfg["n_heads"] + 2 * cfg["n_kv_heads"]) * d
    if kind in ("attn", "layer", "attn_gqa"):
        d = h // cfg["n_heads"]
        fl["attention"] += 4.0 * cfg["seq"] ** 2 * d * cfg["n_heads"] * cfg["batch"] / (
            2 if cfg.get("causal", True) else 1)
        row_block(h // n, res=(kind == "layer" or cfg.get("residual")), ln_after=(kind == "layer"))
    if kind in ("mlp", "layer", "swiglu"):
        F = cfg["ffn"]
        fl["gemm_column_parallel"] += 2.0 * M * h * F * (2 if kind == "swiglu" else 1)
        row_block(F // n, res=(kind == "layer" or cfg.get("residual")))
    fl = {k: v for k, v in fl.items() if v > 0}
    return dict(flops=fl, bytes=by, launch_bytes=launch, total_flops=sum(fl.values()))


# --------------------------------------------------------------------------
# clocks during the timed region
# --------------------------------------------------------------------------

CLOCK_FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")


class ClockSampler:
    def __init__(self, device_index: int):
        self.proc = None
        self.out = []
        try:
            import torch
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            gid = uuid if uuid.startswith("GPU-") else f"GPU-{uuid}"
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", gid, f"--query-gpu={CLOCK_FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self) -> None:
        """End sampling and parse what nvidia-smi printed."""
        self.samples = []
        if self.proc is None:
            return
        self.proc.terminate()
        try:
            text, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            text, _ = self.proc.communicate()
        import datetime
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        samples = []
        for line in text.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 10:
                continue
            try:
                ts = datetime.datetime.strptime(f[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                samples.append((ts, float(f[2]), float(f[3]), float(f[4]) if f[4] else 0.0,
                                [nm for nm, v in zip(names, f[6:10]) if v.lower() == "active"]))
            except ValueError:
                continue
        self.samples = samples

    def window(self, t0: float, t1: float) -> dict:
        """Median SM clock and the throttle reasons seen in samples taken
        between host wall-clock times t0 and t1 (all samples if none are)."""
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        samples = self.samples
        inside = [x for x in samples if t0 <= x[0] <= t1]
        use = inside or samples
        sm = [x[1] for x in use]
        reasons = sorted({r for x in use for r in x[4]})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(x[2] for x in use) if use else None,
                "power_w_max": max(x[3] for x in use) if use else None,
                "reasons": reasons, "samples": len(use),
                "window": "timed region" if inside else "whole run", "source": "nvidia-smi"}


class NvmlSampler:
    """SM clock, power and clock-event reasons read through NVML (read-only
    queries) by a host thread every few milliseconds, so that even a timed
    region of a few tens of milliseconds holds several samples."""

    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"),
               ("hw_power_brake_slowdown", "nvmlClocksEventReasonHwPowerBrakeSlowdown"))

    def __init__(self, device_index: int, period_s: float = 0.004):
        import threading
        import pynvml
        import torch
        self.nv = pynvml
        pynvml.nvmlInit()
        uuid = str(torch.cuda.get_device_properties(device_index).uuid)
        gid = uuid if uuid.startswith("GPU-") else f"GPU-{uuid}"
        self.h = pynvml.nvmlDeviceGetHandleByUUID(gid)
        self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM))
        self.bits = [(nm, getattr(pynvml, attr)) for nm, attr in self.REASONS
                     if hasattr(pynvml, attr)]
        self.samples = []
        self.period = period_s
        self.done = threading.Event()
        self.thread = threading.Thread(target=self._run, daemon=True)
        self.thread.start()

    def _run(self):
        nv, h = self.nv, self.h
        while not self.done.is_set():
            try:
                mhz = float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM))
                mw = float(nv.nvmlDeviceGetPowerUsage(h))
                r = int(nv.nvmlDeviceGetCurrentClocksEventReasons(h))
                self.samples.append((time.time(), mhz, mw / 1000.0,
                                     [nm for nm, b in self.bits if r & b]))
            except Exception:
                pass
            self.done.wait(self.period)

    def window(self, t0: float, t1: float) -> dict:
        """Median SM clock and every reason seen between host times t0 and t1."""
        use = [x for x in self.samples if t0 <= x[0] <= t1]
        where = "timed region"
        if not use:
            use, where = self.samples, "whole run"
        sm = [x[1] for x in use]
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": self.max_mhz,
                "power_w_max": max((x[2] for x in use), default=None),
                "reasons": sorted({r for x in use for r in x[3]}), "samples": len(use),
                "window": where, "source": "nvml"}

    def stop(self) -> None:
        self.done.set()
        self.thread.join(timeout=2)


def clock_sampler(device_index: int):
    """NVML sampler when NVML answers, else the nvidia-smi one."""
    try:
        return NvmlSampler(device_index)
    except Exception:
        return ClockSampler(device_index)


# --------------------------------------------------------------------------
# the CPU oracle as a baseline (test infrastructure; timed, never on the path)
# --------------------------------------------------------------------------

def oracle_sample(cfg: dict, inp: dict, tokens: int):
    """Run the fp64 oracle on the first `tokens` tokens of sequence 0 (a causal
    prefix: its outputs are exactly those rows of the full workload).
    Returns (seconds, algorithmic flops of the sample, threads used)."""
    from threadpoolctl import threadpool_info
    from oracle import tp_oracle as O
    sub = dict(cfg, batch=1, seq=tokens)
    T = tokens
    f64 = synth.bf16_bits_to_f64
    x = f64(inp["X"][:T])
    t0 = time.perf_counter()
    if cfg.get("backward"):
        dY = np.random.default_rng(1).standard_normal(x.shape)
        if cfg["kind"] == "layer":
            p = {k: f64(v) for k, v in inp.items() if k != "X"}
            O.transformer_layer_backward(x, p, dY, 1, T, cfg["n_heads"], cfg["n_shards"],
                                         cfg.get("ln_eps", 1e-5))
        elif cfg["kind"] == "attn_gqa":
            O.gqa_self_attention_backward_sharded(x, f64(inp["Wqkv"]), f64(inp["bqkv"]),
                                                  f64(inp["Wo"]), f64(inp["bo"]), dY, 1, T,
                                                  cfg["n_heads"], cfg["n_kv_heads"],
                                                  cfg["n_shards"], cfg.get("causal", True),
                                                  bool(cfg.get("residual")))
        elif cfg["kind"] == "attn":
            O.self_attention_backward_sharded(x, f64(inp["Wqkv"]), f64(inp["bqkv"]),
                                              f64(inp["Wo"]), f64(inp["bo"]), dY, 1, T,
                                              cfg["n_heads"], cfg["n_shards"],
                                              cfg.get("causal", True), bool(cfg.get("residual")))
        else:
            O.mlp_backward_sharded(x, f64(inp["A"]), f64(inp["b1"]), f64(inp["B"]), dY,
                                   cfg["n_shards"], bool(cfg.get("residual")))
    elif cfg["kind"] == "layer":
        p = {k: f64(v) for k, v in inp.items() if k != "X"}
        O.transformer_layer(x, p, 1, T, cfg["n_heads"], cfg.get("ln_eps", 1e-5))
    elif cfg["kind"] == "attn_gqa":
        R = x if cfg.get("residual") else None
        O.gqa_self_attention(x, f64(inp["Wqkv"]), f64(inp["bqkv"]), f64(inp["Wo"]),
                             f64(inp["bo"]), R, 1, T, cfg["n_heads"], cfg["n_kv_heads"],
                             cfg.get("causal", True))
    elif cfg["kind"] == "swiglu":
        R = x if cfg.get("residual") else None
        O.swiglu_mlp(x, f64(inp["Wg"]), f64(inp["Wu"]), f64(inp["B"]), f64(inp["b2"]), R)
    elif cfg["kind"] == "attn":
        R = x if cfg.get("residual") else None
        O.self_attention(x, f64(inp["Wqkv"]), f64(inp["bqkv"]), f64(inp["Wo"]), f64(inp["bo"]),
                         R, 1, T, cfg["n_heads"], cfg.get("causal", True))
    else:
        R = x if cfg.get("residual") else None
        O.mlp(x, f64(inp["A"]), f64(inp["b1"]), f64(inp["B"]), f64(inp["b2"]), R)
    dt = time.perf_counter() - t0
    threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    return dt, work(sub)["total_flops"], threads


def sample_tokens(cfg: dict) -> int:
    return min(cfg["seq"], 512)


def run_reference(args, cfg) -> None:
    """The reference arm: the fp64 CPU oracle, timed on the host cores."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    inp = synth.make_inputs(cfg)
    T = sample_tokens(cfg)
    times, flops, threads = [], 0.0, 1
    for i in range(args.warmup + args.steps):
        dt, flops, threads = oracle_sample(cfg, inp, T)
        if i >= args.warmup:
            times.append(dt)
    mean = sum(times) / len(times)
    value = flops / mean / 1e12
    sample = (f"first {T} tokens of sequence 0 (causal prefix) of {cfg['name']}, fp64 numpy "
              f"oracle, {flops / 1e9:.1f} GFLOP algorithmic per step")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": mean * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": cfg["name"], "n_shards": cfg["n_shards"], "sample_tokens": T},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# --------------------------------------------------------------------------
# our arm
# --------------------------------------------------------------------------

class Model:
    """Device-resident sharded weights + workspace for one workload."""

    def __init__(self, tp, torch, cfg: dict, inp: dict):
        self.tp, self.torch, self.cfg = tp, torch, cfg
        to_dev = lambda b: torch.from_numpy(np.ascontiguousarray(b).view(np.int16)).cuda()
        dev = {k: to_dev(v) for k, v in inp.items()}
        n, h = cfg["n_shards"], cfg["h"]
        self.M = cfg["batch"] * cfg["seq"]

        def shard(name, h_in, h_out, kind, hd=0):
            out = torch.empty(h_in * h_out, dtype=torch.int16, device="cuda")
            tp.tp_shard_weights(dev[name], h_in, h_out, n, kind, hd, out)
            return out

        self.X = dev["X"]
        kind = cfg["kind"]
        if kind in ("attn", "layer"):
            d = h // cfg["n_heads"]
            self.Wqkv = shard("Wqkv", h, 3 * h, 2, d)
            self.bqkv = shard("bqkv", 1, 3 * h, 2, d)
            self.Wo = shard("Wo", h, h, 1)
            self.bo = dev["bo"]
        if kind in ("mlp", "layer"):
            F = cfg["ffn"]
            self.A = shard("A", h, F, 0)
            self.B = shard("B", F, h, 1)
            self.b1, self.b2 = dev["b1"], dev["b2"]
        if kind == "attn_gqa":
            nq, nkv = cfg["n_heads"], cfg["n_kv_heads"]
            d = h // nq
            kvl = nkv // n if n <= nkv else 1
            cols = (nq // n + 2 * kvl) * d
            self.qkv_cols = n * cols
            self.Wqkv = torch.empty(n * cols * h, dtype=torch.int16, device="cuda")
            tp.tp_shard_qkv_gqa(dev["Wqkv"], h, nq, nkv, d, n, self.Wqkv)
            self.bqkv = torch.empty(n * cols, dtype=torch.int16, device="cuda")
            tp.tp_shard_qkv_gqa(dev["bqkv"], 1, nq, nkv, d, n, self.bqkv)
            self.Wo = shard("Wo", h, h, 1)
            self.bo = dev["bo"]
        if kind == "swiglu":
            F = cfg["ffn"]
            dev["GU"] = torch.cat([dev["Wg"].view(h, F), dev["Wu"].view(h, F)], dim=1).contiguous()
            self.GU = shard("GU", h, 2 * F, 3)
            self.B = shard("B", F, h, 1)
            self.b2 = dev["b2"]
        if kind == "layer":
            self.w = tp.make_layer_weights(
                ln1_gamma=dev["ln1_g"], ln1_beta=dev["ln1_b"], Wqkv_shards=self.Wqkv,
                bqkv_shards=self.bqkv, Wo_shards=self.Wo, bo=self.bo, ln2_gamma=dev["ln2_g"],
                ln2_beta=dev["ln2_b"], A_shards=self.A, b1_shards=self.b1, B_shards=self.B,
                b2=self.b2)
            self.dev_keep = dev
        wsk = {"mlp": tp.TP_WS_MLP, "swiglu": tp.TP_WS_MLP, "attn": tp.TP_WS_ATTN,
               "attn_gqa": tp.TP_WS_ATTN, "layer": tp.TP_WS_LAYER}[kind]
        self.ws_bytes = tp.tp_workspace_bytes(wsk, self.M, h, cfg.get("ffn", 0), n)
        self.ws = torch.empty(self.ws_bytes, dtype=torch.uint8, device="cuda")
        self.Y = torch.empty((self.M, h), dtype=torch.int16, device="cuda")
        if cfg.get("backward"):
            self.setup_backward()
        torch.cuda.synchronize()

    def setup_backward(self):
        """Gradient buffers for the backward step (dY drawn once)."""
        torch, tp, cfg = self.torch, self.tp, self.cfg
        M, h, n, kind = self.M, cfg["h"], cfg["n_shards"], cfg["kind"]
        F = cfg.get("ffn", 0)
        g = torch.Generator(device="cuda").manual_seed(1)
        self.dY = (torch.randn((M, h), device="cuda", generator=g)).to(torch.bfloat16).view(torch.int16)
        self.dX = torch.empty((M, h), dtype=torch.int16, device="cuda")

        def f32(k):
            return torch.empty(k, dtype=torch.float32, device="cuda")
        if kind == "mlp":
            self.dA, self.dB, self.db1, self.db2 = f32(h * F), f32(h * F), f32(F), f32(h)
            wsk = tp.TP_WS_MLP_BWD
        elif kind == "attn_gqa":
            self.dWqkv, self.dbqkv = f32(self.qkv_cols * h), f32(self.qkv_cols)
            self.dWo, self.dbo = f32(h * h), f32(h)
            wsk = tp.TP_WS_ATTN_BWD
        elif kind == "attn":
            self.dWqkv, self.dbqkv, self.dWo, self.dbo = f32(3 * h * h), f32(3 * h), f32(h * h), f32(h)
            wsk = tp.TP_WS_ATTN_BWD
        else:
            sizes = dict(ln1_gamma=h, ln1_beta=h, Wqkv_shards=3 * h * h, bqkv_shards=3 * h,
                         Wo_shards=h * h, bo=h, ln2_gamma=h, ln2_beta=h, A_shards=h * F,
                         b1_shards=F, B_shards=F * h, b2=h)
            self.grad_keep = {k: f32(v) for k, v in sizes.items()}
            self.grads = tp.make_layer_grads(**self.grad_keep)
            wsk = tp.TP_WS_LAYER_BWD
        self.ws_bwd_bytes = tp.tp_workspace_bytes(wsk, M, h, F, n)
        self.ws_bwd = torch.empty(self.ws_bwd_bytes, dtype=torch.uint8, device="cuda")

    def step(self, X=None, Y=None):
        tp, cfg = self.tp, self.cfg
        if cfg.get("backward"):
            X = self.X if X is None else X
            dX = self.dX if Y is None else Y
            n, h, kind = cfg["n_shards"], cfg["h"], cfg["kind"]
            if kind == "mlp":
                tp.tp_mlp_backward(X, self.M, h, cfg["ffn"], n, self.A, self.b1, self.B, self.dY,
                                   cfg.get("residual", False), self.ws_bwd, self.ws_bwd_bytes, dX,
                                   self.dA, self.db1, self.dB, self.db2)
            elif kind == "attn_gqa":
                tp.tp_attn_backward_gqa(X, cfg["batch"], cfg["seq"], h, cfg["n_heads"],
                                        cfg["n_kv_heads"], cfg.get("causal", True), n, self.Wqkv,
                                        self.bqkv, self.Wo, self.dY, cfg.get("residual", False),
                                        self.ws_bwd, self.ws_bwd_bytes, dX, self.dWqkv,
                                        self.dbqkv, self.dWo, self.dbo)
            elif kind == "attn":
                tp.tp_attn_backward(X, cfg["batch"], cfg["seq"], h, cfg["n_heads"],
                                    cfg.get("causal", True), n, self.Wqkv, self.bqkv, self.Wo,
                                    self.dY, cfg.get("residual", False), self.ws_bwd,
                                    self.ws_bwd_bytes, dX, self.dWqkv, self.dbqkv, self.dWo,
                                    self.dbo)
            else:
                tp.tp_layer_backward(X, cfg["batch"], cfg["seq"], h, cfg["n_heads"], cfg["ffn"],
                                     n, self.w, cfg.get("ln_eps", 1e-5), self.dY, self.ws_bwd,
                                     self.ws_bwd_bytes, dX, self.grads)
            return
        X = self.X if X is None else X
        Y = self.Y if Y is None else Y
        n, h = cfg["n_shards"], cfg["h"]
        if cfg["kind"] == "layer" and cfg.get("sequence_parallel"):
            # X and Y hold the N sequence slices [N][b][S/N][h]
            tp.tp_layer_forward_sp(X, cfg["batch"], cfg["seq"], h, cfg["n_heads"], cfg["ffn"], n,
                                   self.w, cfg.get("ln_eps", 1e-5), self.ws, self.ws_bytes, Y)
        elif cfg["kind"] == "layer":
            tp.tp_layer_forward(X, cfg["batch"], cfg["seq"], h, cfg["n_heads"], cfg["ffn"], n,
                                self.w, cfg.get("ln_eps", 1e-5), self.ws, self.ws_bytes, Y)
        elif cfg["kind"] == "attn_gqa":
            tp.tp_attn_forward_gqa(X, cfg["batch"], cfg["seq"], h, cfg["n_heads"],
                                   cfg["n_kv_heads"], cfg.get("causal", True), n, self.Wqkv,
                                   self.bqkv, self.Wo, self.bo,
                                   X if cfg.get("residual") else None, self.ws, self.ws_bytes, Y)
        elif cfg["kind"] == "swiglu":
            tp.tp_mlp_forward_swiglu(X, self.M, h, cfg["ffn"], n, self.GU, self.B, self.b2,
                                     X if cfg.get("residual") else None, self.ws, self.ws_bytes,
                                     Y)
        elif cfg["kind"] == "attn":
            tp.tp_attn_forward(X, cfg["batch"], cfg["seq"], h, cfg["n_heads"],
                               cfg.get("causal", True), n, self.Wqkv, self.bqkv, self.Wo,
                               self.bo, X if cfg.get("residual") else None, self.ws,
                               self.ws_bytes, Y)
        else:
            tp.tp_mlp_forward(X, self.M, h, cfg["ffn"], n, self.A, self.b1, self.B, self.b2,
                              X if cfg.get("residual") else None, self.ws, self.ws_bytes, Y)


def max_over_ranks(x: float, dist, device) -> float:
    """The largest x over all ranks, returned on every rank (x itself
    without a process group): a step time is the slowest rank's."""
    if dist is None:
        return x
    import torch
    t = torch.tensor([x], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_tflops(flops_per_rank: float, world: int, ms: float) -> float:
    """Weak scaling: every rank runs its own replica of the workload, so the
    job's throughput is all ranks' work over the slowest rank's time."""
    return flops_per_rank * world / (ms * 1e-3) / 1e12


def l2_cold_kernels(tp, torch, model, cfg, w, pk, reps: int = 20) -> dict:
    """The HBM-bound kernels of the step timed one launch at a time with the
    L2 emptied first (a read of a buffer twice the L2 size, which leaves the
    L2 holding clean lines of that buffer only), so that every input byte
    comes from HBM: median device time over `reps` launches (CUDA events on
    the launching stream), algorithmic bytes / time against the measured
    copy bandwidth. Inputs are the step's own shapes; the partials hold
    arbitrary values."""
    n, h, M = cfg["n_shards"], cfg["h"], model.M
    stream = torch.cuda.current_stream()
    flush = torch.ones(2 * L2_BYTES // 4, dtype=torch.float32, device="cuda")
    P = torch.randn((n, M, h), dtype=torch.float32, device="cuda")
    Y = torch.empty((M, h), dtype=torch.int16, device="cuda")
    Y2 = torch.empty((M, h), dtype=torch.int16, device="cuda")
    res = model.X if (cfg["kind"] == "layer" or cfg.get("residual")) else None
    bias = model.b2 if hasattr(model, "b2") else getattr(model, "bo", None)
    runs = {"reduce_partials": lambda: tp.tp_reduce_partials(P, n, M, h, bias, res, Y)}
    if cfg["kind"] == "layer":
        g = model.w._tensors
        eps = cfg.get("ln_eps", 1e-5)
        runs["reduce_partials_layernorm"] = lambda: tp.tp_reduce_partials_layernorm(
            P, n, M, h, model.bo, model.X, g["ln2_gamma"], g["ln2_beta"], eps, Y, Y2)
        runs["layernorm"] = lambda: tp.tp_layernorm(model.X, M, h, g["ln1_gamma"],
                                                    g["ln1_beta"], eps, Y)
    out = {}
    # one launch's bytes of each kernel (whether or not the step itself runs it)
    act = M * h * 2
    one = {"reduce_partials": n * M * h * 4 + (act if res is not None else 0) + h * 2 + act,
           "reduce_partials_layernorm": n * M * h * 4 + act + 3 * h * 2 + 2 * act,
           "layernorm": act + 2 * h * 2 + act}
    for name, fn in runs.items():
        fn()
        times = []
        for _ in range(reps):
            flush.sum()
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            b.synchronize()
            times.append(a.elapsed_time(b))
        t = statistics.median(times)
        gbs = one[name] / (t * 1e-3) / 1e9
        out[name] = {"ms": t, "achieved": gbs, "unit": "GB/s", "peak": pk["hbm"],
                     "frac": gbs / pk["hbm"], "bytes": one[name], "reps": reps,
                     "flush": "read of a 2 x L2 buffer before each launch"}
    del flush, P
    torch.cuda.empty_cache()
    if tp.tp_get_last_error() != tp.TP_OK:
        raise RuntimeError("device error in the L2-cold kernel timings")
    return out


def run_ours(args, cfg) -> None:
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))

    from tensor_transformer_layer_linear_b200 import tp

    pk = peaks()
    inp = synth.make_inputs(cfg, seed=rank)
    model = Model(tp, torch, cfg, inp)
    w = work(cfg)

    def barrier():
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()

    for _ in range(args.warmup):
        model.step()
    assert tp.tp_get_last_error() == tp.TP_OK
    barrier()

    # device-timed region (inputs resident in HBM); an event after every step
    # gives the per-step times whose median is reported beside the mean
    stream = torch.cuda.current_stream()
    sampler = clock_sampler(local)
    time.sleep(0.3)
    step_ev = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    tp.tp_trace_begin(64 * args.steps)
    barrier()
    t_wall0 = time.time()
    step_ev[0].record(stream)
    for i in range(args.steps):
        model.step()
        step_ev[i + 1].record(stream)
    barrier()
    t_wall1 = time.time()
    recs, launches = tp.tp_trace_end()
    ms = step_ev[0].elapsed_time(step_ev[-1]) / args.steps
    median_ms = statistics.median(step_ev[i].elapsed_time(step_ev[i + 1])
                                  for i in range(args.steps))
    st = tp.tp_get_last_error()
    if st != tp.TP_OK:
        raise RuntimeError(f"device error during the timed region: {tp.tp_status_string(st)}")
    ms = max_over_ranks(ms, dist, "cuda")
    median_ms = max_over_ranks(median_ms, dist, "cuda")

    # sustained window: the same step back to back for about --sustained-s
    # seconds, long enough for the 1 kW power cap to settle the clocks
    sustained = None
    if args.sustained_s > 0:
        n_sus = max(50, int(args.sustained_s * 1e3 / ms))
        sa = torch.cuda.Event(enable_timing=True)
        sb = torch.cuda.Event(enable_timing=True)
        barrier()
        t_s0 = time.time()
        sa.record(stream)
        for _ in range(n_sus):
            model.step()
        sb.record(stream)
        barrier()
        t_s1 = time.time()
        ms_s = max_over_ranks(sa.elapsed_time(sb) / n_sus, dist, "cuda")
        sustained = {"steps": n_sus, "ms_per_step": ms_s, "window": (t_s0, t_s1)}
    if tp.tp_get_last_error() != tp.TP_OK:
        raise RuntimeError("device error during the sustained window")

    # end-to-end through the public API with host buffers: every step copies
    # its own input (X and, for a backward step, dY) from pinned host memory
    # and its result (Y or dX) back. The copies run on their own streams into
    # and out of double-buffered device tensors, so step i + 1's input and
    # step i - 1's result cross PCIe while step i computes (events order each
    # buffer's reuse); the timed region runs from before the first input copy
    # to after the last result copy.
    M, h = model.M, cfg["h"]
    bwd = bool(cfg.get("backward"))
    Xh = torch.from_numpy(inp["X"].view(np.int16)).pin_memory()
    Yh = torch.empty((M, h), dtype=torch.int16).pin_memory()
    Xd = [torch.empty_like(model.X) for _ in range(2)]
    Yd = [torch.empty_like(model.Y) for _ in range(2)]
    dYh = model.dY.cpu().pin_memory() if bwd else None
    dYd = [torch.empty_like(model.dY) for _ in range(2)] if bwd else None
    dY_keep = model.dY if bwd else None
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev = lambda: [torch.cuda.Event() for _ in range(2)]
    ev_in, ev_comp, ev_out = ev(), ev(), ev()

    def e2e_run(n_steps, start_event):
        s_in.wait_event(start_event)
        for i in range(n_steps):
            b = i & 1
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(ev_comp[b])      # step i - 2 has read buffer b
                Xd[b].copy_(Xh, non_blocking=True)
                if bwd:
                    dYd[b].copy_(dYh, non_blocking=True)
                ev_in[b].record(s_in)
            stream.wait_event(ev_in[b])
            if i >= 2:
                stream.wait_event(ev_out[b])         # step i - 2's result has left Yd[b]
            if bwd:
                model.dY = dYd[b]
            model.step(Xd[b], Yd[b])
            ev_comp[b].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_comp[b])
                Yh.copy_(Yd[b], non_blocking=True)
                ev_out[b].record(s_out)
        stream.wait_event(ev_out[(n_steps - 1) & 1])
    e_start = torch.cuda.Event()
    e_start.record(stream)
    e2e_run(2, e_start)
    barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    e2e_run(args.steps, e0)
    e1.record(stream)
    barrier()
    if bwd:
        model.dY = dY_keep
    e2e_ms = e0.elapsed_time(e1) / args.steps
    e2e_ms = max_over_ranks(e2e_ms, dist, "cuda")

    l2_cold = l2_cold_kernels(tp, torch, model, cfg, w, pk) if not bwd else None
    sampler.stop()
    clocks = sampler.window(t_wall0, t_wall1)
    clocks["kcycles_per_step"] = (ms * clocks["sm_mhz"]) if clocks.get("sm_mhz") else None
    if sustained is not None:
        t_s0, t_s1 = sustained.pop("window")
        c = sampler.window(t_s0, t_s1)
        sustained.update(
            value=whole_job_tflops(w["total_flops"], world, sustained["ms_per_step"]),
            unit="TFLOP/s", clocks=c,
            kcycles_per_step=(sustained["ms_per_step"] * c["sm_mhz"]) if c.get("sm_mhz") else None)

    # per-kernel figures from the trace of the timed region
    per = {}
    for name, kms in recs:
        a = per.setdefault(name, [0, 0.0])
        a[0] += 1
        a[1] += kms
    total_k = sum(v[1] for v in per.values())
    dom = max(per, key=lambda k: per[k][1])
    steps_traced = args.steps

    def kernel_fig(name):
        n_l, t_ms = per[name]
        base = dict(launches=n_l, avg_launch_ms=t_ms / n_l, share=t_ms / total_k,
                    traffic=NCU_TRAFFIC.get((cfg["name"], name)))
        if w["flops"].get(name, 0) > 0:
            units = w["flops"][name] * steps_traced
            achieved = units / (t_ms * 1e-3) / 1e12
            return dict(bound="tensor", achieved=achieved, peak=pk["bf16"], unit="TFLOP/s",
                        frac=achieved / pk["bf16"], **base)
        if name in w["bytes"]:
            units = w["bytes"][name] * steps_traced
            achieved = units / (t_ms * 1e-3) / 1e9
            return dict(bound="hbm", achieved=achieved, peak=pk["hbm"], unit="GB/s",
                        frac=achieved / pk["hbm"], **base)
        return dict(bound="other", achieved=None, peak=None, unit=None, frac=None, **base)

    roof = kernel_fig(dom)
    roof["kernel"] = dom
    roof["peak_source"] = f"{pk['source']} (burst bf16 {pk['bf16']} TFLOP/s, HBM {pk['hbm']} GB/s)"
    kernels = {k: kernel_fig(k) for k in per}
    # launches of one step in order, with their mean device time over the timed steps
    per_step = len(recs) // args.steps if args.steps else 0
    step_breakdown = []
    if per_step and len(recs) == per_step * args.steps:
        for pos in range(per_step):
            times = [recs[s * per_step + pos][1] for s in range(args.steps)]
            step_breakdown.append([recs[pos][0], round(sum(times) / len(times), 5)])
    reduce_fig = kernels.get("reduce_partials") or kernels.get("reduce_partials_layernorm_backward")

    value = whole_job_tflops(w["total_flops"], world, ms)
    e2e_value = whole_job_tflops(w["total_flops"], world, e2e_ms)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        T = sample_tokens(cfg)
        dt, fl, threads = oracle_sample(cfg, inp, T)
        cpu = {"value": fl / dt / 1e12, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
               "sample": f"first {T} tokens of sequence 0 (causal prefix) of {cfg['name']}, "
                         f"fp64 numpy oracle, {fl / 1e9:.1f} GFLOP in {dt:.2f} s"}

    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": cfg["name"] + ("+sequence_parallel" if cfg.get("sequence_parallel")
                                              else "") + ("+backward" if cfg.get("backward") else ""),
                   "tokens": M, "h": h, "n_shards": cfg["n_shards"],
                   "heads": cfg.get("n_heads"), "ffn": cfg.get("ffn"),
                   "l2": "inputs larger than L2 (per-step working set "
                         f"{(w['bytes'].get('reduce_partials', 0) + 4 * h * h * 2) / 1e6:.0f}+ MB "
                         "vs 126 MB L2), no flush",
                   "parallelism": f"{cfg['n_shards']} tensor-parallel shards on one GPU"
                                  + (f", {world} independent replicas" if world > 1 else "")},
        "roofline": roof,
        "partial_reduce": reduce_fig,
        "kernels": kernels,
        "cpu_baseline": cpu,
        "e2e": {"value": e2e_value, "unit": "TFLOP/s",
                "h2d_bytes_per_step": M * h * 2 * (2 if bwd else 1),
                "d2h_bytes_per_step": M * h * 2, "ms_per_step": e2e_ms,
                "copies": "own streams, double-buffered, overlapping the neighbouring steps"},
        "clocks": clocks,
        "median_ms_per_step": median_ms,
        "sustained": sustained,
        "partial_reduce_l2_cold": l2_cold,
        "gpu_launches": launches,
        "gflop_per_step": w["total_flops"] / 1e9,
        "step_breakdown_ms": step_breakdown,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


def run_sweep(args, cfg) -> None:
    """Shard-count sweep of one MLP workload (the large-MLP sweep by default):
    the same inputs run with N = 1, 2, 4, 8, 16 shards; reports TFLOP/s per N
    and the N-overhead t(N) / t(1) - 1 (one JSON line)."""
    import torch
    from tensor_transformer_layer_linear_b200 import tp
    torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
    inp = synth.make_inputs(cfg)
    res = {}
    pk = peaks()
    for n in cfg.get("sweep", (1, 2, 4, 8, 16)):
        c = dict(cfg, n_shards=n)
        model = Model(tp, torch, c, inp)
        for _ in range(args.warmup):
            model.step()
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        tp.tp_trace_begin(8 * args.steps)
        e0.record()
        for _ in range(args.steps):
            model.step()
        e1.record()
        torch.cuda.synchronize()
        recs, _ = tp.tp_trace_end()
        assert tp.tp_get_last_error() == tp.TP_OK
        ms = e0.elapsed_time(e1) / args.steps
        kern = {}
        for name, kms in recs:
            kern[name] = kern.get(name, 0.0) + kms / args.steps
        w = work(c)
        red_bytes = w["bytes"].get("reduce_partials", 0)
        res[n] = {"ms_per_step": ms, "tflops": w["total_flops"] / ms / 1e9,
                  "frac_of_bf16_peak": w["total_flops"] / ms / 1e9 / pk["bf16"],
                  "kernel_ms": {k: round(v, 4) for k, v in kern.items()},
                  "reduce_gbs": red_bytes / (kern["reduce_partials"] * 1e-3) / 1e9}
        del model
        torch.cuda.empty_cache()
    t1 = res[min(res)]["ms_per_step"]
    for n in res:
        res[n]["overhead_vs_n1"] = res[n]["ms_per_step"] / t1 - 1.0
    line = {"metric": "large-MLP shard sweep: TFLOP/s and N-overhead", "unit": "TFLOP/s",
            "value": res[max(res)]["tflops"], "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "higher_is_better": True, "dtype": "bf16",
            "data": "synthetic", "config": {"workload": cfg["name"]},
            "sweep": {str(k): v for k, v in res.items()}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--sustained-s", type=float, default=3.0,
                    help="seconds of back-to-back steps timed after the main region (0: skip)")
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(synth.CONFIGS))
    ap.add_argument("--shards", type=int, default=0, help="override the shard count N")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--sequence-parallel", action="store_true",
                    help="layer workload: run tp_layer_forward_sp on sequence-sharded input")
    ap.add_argument("--backward", action="store_true",
                    help="MLP, attention and layer workloads: time the backward pass "
                         "(tp_mlp_backward / tp_attn_backward / tp_layer_backward)")
    ap.add_argument("--sweep", action="store_true",
                    help="run the workload at every shard count of its sweep (one JSON line)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    cfg = synth.config(args.workload)
    if args.shards:
        cfg["n_shards"] = args.shards
    if args.backward:
        if cfg["kind"] not in ("mlp", "attn", "attn_gqa", "layer"):
            ap.error("--backward applies to the MLP, attention, GQA and layer workloads")
        cfg["backward"] = True
    if args.sequence_parallel:
        if cfg["kind"] != "layer":
            ap.error("--sequence-parallel applies to the layer workload")
        cfg["sequence_parallel"] = True
    if args.sweep:
        run_sweep(args, cfg)
    elif args.impl == "reference":
        run_reference(args, cfg)
    else:
        run_ours(args, cfg)


if __name__ == "__main__":
    main()
