#!/usr/bin/env python
"""Benchmark of the packed-THD sliding-window GQA attention forward on B200.

One step = one forward (thd_attn_fwd through the C ABI) over one synthetic
pack.  Default workload: the 65,536-token pack (log-uniform document lengths
in [1024, 32768], Hq=64, Hkv=8, D=128, full causal, learned sinks).  Metric:
TFLOP/s over valid (unmasked) query-key pairs, FLOP = 4 * pairs * D * Hq.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

The default run prints one JSON line whose headline (`value`) is that pack's
forward, and which also carries, measured in the same run with the same
steps and warm-up:
  per_config  the forward on the other benchmark packs (8,192-token causal,
              32,768-token window 4096, 131,072-token MQA document at D = 256)
  passes      the backward (thd_attn_bwd: dq, dk, dv, dsink; FLOP = 2.5x the
              forward's, the usual count of a backward that recomputes P) on
              the 64k pack and on the 128k document, the in-place Q/K prologue
              (thd_qk_norm_rope; bytes = Q and K read and written once), and
              sparse MLA (thd_sparse_mla_fwd) on its own synthetic workload
              (4,096 tokens, 128 heads, up to 2,048 selected keys, value dim
              128; FLOP = valid slots x heads x 2 x (576 + 512) + the value
              projection).
``--no-extras`` leaves those out.  ``--pass bwd|prologue|sparse_mla`` prints
one line for that pass alone (``--workload`` selects the pack).

Multi-GPU runs are launched with torchrun, one process per GPU; every rank
runs its own pack of the same shape (no data-path collective; "weak"), or,
with ``--shard heads``, its kv-head groups of one pack (cp.head_shard; no
collective either; "strong"), or, with ``--shard tokens``, its token shard of
one pack (cp.cp_attention_fwd_overlapped: the K/V all-gather over NCCL under
the own-slice part; "strong").  The timed region is bracketed by a barrier
and a device synchronisation, and the time is the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from sliding_window_gqa_cu_b200 import metrics, multirank, workloads  # noqa: E402

DEFAULT_WORKLOAD = "pack64k_gqa8_d128_causal_sink"
METRIC = "THD varlen attention fwd TFLOP/s (valid pairs) and % of B200 BF16 peak"
UNIT = "TFLOP/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
DATASHEET_BF16_TFLOPS = 2250.0


def kernel_name(D: int, group: int) -> str:
    """The kernel the library launches for this shape (label only): the
    CTA-pair kernel with the key-split softmax at head dim 256 with an even
    GQA group, else the one-CTA kernel."""
    return "thd_attn_fwd_split_kernel" if D == 256 and group % 2 == 0 else "thd_attn_fwd_kernel"


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=workloads.CONFIG_ORDER)
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--tokens", type=int, default=None,
                    help="truncate the pack to its first N tokens (small profiling cases)")
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="target CPU time of the oracle baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--pass", dest="pass_", choices=["fwd", "bwd", "prologue", "sparse_mla"],
                    default="fwd", help="what one step runs (default: the forward, the headline)")
    ap.add_argument("--no-extras", action="store_true",
                    help="headline only: leave out per_config and passes")
    ap.add_argument("--shard", choices=["packs", "heads", "tokens"], default="packs",
                    help="multi-GPU form: every rank its own pack (weak scaling, default), "
                         "every rank its kv-head groups of one pack (strong scaling, no collective) "
                         "or its token shard of one pack (context parallel, overlapped K/V all-gather)")
    return ap.parse_args(argv)


# ------------------------------------------------------------------ helpers --

def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


# Sources that decide the forward kernels' DRAM traffic: the kernels and the
# schedule (item order).  Host-only entry-point code is not part of it.
E2E_CHUNKS = 16  # token ranges of the end-to-end call (copies overlap the attention)

TRAFFIC_SOURCES = ("sm100_ptx.cuh", "thd_attn_kernel.cuh", "thd_attn_split_kernel.cuh",
                   "scheduler.cpp", "scheduler.h")


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "sliding_window_gqa_cu_b200", "csrc")
    for name in TRAFFIC_SOURCES:
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + b"\0" + f.read())
    return h.hexdigest()[:16]


def traffic_per_launch(workload: str):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current kernel source (else None)."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
    except (OSError, ValueError):
        return None
    e = d.get(workload)
    if not e or e.get("kernel_source_hash") != kernel_source_hash():
        return None
    return e.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples taken during the timed region."""

    FIELDS = ["clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.hw_slowdown",
              "clocks_event_reasons.hw_thermal_slowdown", "clocks_event_reasons.sw_thermal_slowdown",
              "clocks_event_reasons.sw_power_cap"]
    REASONS = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, device: torch.device):
        self.samples = []  # (host time, fields)
        self.proc = None
        self.error = None
        try:
            uuid = "GPU-" + str(torch.cuda.get_device_properties(device).uuid)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", uuid, "--query-gpu=" + ",".join(self.FIELDS),
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
            t0 = time.time()
            while not self.samples and time.time() - t0 < 10 and self.proc.poll() is None:
                time.sleep(0.05)
        except Exception as e:  # no nvidia-smi
            self.error = str(e)
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) == len(self.FIELDS):
                self.samples.append((time.time(), parts))

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self, t0: float, t1: float):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "error": self.error}
        win = [p for (t, p) in self.samples if t0 <= t <= t1] or [p for (_, p) in self.samples[-3:]]
        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = [num(p[0]) for p in win if num(p[0]) is not None]
        mx = [num(p[1]) for p in win if num(p[1]) is not None]
        pw = [num(p[2]) for p in win if num(p[2]) is not None]
        reasons = sorted({r for p in win for r, v in zip(self.REASONS, p[3:]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(win),
                "power_w_max": max(pw) if pw else None}


# ------------------------------------------------------------ CPU baseline --

def cpu_oracle_sample(pack, target_seconds: float, seed: int, max_rows: int = 1 << 20):
    """Time the fp64 CPU oracle on random (token, head) rows of the pack until
    about `target_seconds` of work is done.  Returns (TFLOP/s, seconds, rows,
    flops, threads)."""
    import oracle  # test infrastructure: only the CPU-baseline leg uses it
    cfg = pack["config"]
    T, Hq, D = pack["T"], cfg.Hq, cfg.D
    rng = np.random.default_rng(seed)
    lib = oracle.load()
    done_rows, flops, spent = 0, 0, 0.0
    batch = 64
    while spent < target_seconds and done_rows < max_rows:
        rows = np.stack([rng.integers(0, T, size=batch), rng.integers(0, Hq, size=batch)], axis=1)
        t0 = time.perf_counter()
        oracle.attention_rows(pack["q"], pack["k"], pack["v"], pack["cu_seqlens"], cfg.window,
                              cfg.scale, rows, pack["sinks"], lib=lib)
        spent += time.perf_counter() - t0
        flops += metrics.row_flops(metrics.visible_keys(pack["cu_seqlens"], cfg.window, rows[:, 0]), D)
        done_rows += batch
        if spent < target_seconds / 8:
            batch *= 2
    return flops / spent / 1e12, spent, done_rows, flops, oracle.num_threads(lib)


def workload_config(cfg, cu, pairs, extra=None):
    d = {"workload": cfg.name, "tokens": int(cu[-1]), "documents": int(len(cu) - 1),
         "Hq": cfg.Hq, "Hkv": cfg.Hkv, "head_dim": cfg.D, "window": cfg.window,
         "sinks": cfg.sinks, "valid_pairs": int(pairs), "seed": 0,
         "l2": "inputs larger than L2 (Q+K+V = %.2f GB > 126 MB), no flush"
               % (int(cu[-1]) * (cfg.Hq + 2 * cfg.Hkv) * cfg.D * 2 / 1e9)}
    if extra:
        d.update(extra)
    return d


# ----------------------------------------------------------- reference arm --

def run_reference(args, info):
    """The fp64 CPU oracle timed as the reference arm (rank 0 only)."""
    if not info.is_root:
        return 0
    cfg = workloads.CONFIGS[args.workload]
    pack = workloads.make_pack(cfg, args.seed, T_override=args.tokens)
    cu = pack["cu_seqlens"]
    pairs = metrics.valid_pairs(cu, cfg.window)
    # size one step to about 2 s of CPU work so the whole run stays within minutes
    per_step = max(0.25, min(2.0, 150.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        cpu_oracle_sample(pack, per_step, seed=1000 + _)
    tot_flops, tot_s, tot_rows, threads = 0, 0.0, 0, 1
    for s in range(args.steps):
        _, spent, rows, flops, threads = cpu_oracle_sample(pack, per_step, seed=s)
        tot_flops += flops
        tot_s += spent
        tot_rows += rows
    value = tot_flops / tot_s / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": tot_s / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        # the same config object as the GPU arm's line for this workload
        "config": workload_config(cfg, cu, pairs, {"parallelism": f"pack-parallel x{info.world}",
                                                   "per_rank_tflop": 4 * pairs * cfg.D * cfg.Hq / 1e12}),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": f"{tot_rows} random (token, head) rows of the pack over "
                                   f"{args.steps} steps (~{per_step:.2f} s each)"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ GPU arm --

EXTRA_CONFIGS = ("pack8k_gqa4_d128_causal", "pack32k_gqa4_d128_w4096", "doc128k_mqa_d256_w8192_sink")
BWD_WORKLOADS = ("pack64k_gqa8_d128_causal_sink", "doc128k_mqa_d256_w8192_sink")


def timed_loop(step, args, device, stream, label):
    """W untimed steps, then K steps between a barrier and a device
    synchronisation on both sides, with a CUDA event pair around every step
    on the launching stream.  Returns (max-over-ranks ms of the K steps,
    max-over-ranks mean ms per step, host start, host end)."""
    for _ in range(args.warmup):
        step()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    multirank.barrier(device)
    torch.cuda.synchronize(device)
    h0 = time.time()
    torch.cuda.nvtx.range_push(label)
    start.record(stream)
    for i in range(args.steps):
        ev[i][0].record(stream)
        step()
        ev[i][1].record(stream)
    end.record(stream)
    torch.cuda.nvtx.range_pop()
    torch.cuda.synchronize(device)
    h1 = time.time()
    multirank.barrier(device)
    total = multirank.max_over_ranks(start.elapsed_time(end), device)
    per = multirank.max_over_ranks(statistics.mean(a.elapsed_time(b) for a, b in ev), device)
    return total, per, h0, h1


def check_status(swa, stream, what):
    status = swa.thd_attn_get_error(stream)
    if status != 0:
        raise RuntimeError(f"{what}: kernel reported status {status}")


def fwd_case(swa, cfg, args, info, device, stream, T_override=None):
    """Device tensors of one pack and a step that runs its forward.  With
    ``--shard heads`` every rank holds the same pack and keeps only its head
    slice (cp.head_shard): q/k/v/sinks/out/lse have the slice's head counts."""
    heads = getattr(args, "shard", "packs") == "heads"
    tokens = getattr(args, "shard", "packs") == "tokens"
    seed = args.seed if heads or tokens else multirank.tensor_seed(args.seed, info.rank)
    pack = workloads.make_pack(cfg, args.seed, tensor_seed=seed, T_override=T_override)
    cu = pack["cu_seqlens"]
    if heads:
        from sliding_window_gqa_cu_b200 import cp
        q_lo, q_hi, kv_lo, kv_hi = cp.head_shard(cfg.Hq, cfg.Hkv, info.world, info.rank)
        pack["q"] = pack["q"][:, q_lo:q_hi].contiguous()
        pack["k"] = pack["k"][:, kv_lo:kv_hi].contiguous()
        pack["v"] = pack["v"][:, kv_lo:kv_hi].contiguous()
        if pack["sinks"] is not None:
            pack["sinks"] = pack["sinks"][q_lo:q_hi].contiguous()
    Hq_r = pack["q"].shape[1]
    q, k, v = (pack[n].to(device) for n in "qkv")
    sinks = pack["sinks"].to(device) if pack["sinks"] is not None else None
    T = pack["T"]
    out = torch.empty((T, Hq_r, cfg.D), dtype=torch.bfloat16, device=device)
    lse = torch.empty((T, Hq_r), dtype=torch.float32, device=device)

    if tokens:
        from sliding_window_gqa_cu_b200 import cp
        b, e = cp.shard_bounds(T, info.world)[info.rank]
        ql, kl, vl = q[b:e].contiguous(), k[b:e].contiguous(), v[b:e].contiguous()

        def step():
            cp.cp_attention_fwd_overlapped(ql, kl, vl, cu, cfg.window, cfg.scale, sinks)
        # this rank's launches per step: the own-slice forward, plus the
        # key-bounded range and the merge when a document crosses its start
        step.launches = 1 + (2 if cp.crossing_rows(cu, b, e) > b else 0)
        return pack, dict(q=q, k=k, v=v, sinks=sinks, out=out, lse=lse), step

    def step():
        swa.thd_attn_fwd(q, k, v, cu, cfg.window, cfg.scale, sinks, out=out, lse=lse, stream=stream)
    step.launches = 1
    return pack, dict(q=q, k=k, v=v, sinks=sinks, out=out, lse=lse), step


def summarise(ms_total, per_ms, args, work, unit, peak, peaks, clocks_sum, kernel, extra=None):
    scale = 1e12 if unit == "TFLOP/s" else 1e9
    achieved = work / (per_ms / 1e3) / scale
    d = {"ms_per_step": ms_total / args.steps, "value": work * args.steps / (ms_total / 1e3) / scale,
         "unit": unit, "frac": achieved / peak, "peak": peak, "kernel": kernel,
         "clocks": {k: clocks_sum.get(k) for k in ("sm_mhz", "sm_max_mhz", "reasons")}}
    if unit == "TFLOP/s":
        d["frac_of_sustained"] = achieved / float(peaks.get("bf16_tflops_sustained", peak))
    if extra:
        d.update(extra)
    return d


def measure_fwd_extra(swa, name, args, info, device, stream, clocks, peaks):
    cfg = workloads.CONFIGS[name]
    pack, _, step = fwd_case(swa, cfg, args, info, device, stream)
    pairs = metrics.valid_pairs(pack["cu_seqlens"], cfg.window)
    flops = 4 * pairs * cfg.D * cfg.Hq
    step()
    check_status(swa, stream, name)
    tot, per, h0, h1 = timed_loop(step, args, device, stream, f"thd_attn_fwd {name}")
    check_status(swa, stream, name)
    peak = float(peaks["bf16_tflops"])
    return summarise(tot, per, args, flops * info.world, UNIT, peak * info.world, peaks,
                     clocks.summary(h0, h1), kernel_name(cfg.D, cfg.Hq // cfg.Hkv),
                     {"valid_pairs": int(pairs), "tokens": pack["T"], "gflop_per_step": flops / 1e9,
                      "traffic": traffic_per_launch(name)})


def measure_bwd(swa, name, args, info, device, stream, clocks, peaks):
    cfg = workloads.CONFIGS[name]
    pack, t, _ = fwd_case(swa, cfg, args, info, device, stream, T_override=args.tokens)
    cu, T = pack["cu_seqlens"], pack["T"]
    pairs = metrics.valid_pairs(cu, cfg.window)
    out, lse = swa.thd_attn_fwd(t["q"], t["k"], t["v"], cu, cfg.window, cfg.scale, t["sinks"],
                                stream=stream)
    g = torch.Generator(device="cpu").manual_seed(7)
    dout = torch.randn((T, cfg.Hq, cfg.D), generator=g).to(torch.bfloat16).to(device)
    ws = torch.empty((max(16, swa.thd_attn_bwd_workspace_bytes(T, cfg.Hq)),), dtype=torch.uint8,
                     device=device)
    dq, dk, dv = torch.empty_like(t["q"]), torch.empty_like(t["k"]), torch.empty_like(t["v"])
    work = 2.5 * 4 * pairs * cfg.D * cfg.Hq

    def step():
        swa.thd_attn_bwd(t["q"], t["k"], t["v"], out, lse, dout, cu, cfg.window, cfg.scale,
                         t["sinks"], dq=dq, dk=dk, dv=dv, workspace=ws, stream=stream)
    step()
    check_status(swa, stream, f"bwd {name}")
    tot, per, h0, h1 = timed_loop(step, args, device, stream, f"thd_attn_bwd {name}")
    check_status(swa, stream, f"bwd {name}")
    peak = float(peaks["bf16_tflops"])
    return summarise(tot, per, args, work * info.world, UNIT, peak * info.world, peaks,
                     clocks.summary(h0, h1), "thd_attn_bwd_dq_kernel + thd_attn_bwd_dkdv_kernel",
                     {"workload": name, "valid_pairs": int(pairs), "tokens": T,
                      # preprocess, dq, dk/dv (dv and dk apart at D = 256), dsink with sinks
                      "launches_per_step": (4 if cfg.D == 256 else 3) + (1 if t["sinks"] is not None else 0),
                      "metric": "THD varlen attention bwd TFLOP/s (valid pairs, 2.5x forward FLOP)"})


def measure_prologue(swa, name, args, info, device, stream, clocks, peaks):
    cfg = workloads.CONFIGS[name]
    pack, t, _ = fwd_case(swa, cfg, args, info, device, stream, T_override=args.tokens)
    cu, T = pack["cu_seqlens"], pack["T"]
    work = 2 * T * (cfg.Hq + cfg.Hkv) * cfg.D * 2  # bytes: Q and K read and written once

    def step():
        swa.thd_qk_norm_rope(t["q"], t["k"], cu, stream=stream)
    step()
    check_status(swa, stream, "prologue")
    tot, per, h0, h1 = timed_loop(step, args, device, stream, f"thd_qk_norm_rope {name}")
    check_status(swa, stream, "prologue")
    peak = float(peaks["hbm_gbs"])
    return summarise(tot, per, args, work * info.world, "GB/s", peak * info.world, peaks,
                     clocks.summary(h0, h1), "thd_qk_norm_rope_kernel",
                     {"workload": name, "tokens": T, "bound": "hbm",
                      "metric": "Q/K prologue (scaleless RMSNorm + split-half RoPE) GB/s"})


SPARSE_MLA_WORKLOAD = dict(name="sparse_mla_t4096_h128_k2048_v128", lens=[4096], H=128, K=2048, vd=128)


def measure_sparse_mla(swa, args, info, device, stream, clocks, peaks):
    w = SPARSE_MLA_WORKLOAD
    c = workloads.sparse_mla_case(args.seed + 7919 * info.rank, w["lens"], w["H"], w["K"], w["vd"])
    q, kv, idx, wt = (c[n].to(device) for n in ("q", "kv", "indices", "value_weight"))
    T, H, vd = c["T"], w["H"], w["vd"]
    valid = int((c["indices"] >= 0).sum())
    flop = valid * H * 2 * (576 + 512) + T * H * 512 * vd * 2
    out = torch.empty((T, H, vd), dtype=torch.bfloat16, device=device)
    ws = torch.empty((swa.thd_sparse_mla_workspace_bytes(T, H, w["K"]),), dtype=torch.uint8,
                     device=device)

    def step():
        swa.thd_sparse_mla_fwd(q, kv, idx, wt, c["scale"], out=out, workspace=ws, stream=stream)
    step()
    if swa.thd_sparse_mla_get_error(stream) != 0:
        raise RuntimeError("sparse MLA: kernel reported an error status")
    tot, per, h0, h1 = timed_loop(step, args, device, stream, "thd_sparse_mla_fwd")
    if swa.thd_sparse_mla_get_error(stream) != 0:
        raise RuntimeError("sparse MLA: kernel reported an error status")
    peak = float(peaks["bf16_tflops"])
    return summarise(tot, per, args, flop * info.world, UNIT, peak * info.world, peaks,
                     clocks.summary(h0, h1), "thd_sparse_mla_attn_kernel + thd_sparse_mla_proj_kernel",
                     {"workload": w["name"], "tokens": T, "heads": H, "selected_keys": w["K"],
                      "value_dim": vd, "valid_slots": valid,
                      "launches_per_step": 3,  # slot compaction, attention, projection
                      "metric": "sparse MLA fwd TFLOP/s (valid slots, incl. value projection)"})


def run_ours(args, info):
    import sliding_window_gqa_cu_b200 as swa

    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (the CUDA path has no CPU fallback)")
    multirank.init("nccl")
    device = torch.device("cuda", info.local_rank)
    torch.cuda.set_device(device)
    swa.load_library()
    stream = torch.cuda.current_stream(device)
    peaks, peak_src = measured_peaks()
    peak = float(peaks["bf16_tflops"])

    cfg = workloads.CONFIGS[args.workload]
    pack, t, step = fwd_case(swa, cfg, args, info, device, stream, T_override=args.tokens)
    cu, T = pack["cu_seqlens"], pack["T"]
    pairs = metrics.valid_pairs(cu, cfg.window)
    Hq_r = t["q"].shape[1]  # query heads this rank computes (all of them unless --shard heads)
    flops = 4 * pairs * cfg.D * Hq_r

    t_plan0 = time.perf_counter()
    step()  # first call builds and uploads the tile schedule
    torch.cuda.synchronize(device)
    first_call_ms = (time.perf_counter() - t_plan0) * 1e3
    check_status(swa, stream, cfg.name)

    clocks = ClockSampler(device)
    max_ms, max_launch, h0, h1 = timed_loop(step, args, device, stream, f"thd_attn_fwd {cfg.name}")
    check_status(swa, stream, cfg.name)
    csum = clocks.summary(h0, h1)
    if args.shard == "tokens":  # flops is the whole pack's, shared by the ranks
        value = flops * args.steps / (max_ms / 1e3) / 1e12
    else:
        value = multirank.aggregate_rate(flops * args.steps, info.world, max_ms / 1e3) / 1e12
    launches = step.launches

    # end to end through the public API with pinned host buffers
    e2e = None
    if not args.no_e2e and args.shard == "packs":
        qh, kh, vh = (pack[n].pin_memory() for n in "qkv")
        sh = pack["sinks"].pin_memory() if pack["sinks"] is not None else None
        oh = torch.empty(t["out"].shape, dtype=t["out"].dtype).pin_memory()
        lh = torch.empty(t["lse"].shape, dtype=t["lse"].dtype).pin_memory()
        h2d = sum(x.numel() * x.element_size() for x in (qh, kh, vh) + ((sh,) if sh is not None else ()))
        d2h = oh.numel() * oh.element_size() + lh.numel() * lh.element_size()
        bufs = {n: t[n] for n in ("q", "k", "v", "out", "lse")}
        if sh is not None:
            bufs["sinks"] = t["sinks"]

        def e2e_step():
            # host -> device copies, attention and device -> host copies of
            # E2E_CHUNKS token ranges, overlapped (one call)
            swa.thd_attn_fwd_host(qh, kh, vh, cu, cfg.window, cfg.scale, sh, out_host=oh, lse_host=lh,
                                  device_buffers=bufs, n_chunks=E2E_CHUNKS, stream=stream)

        for _ in range(2):
            e2e_step()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        multirank.barrier(device)
        torch.cuda.synchronize(device)
        e0.record(stream)
        for _ in range(args.e2e_steps):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize(device)
        check_status(swa, stream, "e2e")
        e2e_ms = multirank.max_over_ranks(e0.elapsed_time(e1), device)
        e2e = {"value": multirank.aggregate_rate(flops * args.e2e_steps, info.world, e2e_ms / 1e3) / 1e12,
               "unit": UNIT, "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "ms_per_step": e2e_ms / args.e2e_steps,
               "path": f"thd_attn_fwd_host, pinned host buffers, {E2E_CHUNKS} overlapped token ranges"}

    # per GPU: the whole pack's flops over the ranks with --shard tokens
    achieved = flops / (info.world if args.shard == "tokens" else 1) / (max_launch / 1e3) / 1e12
    roofline = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak,
                # a full-pack launch's DRAM bytes: packs mode, or a single GPU
                "traffic": traffic_per_launch(cfg.name) if args.shard == "packs" or info.world == 1 else None,
                "peak_source": f"{peak_src} bf16 burst (MEASURED_PEAKS.json)" if peak_src == "measured"
                else "fallback 1.59 PFLOP/s",
                "frac_of_sustained": achieved / float(peaks.get("bf16_tflops_sustained", peak)),
                "frac_of_datasheet_2250": achieved / DATASHEET_BF16_TFLOPS,
                "kernel": kernel_name(cfg.D, Hq_r // t["k"].shape[1]),
                "algorithmic_flops_per_launch": flops,
                "algorithmic_bytes_per_launch": metrics.algorithmic_bytes(T, Hq_r, t["k"].shape[1],
                                                                          cfg.D)}
    del pack, t, step

    cpu = None
    if info.is_root and info.world == 1 and not args.no_cpu_baseline:
        cpack = workloads.make_pack(cfg, args.seed, T_override=args.tokens)
        tf, spent, rows, fl, threads = cpu_oracle_sample(cpack, args.cpu_seconds, seed=12345)
        cpu = {"value": tf, "unit": UNIT, "cores": threads, "kind": "oracle",
               "sample": f"{rows} random (token, head) rows of the same pack, fp64, "
                         f"{fl / 1e9:.1f} GFLOP in {spent:.1f} s"}
        del cpack

    per_config, passes = None, None
    if not args.no_extras and args.tokens is None and args.shard == "packs":
        per_config = {}
        for name in EXTRA_CONFIGS:
            if name == cfg.name:
                continue
            per_config[name] = measure_fwd_extra(swa, name, args, info, device, stream, clocks, peaks)
            torch.cuda.empty_cache()
        passes = {}
        for name in BWD_WORKLOADS:
            try:
                passes["bwd " + name] = measure_bwd(swa, name, args, info, device, stream, clocks,
                                                    peaks)
            except swa.ThdAttnError as e:  # a head dim the backward does not support
                if e.code != -2:
                    raise
                passes["bwd " + name] = {"unsupported": str(e)}
            torch.cuda.empty_cache()
        passes["prologue " + DEFAULT_WORKLOAD] = measure_prologue(swa, DEFAULT_WORKLOAD, args, info,
                                                                  device, stream, clocks, peaks)
        torch.cuda.empty_cache()
        passes["sparse_mla"] = measure_sparse_mla(swa, args, info, device, stream, clocks, peaks)
    clocks.stop()

    if info.is_root:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": info.world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": max_ms / args.steps,
            "higher_is_better": True, "scaling": "weak" if args.shard == "packs" else "strong",
            "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": workload_config(cfg, cu, pairs, {
                "parallelism": (f"head-sharded x{info.world} (one pack, no collective)"
                                if args.shard == "heads" else
                                f"context-parallel x{info.world} (token shards of one pack, "
                                f"K/V all-gather overlapped with the own-slice part)"
                                if args.shard == "tokens" else f"pack-parallel x{info.world}"),
                "per_rank_tflop": flops / 1e12}),
            "pct_of_peak": 100.0 * value / info.world / peak,
            "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": args.steps * launches, "clocks": {k: csum[k] for k in ("sm_mhz", "sm_max_mhz", "reasons")},
            "first_call_ms_with_schedule_build": first_call_ms,
            "per_config": per_config, "passes": passes,
        }
        log(f"[bench] {cfg.name}: {max_ms / args.steps:.3f} ms/step, {value:.1f} TFLOP/s "
            f"({100 * value / info.world / peak:.1f}% of {peak_src} {peak:.0f}, "
            f"{100 * value / info.world / DATASHEET_BF16_TFLOPS:.1f}% of 2250), clocks {csum}")
        for group in (per_config or {}), (passes or {}):
            for name, d in group.items():
                if "unsupported" in d:
                    log(f"[bench]   {name}: {d['unsupported']}")
                    continue
                log(f"[bench]   {name}: {d['ms_per_step']:.3f} ms/step, {d['value']:.1f} {d['unit']} "
                    f"({100 * d['frac']:.1f}% of {d['peak'] / info.world:.0f}), clocks {d['clocks']}")
        print(json.dumps(line), flush=True)
    multirank.shutdown()
    return 0


def run_other_pass(args, info):
    """--pass bwd / prologue / sparse_mla: one line for that pass alone."""
    import sliding_window_gqa_cu_b200 as swa

    if args.shard != "packs":
        raise SystemExit("--shard heads / tokens apply to the forward only")

    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (the CUDA path has no CPU fallback)")
    multirank.init("nccl")
    device = torch.device("cuda", info.local_rank)
    torch.cuda.set_device(device)
    swa.load_library()
    stream = torch.cuda.current_stream(device)
    peaks, peak_src = measured_peaks()
    clocks = ClockSampler(device)
    if args.pass_ == "bwd":
        d = measure_bwd(swa, args.workload, args, info, device, stream, clocks, peaks)
    elif args.pass_ == "prologue":
        d = measure_prologue(swa, args.workload, args, info, device, stream, clocks, peaks)
    else:
        d = measure_sparse_mla(swa, args, info, device, stream, clocks, peaks)
    clocks.stop()
    if info.is_root:
        cfg = workloads.CONFIGS[args.workload]
        launches = d.pop("launches_per_step", 1)
        line = {
            "metric": d.pop("metric"), "value": d["value"], "unit": d["unit"], "n_gpus": info.world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": d["ms_per_step"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic", "pass": args.pass_,
            "config": ({"workload": d["workload"]} if args.pass_ == "sparse_mla" else
                       workload_config(cfg, workloads.pack_cu_seqlens(cfg, args.seed) if args.tokens is None
                                       else np.array([0, d["tokens"]]), d.get("valid_pairs", 0),
                                       {"parallelism": f"pack-parallel x{info.world}"})),
            "roofline": {"bound": d.get("bound", "tensor"), "achieved": d["frac"] * d["peak"] / info.world,
                         "peak": d["peak"] / info.world, "unit": d["unit"], "frac": d["frac"],
                         "traffic": None, "kernel": d["kernel"],
                         "peak_source": f"{peak_src} (MEASURED_PEAKS.json)"},
            "cpu_baseline": None, "e2e": None, "gpu_launches": launches * args.steps,
            "clocks": d["clocks"],
        }
        log(f"[bench] {args.pass_}: {d['ms_per_step']:.3f} ms/step, {d['value']:.1f} {d['unit']} "
            f"({100 * d['frac']:.1f}% of {peak_src} {d['peak'] / info.world:.0f}), clocks {d['clocks']}")
        print(json.dumps(line), flush=True)
    multirank.shutdown()
    return 0


def main(argv=None):
    args = parse_args(argv)
    info = multirank.rank_info()
    if args.impl == "reference":
        return run_reference(args, info)
    if args.pass_ != "fwd":
        return run_other_pass(args, info)
    return run_ours(args, info)


if __name__ == "__main__":
    sys.exit(main())
