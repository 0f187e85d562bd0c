#!/usr/bin/env python
"""Benchmark of exact attention (forward + backward) on B200.

One step = the whole hot path on one batch: fa_fwd, then the three backward
stages (fa_bwd_preprocess, fa_bwd_main, fa_bwd_dq_convert), through the C ABI.
Throughput is TFLOP/s by the FlashAttention-2 convention: forward
4*B*H*N^2*d (halved when causal), backward 2.5x forward.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
  python bench.py --impl reference ...   # the fp64 CPU oracle on the host cores

With N > 1 (launched by torchrun) every rank runs its own independent shard of
heads (weak scaling, no data-path collective); the time is the max over ranks.
Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = ("attention fwd / fwd+bwd TFLOP/s (bf16, d=64/128, causal) and % of B200 "
          "BF16 peak")

# Points of the 16k-token sweep (width 2048, B = 16384 / N) and the GPT layers.
WORKLOADS = {
    "fwd_bwd_sweep_N8192_d128_causal": dict(B=2, H=16, N=8192, d=128, causal=True,
                                            dist="normal", seed=2),
    "fwd_bwd_sweep_N16384_d128_causal": dict(B=1, H=16, N=16384, d=128, causal=True,
                                             dist="normal", seed=2),
    "fwd_bwd_sweep_N2048_d128_causal": dict(B=8, H=16, N=2048, d=128, causal=True,
                                            dist="normal", seed=2),
    "fwd_bwd_sweep_N8192_d64_causal": dict(B=2, H=32, N=8192, d=64, causal=True,
                                           dist="normal", seed=2),
    "fwd_bwd_sweep_N2048_d64_causal": dict(B=8, H=32, N=2048, d=64, causal=True,
                                           dist="normal", seed=2),
    "fwd_bwd_sweep_N8192_d128_noncausal": dict(B=2, H=16, N=8192, d=128, causal=False,
                                               dist="normal", seed=2),
    "gpt_layer_a_B8_N2048_H16_d128": dict(B=8, H=16, N=2048, d=128, causal=True,
                                          dist="row_scaled", seed=4),
    "gpt_layer_b_B2_N8192_H20_d128": dict(B=2, H=20, N=8192, d=128, causal=True,
                                          dist="row_scaled", seed=5),
    "long_B1_H16_N65536_d128_causal": dict(B=1, H=16, N=65536, d=128, causal=True,
                                           dist="normal", seed=3),
}

# Forward with e4m3 Q, K (fa_fwd_qk8): the 16k-token sweep point at d=128.
QK8_WORKLOADS = {
    "fwd_qk8_sweep_N8192_d128_causal": dict(B=2, H=16, N=8192, d=128, causal=True,
                                            dist="normal", seed=2),
    "fwd_qk8_sweep_N8192_d128_noncausal": dict(B=2, H=16, N=8192, d=128, causal=False,
                                               dist="normal", seed=2),
    # fa_fwd_fp8: V in e4m3 too, both products on the 8-bit path
    "fwd_fp8_sweep_N8192_d128_causal": dict(B=2, H=16, N=8192, d=128, causal=True,
                                            dist="normal", seed=2, pv8=True),
    "fwd_fp8_sweep_N8192_d128_noncausal": dict(B=2, H=16, N=8192, d=128, causal=False,
                                               dist="normal", seed=2, pv8=True),
}

# Additive score bias (fa_fwd_bias / fa_bwd_bias): 16k tokens, a bias shared
# by the batch ([1, H, N, N] bf16), dBias [B, H, N, N] written.
BIAS_WORKLOADS = {
    "fwd_bwd_bias_B4_H16_N4096_d128_causal": dict(B=4, H=16, N=4096, d=128, causal=True,
                                                  dist="normal", seed=2),
}

# Sequence-sharded (ring) attention, G virtual ranks on one GPU: the long
# single-sequence shape split into G shards of N/G tokens.
RING_WORKLOADS = {
    "ring_G4_B1_H16_N65536_d128_causal": dict(B=1, H=16, N=65536, d=128, causal=True,
                                              dist="normal", seed=3, G=4, layout="contiguous"),
    "ring_G4_B1_H16_N65536_d128_causal_striped": dict(B=1, H=16, N=65536, d=128, causal=True,
                                                      dist="normal", seed=3, G=4,
                                                      layout="striped"),
    "ring_G2_B2_H16_N8192_d128_causal": dict(B=2, H=16, N=8192, d=128, causal=True,
                                             dist="normal", seed=2, G=2, layout="contiguous"),
}
DEFAULT_WORKLOAD = "fwd_bwd_sweep_N8192_d128_causal"

# Decoding (fa_fwd_decode): Nq query rows per sequence against a cache of Nk
# keys, model width 2048 (H = 16, d = 128); K/V of every workload exceed L2.
DECODE_WORKLOADS = {
    "decode_B16_H16_Nq1_Nk8192_d128": dict(B=16, H=16, Nq=1, Nk=8192, d=128, causal=True,
                                           dist="normal", seed=6),
    "decode_B1_H16_Nq1_Nk65536_d128": dict(B=1, H=16, Nq=1, Nk=65536, d=128, causal=True,
                                           dist="normal", seed=6),
    "decode_B4_H16_Nq4_Nk16384_d128": dict(B=4, H=16, Nq=4, Nk=16384, d=128, causal=True,
                                           dist="normal", seed=6),
    "decode_B32_H32_Nq1_Nk4096_d64": dict(B=32, H=32, Nq=1, Nk=4096, d=64, causal=True,
                                          dist="normal", seed=6),
}
DECODE_METRIC = "attention decode (split-KV) HBM GB/s: K/V cache + Q + O bytes per step"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}
DATASHEET_BF16_TFLOPS = 2250.0


def fwd_flops(w) -> float:
    f = 4.0 * w["B"] * w["H"] * w["N"] ** 2 * w["d"]
    return f * (0.5 if w["causal"] else 1.0)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", 0) or 0),
                "source": "measured"}
    except Exception:
        return dict(FALLBACK_PEAKS, source="fallback")


KERNEL_SOURCES = {
    "fa_fwd_kernel": ("fa_fwd_kernel.cuh",),
    "fa_fwd1_kernel": ("fa_fwd1_kernel.cuh", "fa_fwd_kernel.cuh"),
    "fa_fwd64_kernel": ("fa_fwd64_kernel.cuh", "fa_fwd_kernel.cuh"),
    "fa_bwd_main_kernel": ("fa_bwd_kernels.cuh",),
    "fa_bwd_main64_kernel": ("fa_bwd64_kernel.cuh", "fa_bwd_kernels.cuh"),
    "fa_decode_kernel": ("fa_decode_kernel.cuh",),
}


def fwd_kernel_name(N: int, d: int) -> str:
    """The forward kernel fa_fwd launches for this shape (the shape rule in
    csrc/fa_api.cu, use_fwd64 and use_fwd1)."""
    if d == 64 and N <= 2048:
        return "fa_fwd64_kernel"
    if d == 128 and N <= 512:
        return "fa_fwd1_kernel"
    return "fa_fwd_kernel"


def bwd_main_kernel_name(d: int) -> str:
    """The backward main-stage kernel fa_bwd_main launches (no bias)."""
    return "fa_bwd_main64_kernel" if d == 64 else "fa_bwd_main_kernel"


# Files besides the kernel's own that decide what it does: the PTX helpers
# (descriptors, MMA and copy wrappers) and the host code that sets its launch.
SHARED_SOURCES = ("sm100_ptx.cuh", "fa_api.cu")


def kernel_sources_hash(kernel: str) -> str:
    """Hash of the kernel's own source file and of the shared sources above."""
    h = hashlib.sha256()
    for name in KERNEL_SOURCES[kernel] + SHARED_SOURCES:
        with open(os.path.join(ROOT, "exact_attention_109_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    the current source of that kernel and this workload; otherwise None."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
        ent = rec[kernel][workload]
        if ent.get("sources_hash") != kernel_sources_hash(kernel):
            return None
        return float(ent["dram_bytes_per_launch"])
    except Exception:
        return None


# ---------------------------------------------------------------- clocks


class ClockSampler:
    """nvidia-smi sampling of SM clock and throttle reasons (read-only)."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        import torch
        self.proc = None
        sel = []
        try:
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            sel = ["-i", uuid if uuid.startswith("GPU-") else "GPU-" + uuid]
        except Exception:
            sel = []
        self.cmd = ["nvidia-smi", *sel, f"--query-gpu={self.FIELDS}",
                    "--format=csv,noheader,nounits", "-lms", "100"]

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(self.cmd, stdout=subprocess.PIPE,
                                         stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]
        return False

    def summary(self):
        rows = []
        for line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                rows.append((float(parts[0]), float(parts[1]), parts[4:8]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"],
                    "samples": 0}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown",
                 "sw_power_cap"]
        seen = set()
        for _, _, flags in rows:
            for n, fl in zip(names, flags):
                if fl.lower().startswith("active"):
                    seen.add(n)
        return {"sm_mhz": statistics.median(r[0] for r in rows),
                "sm_max_mhz": max(r[1] for r in rows),
                "reasons": sorted(seen), "samples": len(rows)}


# ---------------------------------------------------------------- CPU oracle


def oracle_sample(w, seconds: float, seed: int = 0):
    """Time the fp64 oracle on sampled rows of head 0 of the workload.

    Each timed pass first computes the per-row softmax statistics (LSE_i, D_i)
    of the whole head, which every dK/dV row needs, and then O, LSE and dQ for
    R query rows and dK, dV for R key rows, i.e. R/N of the head's outputs,
    credited R/N of the head's fwd+bwd FLOPs (the statistics pass is timed
    but earns no extra credit).  R is sized so one pass takes about `seconds`.
    Returns (run(R) -> seconds, R, cores, flops_per_pass(R)).
    """
    import numpy as np
    import oracle
    from exact_attention_109_b200.inputs import attention_inputs, default_scale, to_f64

    inp = attention_inputs(1, 1, w["N"], w["d"], w["seed"], w["dist"], with_dout=True)
    q, k, v, dO = (to_f64(inp[x])[0, 0] for x in ("q", "k", "v", "dO"))
    scale = default_scale(w["d"])
    causal = w["causal"]
    rng = np.random.default_rng(seed)
    N = w["N"]
    head = dict(w, B=1, H=1)
    per_head = 3.5 * fwd_flops(head)

    def run(R):
        rows = np.sort(rng.choice(N, size=R, replace=False))
        t0 = time.perf_counter()
        lse, D = oracle.ref_head_stats(q, k, v, dO, causal, scale)
        oracle.ref_fwd_rows(q, k, v, rows, causal, scale)
        oracle.ref_dq_rows(q, k, v, dO, rows, causal, scale)
        oracle.ref_dkdv_rows(q, k, v, dO, lse, D, rows, causal, scale)
        return time.perf_counter() - t0

    r0 = min(N, 256)
    t = run(r0)
    t_stats = run(1)
    per_row = max(t - t_stats, 1e-6) / r0
    R = int(min(N, max(8, math.ceil((seconds - t_stats) / per_row))))
    return run, R, oracle.num_threads(), (lambda r: per_head * r / N)


def oracle_whole_heads(w, seconds: float):
    """Time the fp64 oracle's full forward and backward (ref_fwd, ref_bwd) on
    whole heads of the workload: as many heads as the host has threads (at most
    B*H), fewer if one head alone already takes `seconds`."""
    import oracle
    from exact_attention_109_b200.inputs import attention_inputs, default_scale, to_f64

    cores = oracle.num_threads()
    heads = max(1, min(w["B"] * w["H"], cores))
    inp = attention_inputs(1, heads, w["N"], w["d"], w["seed"], w["dist"], with_dout=True)
    q, k, v, dO = (to_f64(inp[x]) for x in ("q", "k", "v", "dO"))
    scale = default_scale(w["d"])
    t0 = time.perf_counter()
    oracle.ref_fwd(q, k, v, w["causal"], scale)
    oracle.ref_bwd(q, k, v, dO, w["causal"], scale)
    t = time.perf_counter() - t0
    flops = 3.5 * fwd_flops(dict(w, B=1, H=heads))
    return flops / t / 1e12, t, heads, cores


def reference_arm(args, w, wname):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    steps, warmup = args.steps, args.warmup
    per_step = max(0.05, 150.0 / max(1, steps + warmup))
    run, R, cores, credit = oracle_sample(w, per_step)
    for _ in range(warmup):
        run(R)
    times = [run(R) for _ in range(steps)]
    total = sum(times)
    value = credit(R) * steps / total / 1e12
    sample = (f"{R} of {w['N']} query rows (O, LSE, dQ) and key rows (dK, dV) of one "
              f"head per step, credited {R}/{w['N']} of the head's fwd+bwd FLOPs; "
              f"each step also recomputes the head's per-row LSE/D statistics (timed)")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": steps, "warmup": warmup,
        "ms_per_step": 1e3 * total / steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(w, wname),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores,
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def shard_heads(heads_per_rank: int, world: int, rank: int):
    """Global head range [start, stop) that `rank` owns when every rank runs
    its own heads_per_rank independent heads (weak scaling: the per-GPU work
    is fixed, the global problem grows with the number of ranks)."""
    start = rank * heads_per_rank
    return start, start + heads_per_rank


def max_over_ranks(value_ms: float, device=None) -> float:
    """The slowest rank's time (max-reduce when a process group is active)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value_ms)], dtype=torch.float64,
                     device=device if device is not None else "cpu")
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(flops_per_rank_step: float, steps: int, world: int,
                   max_ms: float) -> float:
    """Whole-job TFLOP/s: the work of all ranks over the slowest rank's time."""
    return flops_per_rank_step * steps * world / (max_ms * 1e-3) / 1e12


def workload_config(w, wname):
    bh, N, d = w["B"] * w["H"], w["N"], w["d"]
    n_pad = (N + 127) // 128 * 128
    # q, k, v, o, dO, dq, dk, dv bf16 + LSE, and the fp32 workspace
    working_set = 8 * bh * N * d * 2 + bh * N * 4 + bh * n_pad * (d + 2) * 4
    return {"workload": wname, "B": w["B"], "H": w["H"], "N": N, "d": d,
            "causal": w["causal"], "inputs": w["dist"], "pass": "fwd+bwd",
            "global_batch": w["B"], "seq_len": N,
            "parallelism": "independent head shards per GPU",
            "l2": f"no flush: per-step working set {working_set / 1e6:.0f} MB > 126 MB L2"}


# ---------------------------------------------------------------- GPU arm


def gpu_arm(args, w, wname):
    import numpy as np
    import torch
    import torch.distributed as dist

    import exact_attention_109_b200 as fa
    from exact_attention_109_b200.inputs import attention_inputs, default_scale

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=180),
                                device_id=torch.device("cuda", local))

    B, H, N, d, causal = w["B"], w["H"], w["N"], w["d"], w["causal"]
    scale = default_scale(d)
    head0, _ = shard_heads(B * H, world, rank)
    host = attention_inputs(B, H, N, d, w["seed"] + head0, w["dist"], with_dout=True)
    dev = {k_: v_.cuda() for k_, v_ in host.items()}
    q, k, v, dO = dev["q"], dev["k"], dev["v"], dev["dO"]
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
    ws_bytes = fa.fa_bwd_workspace_size(B, H, N, d)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=q.device)
    stream = torch.cuda.current_stream()
    s = stream.cuda_stream
    P = {x: t.data_ptr() for x, t in dict(q=q, k=k, v=v, dO=dO, o=o, lse=lse, dq=dq,
                                         dk=dk, dv=dv, ws=ws).items()}

    def stage_fwd():
        return fa.fa_fwd(P["q"], P["k"], P["v"], P["o"], P["lse"], B, H, N, d, causal,
                         scale, s)

    def stage_pre():
        return fa.fa_bwd_preprocess(P["o"], P["lse"], P["dO"], B, H, N, d, P["ws"],
                                    ws_bytes, s)

    def stage_main():
        return fa.fa_bwd_main(P["q"], P["k"], P["v"], P["dO"], P["dk"], P["dv"], B, H, N,
                              d, causal, scale, P["ws"], ws_bytes, s)

    def stage_conv():
        return fa.fa_bwd_dq_convert(P["dq"], B, H, N, d, scale, P["ws"], ws_bytes, s)

    stages = [(fwd_kernel_name(N, d), stage_fwd), ("fa_bwd_pre_kernel", stage_pre),
              (bwd_main_kernel_name(d), stage_main), ("fa_bwd_dq_convert_kernel", stage_conv)]

    def step(events=None):
        for i, (_, fn) in enumerate(stages):
            if events is not None:
                events[i].record(stream)
            st = fn()
            if st != fa.FA_OK:
                raise fa.FaError(st, "bench step")
        if events is not None:
            events[len(stages)].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    status = fa.fa_get_device_error()
    if status != fa.FA_OK:
        raise fa.FaError(status, "warm-up")
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()

    K = args.steps
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(len(stages) + 1)]
           for _ in range(K)]
    with ClockSampler(local) as clk:
        time.sleep(0.3)  # let the sampler start before the timed region
        torch.cuda.synchronize()
        for i in range(K):
            step(evs[i])
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    status = fa.fa_get_device_error()
    if status != fa.FA_OK:
        raise fa.FaError(status, "timed region")

    elapsed_ms = evs[0][0].elapsed_time(evs[-1][-1])
    per_stage = [sum(evs[i][j].elapsed_time(evs[i][j + 1]) for i in range(K)) / K
                 for j in range(len(stages))]
    elapsed_max = max_over_ranks(elapsed_ms, q.device)
    flops_step = 3.5 * fwd_flops(w)
    value = job_throughput(flops_step, K, world, elapsed_max)

    # ---- end to end through the public API with pinned host buffers.  Every
    # step copies its q, k, v, dO in from pinned host memory and its O, LSE,
    # dQ, dK, dV back out; three streams (host->device, compute,
    # device->host) and two device buffer sets let step i's copies overlap
    # the neighbouring steps' compute, as a pipelined caller would run it.
    pin = {x: host[x].pin_memory() for x in ("q", "k", "v", "dO")}
    outs = ("o", "lse", "dq", "dk", "dv")
    out_host = {x: torch.empty(t_.shape, dtype=t_.dtype, pin_memory=True)
                for x, t_ in dict(o=o, lse=lse, dq=dq, dk=dk, dv=dv).items()}
    h2d = sum(t_.numel() * t_.element_size() for t_ in pin.values())
    d2h = sum(t_.numel() * t_.element_size() for t_ in out_host.values())
    bufs = []
    for _ in range(2):
        bq = {x: torch.empty_like(dev[x]) for x in ("q", "k", "v", "dO")}
        bo = {"o": torch.empty_like(o), "lse": torch.empty_like(lse),
              "dq": torch.empty_like(dq), "dk": torch.empty_like(dk), "dv": torch.empty_like(dv)}
        bufs.append((bq, bo))
    s_in, s_cmp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_cmp = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def e2e_step(i):
        bq, bo = bufs[i % 2]
        with torch.cuda.stream(s_in):
            s_in.wait_event(ev_cmp[i % 2])      # step i-2 has finished reading bq
            for x in ("q", "k", "v", "dO"):
                bq[x].copy_(pin[x], non_blocking=True)
            ev_in[i % 2].record(s_in)
        with torch.cuda.stream(s_cmp):
            s_cmp.wait_event(ev_in[i % 2])
            s_cmp.wait_event(ev_out[i % 2])     # step i-2's results have left bo
            fa.attention_forward(bq["q"], bq["k"], bq["v"], causal, scale, out=bo["o"],
                                 lse=bo["lse"], stream=s_cmp)
            fa.attention_backward(bq["q"], bq["k"], bq["v"], bo["o"], bo["lse"], bq["dO"],
                                  causal, scale, dq=bo["dq"], dk=bo["dk"], dv=bo["dv"],
                                  workspace=ws, stream=s_cmp)
            ev_cmp[i % 2].record(s_cmp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_cmp[i % 2])
            for x in outs:
                out_host[x].copy_(bo[x], non_blocking=True)
            ev_out[i % 2].record(s_out)

    for i in range(4):
        e2e_step(i)
    torch.cuda.synchronize()
    Ke = max(4, min(K, 20))
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    for i in range(Ke):
        e2e_step(i)
    s_in.wait_stream(s_out)
    e1.record(s_in)
    torch.cuda.synchronize()
    e2e_value = job_throughput(flops_step, Ke, world,
                               max_over_ranks(e0.elapsed_time(e1), q.device))
    status = fa.fa_get_device_error()
    if status != fa.FA_OK:
        raise fa.FaError(status, "e2e")

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0

    # ---- roofline of the dominant kernel
    peaks = load_peaks()
    names = [n for n, _ in stages]
    dom = int(np.argmax(per_stage))
    bh = B * H
    n_pad = (N + 127) // 128 * 128
    algo = {
        fwd_kernel_name(N, d): ("tensor", fwd_flops(w)),
        bwd_main_kernel_name(d): ("tensor", 2.5 * fwd_flops(w)),
        "fa_bwd_pre_kernel": ("hbm", 2 * bh * N * d * 2 + bh * N * 4 + 2 * bh * n_pad * 4
                              + bh * n_pad * d * 4),
        "fa_bwd_dq_convert_kernel": ("hbm", bh * N * d * 4 + bh * N * d * 2),
    }
    bound, amount = algo[names[dom]]
    sec = per_stage[dom] * 1e-3
    if bound == "tensor":
        achieved = amount / sec / 1e12
        peak = peaks["bf16_tflops"]
        unit = "TFLOP/s"
    else:
        achieved = amount / sec / 1e9
        peak = peaks["hbm_gbs"]
        unit = "GB/s"
    roofline = {"kernel": names[dom], "bound": bound, "achieved": achieved, "peak": peak,
                "unit": unit, "frac": achieved / peak,
                "peak_source": f"{peaks['source']} (burst)",
                "traffic": recorded_traffic(names[dom], wname)}
    fwd_t = fwd_flops(w) / (per_stage[0] * 1e-3) / 1e12
    bwd_ms = sum(per_stage[1:])
    bwd_t = 2.5 * fwd_flops(w) / (bwd_ms * 1e-3) / 1e12

    # ---- CPU baseline: the oracle on the host cores, bounded sample
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        val, tcpu, heads, cores = oracle_whole_heads(w, 30.0)
        cpu = {"value": val, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
               "sample": (f"oracle ref_fwd + ref_bwd on {heads} whole heads of the "
                          f"workload (N={N}, d={d}, causal={causal}), {tcpu:.1f} s")}

    # ---- the rest of the pages' sweep, measured in the same run (one GPU)
    sweep = None
    if world == 1 and not args.no_sweep:
        sweep = {"note": "fa_fwd / fa_bwd (three launches) per shape through the C ABI; "
                         "inputs drawn on the device; every working set exceeds L2",
                 "shapes": measure_sweep(args.warmup, local)}

    clocks = clk.summary()
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": K, "warmup": args.warmup, "ms_per_step": elapsed_max / K,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic",
        "config": workload_config(w, wname),
        "fwd_tflops": fwd_t, "bwd_tflops": bwd_t,
        "frac_of_peak": value / peaks["bf16_tflops"],
        "frac_of_datasheet_bf16": value / DATASHEET_BF16_TFLOPS,
        "kernel_ms": {n: round(t_, 4) for n, t_ in zip(names, per_stage)},
        "roofline": roofline,
        "cpu_baseline": cpu,
        "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h,
                "note": "public API, pinned host buffers, copies of each step overlap "
                        "neighbouring steps on separate streams"},
        "gpu_launches": len(stages) * K,
        "clocks": clocks,
        "sweep": sweep,
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------- decoding


def decode_bytes(w) -> int:
    """Algorithmic HBM bytes of one decoding step: every cached key and value
    row read once, the query rows read, O written (bf16), LSE written (fp32)."""
    bh = w["B"] * w["H"]
    return bh * (2 * w["Nk"] * w["d"] * 2 + 2 * w["Nq"] * w["d"] * 2 + w["Nq"] * 4)


def decode_config(w, wname):
    return {"workload": wname, "B": w["B"], "H": w["H"], "Nq": w["Nq"], "Nk": w["Nk"],
            "d": w["d"], "causal": w["causal"], "inputs": w["dist"], "pass": "decode fwd",
            "global_batch": w["B"], "seq_len": w["Nk"],
            "parallelism": "independent head shards per GPU"}


def oracle_decode(w, seconds: float):
    """Time the oracle's decoding reference on whole heads of the workload: as
    many as fit in about `seconds` (at least one).  Returns (GB/s credited by
    the same byte count as the GPU line, seconds, heads, cores)."""
    import oracle
    from exact_attention_109_b200.inputs import decode_inputs, default_scale, to_f64

    cores = oracle.num_threads()
    scale = default_scale(w["d"])
    heads = max(1, min(w["B"] * w["H"], cores))
    while True:
        inp = decode_inputs(1, heads, w["Nq"], w["Nk"], w["d"], w["seed"], w["dist"])
        q, k, v = (to_f64(inp[x]) for x in ("q", "k", "v"))
        t0 = time.perf_counter()
        oracle.ref_fwd_decode(q, k, v, w["causal"], scale)
        t = time.perf_counter() - t0
        if t * 2 > seconds or heads >= w["B"] * w["H"]:
            break
        heads = min(w["B"] * w["H"], heads * 2)
    return decode_bytes(dict(w, B=1, H=heads)) / t / 1e9, t, heads, cores


def decode_reference_arm(args, w, wname):
    if int(os.environ.get("RANK", "0")) != 0:
        return 0
    per_step = max(0.05, 150.0 / max(1, args.steps + args.warmup))
    _, _, heads, cores = oracle_decode(w, per_step)
    import oracle
    from exact_attention_109_b200.inputs import decode_inputs, default_scale, to_f64
    inp = decode_inputs(1, heads, w["Nq"], w["Nk"], w["d"], w["seed"], w["dist"])
    q, k, v = (to_f64(inp[x]) for x in ("q", "k", "v"))
    scale = default_scale(w["d"])
    for _ in range(args.warmup):
        oracle.ref_fwd_decode(q, k, v, w["causal"], scale)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.ref_fwd_decode(q, k, v, w["causal"], scale)
    total = time.perf_counter() - t0
    value = decode_bytes(dict(w, B=1, H=heads)) * args.steps / total / 1e9
    sample = (f"oracle ref_fwd_decode on {heads} of {w['B'] * w['H']} heads per step, "
              f"credited those heads' bytes")
    print(json.dumps({
        "impl": "reference", "metric": DECODE_METRIC, "value": value, "unit": "GB/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": decode_config(w, wname),
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0}}), flush=True)
    return 0


def decode_arm(args, w, wname):
    import torch
    import torch.distributed as dist

    import exact_attention_109_b200 as fa
    from exact_attention_109_b200.inputs import decode_inputs, default_scale

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=180),
                                device_id=torch.device("cuda", local))
    B, H, Nq, Nk, d, causal = w["B"], w["H"], w["Nq"], w["Nk"], w["d"], w["causal"]
    scale = default_scale(d)
    head0, _ = shard_heads(B * H, world, rank)
    host = decode_inputs(B, H, Nq, Nk, d, w["seed"] + head0, w["dist"])
    q, k, v = (host[x].cuda() for x in ("q", "k", "v"))
    o = torch.empty_like(q)
    lse = torch.empty((B, H, Nq), dtype=torch.float32, device=q.device)
    ws_bytes = fa.fa_decode_workspace_size(B, H, Nq, Nk, d)
    ws = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=q.device)
    stream = torch.cuda.current_stream()
    s = stream.cuda_stream
    P = [q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr()]

    def step():
        st = fa.fa_fwd_decode(*P, B, H, Nq, Nk, Nk, d, int(causal), scale,
                              ws.data_ptr() if ws_bytes else 0, ws_bytes, s)
        if st != fa.FA_OK:
            raise fa.FaError(st, "decode step")

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if fa.fa_get_device_error() != fa.FA_OK:
        raise RuntimeError("decode warm-up: device error")
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    K = args.steps
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(K + 1)]
    with ClockSampler(local) as clk:
        time.sleep(0.3)
        torch.cuda.synchronize()
        for i in range(K):
            evs[i].record(stream)
            step()
        evs[K].record(stream)
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    if fa.fa_get_device_error() != fa.FA_OK:
        raise RuntimeError("decode timed region: device error")
    per_step = [evs[i].elapsed_time(evs[i + 1]) for i in range(K)]
    elapsed_max = max_over_ranks(sum(per_step), q.device)
    nbytes = decode_bytes(w)
    value = nbytes * K * world / (elapsed_max * 1e-3) / 1e9

    # End to end through the public API: the cache stays resident on the
    # device (it is the decoding state); each step's query rows come in from
    # pinned host memory and O, LSE go back out.
    q_pin = host["q"].pin_memory()
    o_host = torch.empty(o.shape, dtype=o.dtype, pin_memory=True)
    l_host = torch.empty(lse.shape, dtype=lse.dtype, pin_memory=True)
    qd = torch.empty_like(q)

    def e2e_step():
        qd.copy_(q_pin, non_blocking=True)
        fa.attention_decode(qd, k, v, causal, scale, out=o, lse=lse,
                            workspace=ws if ws_bytes else None)
        o_host.copy_(o, non_blocking=True)
        l_host.copy_(lse, non_blocking=True)

    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize()
    Ke = max(4, min(K, 50))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(Ke):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_value = nbytes * Ke * world / (max_over_ranks(e0.elapsed_time(e1), q.device)
                                       * 1e-3) / 1e9
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0

    peaks = load_peaks()
    st, qg, n_splits, chunk = fa.fa_decode_split_plan(
        B, H, Nq, Nk, d, torch.cuda.get_device_properties(local).multi_processor_count,
        2 if d == 128 else 3)
    mean_ms = sum(per_step) / K
    achieved = nbytes / (mean_ms * 1e-3) / 1e9
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        val, tcpu, heads, cores = oracle_decode(w, 20.0)
        cpu = {"value": val, "unit": "GB/s", "cores": cores, "kind": "oracle",
               "sample": f"oracle ref_fwd_decode on {heads} whole heads, {tcpu:.2f} s"}
    line = {
        "metric": DECODE_METRIC, "value": value, "unit": "GB/s", "n_gpus": world,
        "steps": K, "warmup": args.warmup, "ms_per_step": elapsed_max / K,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32 (bf16 inputs)", "data": "synthetic",
        "config": dict(decode_config(w, wname),
                       l2=f"no flush: K/V {2 * B * H * Nk * d * 2 / 1e6:.0f} MB > 126 MB L2",
                       split=f"{n_splits} key splits of {chunk}, {qg} query rows per CTA"),
        "tokens_per_s": B * Nq * K * world / (elapsed_max * 1e-3),
        "roofline": {"kernel": "fa_decode_kernel (+ fa_decode_combine_kernel)",
                     "bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"],
                     "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"],
                     "peak_source": f"{peaks['source']} copy bandwidth",
                     "traffic": recorded_traffic("fa_decode_kernel", wname)},
        "cpu_baseline": cpu,
        "e2e": {"value": e2e_value, "unit": "GB/s", "h2d_bytes_per_step": q.numel() * 2,
                "d2h_bytes_per_step": o.numel() * 2 + lse.numel() * 4,
                "note": "public API; K/V cache resident on the device, query rows in "
                        "from pinned host memory, O and LSE back, every step"},
        "gpu_launches": K * (2 if n_splits > 1 else 1),
        "clocks": clk.summary(),
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------- ring


class _TimedRingOps:
    """The ring's CUDA ops with CUDA events around every call, so that each
    virtual rank's own device time can be summed."""

    def __init__(self):
        from exact_attention_109_b200 import ring
        self._ops = ring.CudaOps()
        self._events = []

    def _timed(self, name):
        import torch
        fn = getattr(self._ops, name)

        def call(*a, **kw):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            out = fn(*a, **kw)
            e1.record()
            self._events.append((e0, e1))
            return out
        return call

    def __getattr__(self, name):
        return self._timed(name)

    def total_ms(self):
        return sum(a.elapsed_time(b) for a, b in self._events)


def ring_arm(args, w, wname):
    """G virtual ranks on this GPU (exact_attention_109_b200.ring.run_local):
    one step = the ring forward and backward over the whole sequence, every
    (query shard, key shard) pair through the CUDA kernels, every rotation a
    device copy of the bytes a ring would move."""
    import torch

    import exact_attention_109_b200 as fa
    from exact_attention_109_b200 import ring
    from exact_attention_109_b200.inputs import attention_inputs, default_scale

    if int(os.environ.get("WORLD_SIZE", "1")) > 1:
        print(json.dumps({"metric": METRIC, "error": "ring workloads run G virtual ranks on "
                          "one GPU; across GPUs the ring runs through ring.run_nccl"}))
        return 1
    torch.cuda.set_device(0)
    B, H, N, d, causal, G = w["B"], w["H"], w["N"], w["d"], w["causal"], w["G"]
    scale = default_scale(d)
    host = attention_inputs(B, H, N, d, w["seed"], w["dist"], with_dout=True)
    q, k, v, dO = (host[x].cuda() for x in ("q", "k", "v", "dO"))
    stream = torch.cuda.current_stream()

    layout = w.get("layout", "contiguous")

    def step():
        return ring.local_ring_attention(q, k, v, dO, causal, scale, G, layout=layout)

    def plain_step():
        o, lse = fa.attention_forward(q, k, v, causal, scale)
        fa.attention_backward(q, k, v, o, lse, dO, causal, scale)

    for _ in range(args.warmup):
        step()
        plain_step()
    torch.cuda.synchronize()
    if fa.fa_get_device_error() != fa.FA_OK:
        raise RuntimeError("ring warm-up: device error")
    K = args.steps
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(K + 1)]
    with ClockSampler(0) as clk:
        time.sleep(0.3)
        torch.cuda.synchronize()
        for i in range(K):
            ev[i].record(stream)
            step()
        ev[K].record(stream)
        torch.cuda.synchronize()
    ring_ms = ev[0].elapsed_time(ev[K]) / K
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(K):
        plain_step()
    e1.record(stream)
    torch.cuda.synchronize()
    plain_ms = e0.elapsed_time(e1) / K
    if fa.fa_get_device_error() != fa.FA_OK:
        raise RuntimeError("ring timed region: device error")
    flops = 3.5 * fwd_flops(w)
    value = flops / (ring_ms * 1e-3) / 1e12

    # end to end: q, k, v, dO in from pinned host memory, O, LSE, dQ, dK, dV out
    pin = {x: host[x].pin_memory() for x in ("q", "k", "v", "dO")}
    dev = {x: torch.empty_like(q) for x in pin}
    outs = None
    Ke = max(2, min(K, 5))
    e0.record(stream)
    for _ in range(Ke):
        for x in pin:
            dev[x].copy_(pin[x], non_blocking=True)
        got = ring.local_ring_attention(dev["q"], dev["k"], dev["v"], dev["dO"], causal, scale, G,
                                        layout=layout)
        outs = [t.to("cpu", non_blocking=True) for t in got]
    e1.record(stream)
    torch.cuda.synchronize()
    e2e = flops / (e0.elapsed_time(e1) / Ke * 1e-3) / 1e12
    h2d = sum(t.numel() * t.element_size() for t in pin.values())
    d2h = sum(t.numel() * t.element_size() for t in outs)

    # Per-rank work: the device time of each virtual rank's own kernels (its
    # pair attention, merges and conversions; rotations excluded).  On G
    # GPUs with overlapped transfers the slowest rank sets the ring's time,
    # which is what the layouts differ in under the causal mask.
    per_rank = {}
    for lay in ring.LAYOUTS:
        timers = [_TimedRingOps() for _ in range(G)]
        ring.local_ring_attention(q, k, v, dO, causal, scale, G, ops=timers, layout=lay)
        torch.cuda.synchronize()
        ms = [t.total_ms() for t in timers]
        per_rank[lay] = {"per_rank_ms": [round(x, 3) for x in ms],
                         "critical_path_ms": round(max(ms), 3)}

    peaks = load_peaks()
    cpu = None
    if not args.no_cpu_baseline:
        run, R, cores, credit = oracle_sample(w, 20.0)
        t = run(R)
        cpu = {"value": credit(R) / t / 1e12, "unit": "TFLOP/s", "cores": cores,
               "kind": "oracle",
               "sample": f"{R} of {N} query rows and key rows of one head (whole-sequence "
                         f"fwd+bwd outputs), credited {R}/{N} of the head's FLOPs"}
    achieved = value
    print(json.dumps({
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": 1, "steps": K,
        "warmup": args.warmup, "ms_per_step": ring_ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": dict(workload_config(w, wname), **{
            "G": G, "layout": layout, "pass": "ring fwd+bwd",
            "parallelism": f"ring of {G} virtual ranks on one GPU",
            "l2": f"no flush: per-step working set {9 * B * H * N * d * 2 / 1e6:.0f} MB"}),
        "plain_fwd_bwd_tflops": flops / (plain_ms * 1e-3) / 1e12,
        "ring_overhead": ring_ms / plain_ms - 1.0,
        "layout": layout,
        "per_rank_work": per_rank,
        "roofline": {"kernel": "whole ring step (fa_fwd, fa_lse_merge, fa_bwd_*)",
                     "bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"],
                     "unit": "TFLOP/s", "frac": achieved / peaks["bf16_tflops"],
                     "peak_source": f"{peaks['source']} (burst)", "traffic": None},
        "cpu_baseline": cpu,
        "e2e": {"value": e2e, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "note": "public API, serial copies"},
        "gpu_launches": None,
        "clocks": clk.summary()}), flush=True)
    return 0


# ---------------------------------------------------------------- e4m3 scores


def qk8_arm(args, w, wname):
    """Forward only: fa_fwd_qk8 (e4m3 Q, K; bf16 V) timed beside fa_fwd on the
    dequantised bf16 inputs.  S = QK^T runs at the e4m3 rate and P V at the
    bf16 rate, so the roofline peak is the harmonic mix of the two: half the
    FLOPs at 2x the measured bf16 peak (the nominal e4m3:bf16 ratio of 2),
    half at 1x, i.e. 4/3 of the bf16 peak.  With pv8 the workload runs
    fa_fwd_fp8 instead (V e4m3 too, both products at the e4m3 rate: peak 2x
    the bf16 one), timed beside fa_fwd_qk8 and fa_fwd."""
    import torch

    import exact_attention_109_b200 as fa
    from exact_attention_109_b200.inputs import attention_inputs, default_scale, to_e4m3

    if int(os.environ.get("WORLD_SIZE", "1")) > 1:
        print(json.dumps({"metric": METRIC, "error": "e4m3 workloads run on one GPU"}))
        return 1
    torch.cuda.set_device(0)
    B, H, N, d, causal = w["B"], w["H"], w["N"], w["d"], w["causal"]
    scale = default_scale(d)
    host = attention_inputs(B, H, N, d, w["seed"], w["dist"])
    q8, qs = to_e4m3(host["q"])
    k8, ks = to_e4m3(host["k"])
    pv8 = bool(w.get("pv8"))
    v8, vs = to_e4m3(host["v"])
    q8d, k8d, v = q8.cuda(), k8.cuda(), host["v"].cuda()
    v8d = v8.cuda()
    qd = (q8.to(torch.float32) * qs).to(torch.bfloat16).cuda()
    kd = (k8.to(torch.float32) * ks).to(torch.bfloat16).cuda()
    vd = (v8.to(torch.float32) * vs).to(torch.bfloat16).cuda() if pv8 else v
    o = torch.empty_like(v)
    lse = torch.empty((B, H, N), dtype=torch.float32, device="cuda")
    s = torch.cuda.current_stream()

    def qk8_step():
        st = fa.fa_fwd_qk8(q8d.data_ptr(), k8d.data_ptr(), vd.data_ptr(), qs, ks, o.data_ptr(),
                           lse.data_ptr(), B, H, N, d, int(causal), scale, s.cuda_stream)
        if st != fa.FA_OK:
            raise fa.FaError(st, "qk8 step")

    def fp8_step():
        st = fa.fa_fwd_fp8(q8d.data_ptr(), k8d.data_ptr(), v8d.data_ptr(), qs, ks, vs,
                           o.data_ptr(), lse.data_ptr(), B, H, N, d, int(causal), scale,
                           s.cuda_stream)
        if st != fa.FA_OK:
            raise fa.FaError(st, "fp8 step")

    step = fp8_step if pv8 else qk8_step

    def bf16_step():
        fa.attention_forward(qd, kd, vd, causal, scale, out=o, lse=lse)

    for _ in range(args.warmup):
        step()
        qk8_step()
        bf16_step()
    torch.cuda.synchronize()
    K = args.steps
    e = [torch.cuda.Event(enable_timing=True) for _ in range(5)]
    with ClockSampler(0) as clk:
        time.sleep(0.3)
        torch.cuda.synchronize()
        e[0].record(s)
        for _ in range(K):
            step()
        e[1].record(s)
        for _ in range(K):
            bf16_step()
        e[2].record(s)
        for _ in range(K):
            qk8_step()
        e[4].record(s)
        torch.cuda.synchronize()
    if fa.fa_get_device_error() != fa.FA_OK:
        raise RuntimeError("e4m3 timed region: device error")
    ms = e[0].elapsed_time(e[1]) / K
    bf16_ms = e[1].elapsed_time(e[2]) / K
    qk8_ms = e[2].elapsed_time(e[4]) / K
    flops = fwd_flops(w)
    value = flops / (ms * 1e-3) / 1e12
    # end to end: q8, k8, v in from pinned host memory, O and LSE out
    pin = [q8.pin_memory(), k8.pin_memory(), (v8 if pv8 else host["v"]).pin_memory()]
    dst = [torch.empty_like(q8d), torch.empty_like(k8d), torch.empty_like(v8d if pv8 else v)]
    oh = torch.empty(o.shape, dtype=o.dtype, pin_memory=True)
    lh = torch.empty(lse.shape, dtype=lse.dtype, pin_memory=True)
    Ke = max(4, min(K, 20))
    e[0].record(s)
    for _ in range(Ke):
        for a, b in zip(pin, dst):
            b.copy_(a, non_blocking=True)
        if pv8:
            fa.attention_forward_fp8(dst[0], dst[1], dst[2], qs, ks, vs, causal, scale, out=o,
                                     lse=lse)
        else:
            fa.attention_forward_qk8(dst[0], dst[1], dst[2], qs, ks, causal, scale, out=o,
                                     lse=lse)
        oh.copy_(o, non_blocking=True)
        lh.copy_(lse, non_blocking=True)
    e[3].record(s)
    torch.cuda.synchronize()
    e2e = flops / (e[0].elapsed_time(e[3]) / Ke * 1e-3) / 1e12
    peaks = load_peaks()
    mixed_peak = peaks["bf16_tflops"] * (2.0 if pv8 else 4.0 / 3.0)
    cpu = None
    if not args.no_cpu_baseline:
        val, tcpu, heads, cores = oracle_whole_heads(w, 20.0)
        cpu = {"value": val / 3.5, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
               "sample": f"oracle ref_fwd + ref_bwd on {heads} whole heads, {tcpu:.1f} s, "
                         f"credited the forward's share of the FLOPs"}
    print(json.dumps({
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": 1, "steps": K,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "e4m3 QK^T and PV" if pv8 else "e4m3 QK^T, bf16 PV",
        "data": "synthetic",
        "config": dict(workload_config(w, wname), **{"pass": "fwd", "quant": "per-tensor e4m3 "
                       + ("Q, K, V" if pv8 else "Q, K") + " (descale = amax / 448)",
                       "l2": f"no flush: per-step working set {(2 + 4) * B * H * N * d / 1e6:.0f} MB"}),
        "bf16_fwd_tflops": flops / (bf16_ms * 1e-3) / 1e12,
        "qk8_fwd_tflops": flops / (qk8_ms * 1e-3) / 1e12,
        "speedup_vs_bf16": bf16_ms / ms,
        "roofline": {"kernel": "fa_fwd_kernel<128, causal, e4m3" + (" QK and PV>" if pv8
                                                                    else " QK>"),
                     "bound": "tensor",
                     "achieved": value, "peak": mixed_peak, "unit": "TFLOP/s",
                     "frac": value / mixed_peak,
                     "peak_source": f"{peaks['source']} bf16 burst x " + (
                         "2 (all FLOPs at the nominal 2x e4m3 rate)" if pv8 else
                         "4/3 (half the FLOPs at the nominal 2x e4m3 rate)"), "traffic": None},
        "cpu_baseline": cpu,
        "e2e": {"value": e2e, "unit": "TFLOP/s",
                "h2d_bytes_per_step": sum(t.numel() * t.element_size() for t in pin),
                "d2h_bytes_per_step": oh.numel() * 2 + lh.numel() * 4},
        "gpu_launches": K, "clocks": clk.summary()}), flush=True)
    return 0


# ---------------------------------------------------------------- bias


def bias_arm(args, w, wname):
    """One step = fa_fwd_bias + fa_bwd_bias (with dBias), timed beside the
    plain fa_fwd + fa_bwd on the same q, k, v, dO.  TFLOP/s by the same
    convention; the bias adds HBM traffic (the bias read in both passes,
    dBias written), reported as bias_bytes_per_step."""
    import torch

    import exact_attention_109_b200 as fa
    from exact_attention_109_b200.inputs import attention_inputs, default_scale

    if int(os.environ.get("WORLD_SIZE", "1")) > 1:
        print(json.dumps({"metric": METRIC, "error": "bias workloads run on one GPU"}))
        return 1
    torch.cuda.set_device(0)
    B, H, N, d, causal = w["B"], w["H"], w["N"], w["d"], w["causal"]
    scale = default_scale(d)
    host = attention_inputs(B, H, N, d, w["seed"], w["dist"], with_dout=True)
    q, k, v, dO = (host[x].cuda() for x in ("q", "k", "v", "dO"))
    g = torch.Generator().manual_seed(w["seed"] + 7)
    bias = (torch.randn((1, H, N, N), generator=g) * 2).to(torch.bfloat16).cuda()
    ws = torch.empty(fa.fa_bwd_workspace_size(B, H, N, d), dtype=torch.uint8, device="cuda")
    s = torch.cuda.current_stream()

    ob, lb = fa.attention_forward_bias(q, k, v, bias, causal, scale)

    def fwd_only():
        fa.attention_forward_bias(q, k, v, bias, causal, scale, out=ob, lse=lb)

    def bwd_only():
        fa.attention_backward_bias(q, k, v, bias, ob, lb, dO, causal, scale, workspace=ws)

    def step():
        fwd_only()
        bwd_only()

    def plain_step():
        o, lse = fa.attention_forward(q, k, v, causal, scale)
        fa.attention_backward(q, k, v, o, lse, dO, causal, scale, workspace=ws)

    for _ in range(args.warmup):
        step()
        plain_step()
    torch.cuda.synchronize()
    K = args.steps
    e = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    with ClockSampler(0) as clk:
        time.sleep(0.3)
        torch.cuda.synchronize()
        e[0].record(s)
        for _ in range(K):
            step()
        e[1].record(s)
        for _ in range(K):
            plain_step()
        e[2].record(s)
        torch.cuda.synchronize()
    f = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    f[0].record(s)
    for _ in range(K):
        fwd_only()
    f[1].record(s)
    for _ in range(K):
        bwd_only()
    f[2].record(s)
    torch.cuda.synchronize()
    if fa.fa_get_device_error() != fa.FA_OK:
        raise RuntimeError("bias timed region: device error")
    ms, plain_ms = e[0].elapsed_time(e[1]) / K, e[1].elapsed_time(e[2]) / K
    pass_ms = {"fwd_bias": f[0].elapsed_time(f[1]) / K, "bwd_bias": f[1].elapsed_time(f[2]) / K}
    flops = 3.5 * fwd_flops(w)
    value = flops / (ms * 1e-3) / 1e12
    frac_causal = 0.5 if causal else 1.0
    bias_bytes = int(B * H * N * N * 2 * frac_causal * 3)  # read twice, dBias written once
    peaks = load_peaks()
    cpu = None
    if not args.no_cpu_baseline:
        val, tcpu, heads, cores = oracle_whole_heads(w, 20.0)
        cpu = {"value": val, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
               "sample": f"oracle ref_fwd + ref_bwd (without the bias term) on {heads} whole "
                         f"heads, {tcpu:.1f} s"}
    print(json.dumps({
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": 1, "steps": K,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": dict(workload_config(w, wname), **{
            "pass": "fwd+bwd with additive bias", "bias": f"[1, {H}, {N}, {N}] bf16",
            "l2": "no flush: per-step working set > 126 MB"}),
        "plain_fwd_bwd_tflops": flops / (plain_ms * 1e-3) / 1e12,
        "bias_overhead": ms / plain_ms - 1.0, "bias_bytes_per_step": bias_bytes,
        "pass_ms": pass_ms,
        "roofline": {"kernel": "whole step (fa_fwd_kernel, fa_bwd_main_kernel with bias)",
                     "bound": "tensor", "achieved": value, "peak": peaks["bf16_tflops"],
                     "unit": "TFLOP/s", "frac": value / peaks["bf16_tflops"],
                     "peak_source": f"{peaks['source']} (burst)", "traffic": None},
        "cpu_baseline": cpu, "e2e": None, "gpu_launches": 4 * K,
        "clocks": clk.summary()}), flush=True)
    return 0


SWEEP_CASES = ([(16384 // n, 32 if d == 64 else 16, n, d, c, "normal", 2)
                for n in (512, 1024, 2048, 4096, 8192, 16384) for d in (64, 128)
                for c in (False, True)]
               + [(8, 16, 2048, 128, True, "row_scaled", 4),
                  (2, 20, 8192, 128, True, "row_scaled", 5),
                  (1, 16, 65536, 128, True, "normal", 3)])


def measure_sweep(warmup: int, device_index: int = 0, min_ms: float = 150.0):
    """The whole kernel sweep of the pages' benchmark on one GPU: the 16k-token
    shapes (B*N = 16384, width 2048) for d = 64 and 128, both masks, the two
    GPT-layer shapes (row-scaled inputs) and the N = 65536 sequence, forward
    and backward through the C ABI (fa_fwd, fa_bwd) with preallocated outputs
    and workspace, inputs drawn on the device.  Per shape: TFLOP/s of the forward,
    the backward (2.5x the forward's FLOPs) and both, the forward and backward
    call times in ms (each the median of three CUDA-event-timed runs of R
    calls, R chosen so a run lasts at least `min_ms` / 3), and the SM clock
    sampled during those runs.  Every shape's working set exceeds L2."""
    import numpy as np
    import torch
    import exact_attention_109_b200 as fa
    from exact_attention_109_b200.inputs import attention_inputs_device, default_scale
    rows = []
    for (B, H, N, d, causal, dist, seed) in SWEEP_CASES:
        dev = attention_inputs_device(B, H, N, d, seed, dist=dist)
        q, k, v, dO = dev["q"], dev["k"], dev["v"], dev["dO"]
        sc = default_scale(d)
        ws = torch.empty(fa.fa_bwd_workspace_size(B, H, N, d), dtype=torch.uint8, device="cuda")
        o = torch.empty_like(q)
        lse = torch.empty(B, H, N, device="cuda")
        dq, dk, dv = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)

        stream = torch.cuda.current_stream().cuda_stream
        P = {x: t.data_ptr() for x, t in dict(q=q, k=k, v=v, dO=dO, o=o, lse=lse, dq=dq, dk=dk,
                                             dv=dv, ws=ws).items()}
        nws = ws.numel()

        def fwd():
            st = fa.fa_fwd(P["q"], P["k"], P["v"], P["o"], P["lse"], B, H, N, d, causal, sc,
                           stream)
            if st != fa.FA_OK:
                raise fa.FaError(st, "sweep fa_fwd")

        def bwd():
            st = fa.fa_bwd(P["q"], P["k"], P["v"], P["o"], P["lse"], P["dO"], P["dq"], P["dk"],
                           P["dv"], B, H, N, d, causal, sc, P["ws"], nws, stream)
            if st != fa.FA_OK:
                raise fa.FaError(st, "sweep fa_bwd")

        for _ in range(max(3, warmup)):
            fwd()
            bwd()
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        ev[0].record()
        fwd()
        bwd()
        ev[1].record()
        torch.cuda.synchronize()
        reps = max(3, int(math.ceil(min_ms / 3 / max(ev[0].elapsed_time(ev[1]), 1e-3))))
        tf, tb = [], []
        with ClockSampler(device_index) as clk:
            time.sleep(0.25)
            for _ in range(3):
                ev[0].record()
                for _ in range(reps):
                    fwd()
                ev[1].record()
                for _ in range(reps):
                    bwd()
                ev[2].record()
                torch.cuda.synchronize()
                tf.append(ev[0].elapsed_time(ev[1]) / reps)
                tb.append(ev[1].elapsed_time(ev[2]) / reps)
        status = fa.fa_get_device_error()
        if status != fa.FA_OK:
            raise fa.FaError(status, "sweep")
        fl = 4.0 * B * H * N * N * d * (0.5 if causal else 1.0)
        f_ms, b_ms = float(np.median(tf)), float(np.median(tb))
        cl = clk.summary()
        rows.append({"B": B, "H": H, "N": N, "d": d, "causal": causal, "inputs": dist,
                     "fwd_tflops": round(fl / f_ms / 1e9, 1),
                     "bwd_tflops": round(2.5 * fl / b_ms / 1e9, 1),
                     "fwd_bwd_tflops": round(3.5 * fl / (f_ms + b_ms) / 1e9, 1),
                     "fwd_ms": round(f_ms, 4), "bwd_ms": round(b_ms, 4), "calls": reps,
                     "clocks": {"sm_mhz": cl["sm_mhz"], "reasons": cl["reasons"],
                                "samples": cl["samples"]}})
        del dev, q, k, v, dO, ws, o, lse, dq, dk, dv
    return rows


def sweep_arm(args):
    """--sweep: print the sweep, one JSON line per shape (not the benchmark
    contract's single line)."""
    import torch
    torch.cuda.set_device(0)
    for row in measure_sweep(args.warmup):
        print(json.dumps(row), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS) + sorted(DECODE_WORKLOADS)
                    + sorted(RING_WORKLOADS) + sorted(QK8_WORKLOADS)
                    + sorted(BIAS_WORKLOADS),
                    default=DEFAULT_WORKLOAD)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-sweep", action="store_true",
                    help="leave the per-shape sweep out of the one-GPU line")
    ap.add_argument("--sweep", action="store_true",
                    help="time the whole shape sweep (one JSON line per shape) and exit")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)  # at least three untimed warm-up steps
    if args.sweep:
        return sweep_arm(args)
    if args.workload in BIAS_WORKLOADS:
        if args.impl == "reference":
            return reference_arm(args, BIAS_WORKLOADS[args.workload], args.workload)
        return bias_arm(args, BIAS_WORKLOADS[args.workload], args.workload)
    if args.workload in QK8_WORKLOADS:
        if args.impl == "reference":
            return reference_arm(args, QK8_WORKLOADS[args.workload], args.workload)
        return qk8_arm(args, QK8_WORKLOADS[args.workload], args.workload)
    if args.workload in RING_WORKLOADS:
        if args.impl == "reference":
            return reference_arm(args, RING_WORKLOADS[args.workload], args.workload)
        return ring_arm(args, RING_WORKLOADS[args.workload], args.workload)
    if args.workload in DECODE_WORKLOADS:
        w = DECODE_WORKLOADS[args.workload]
        if args.impl == "reference":
            return decode_reference_arm(args, w, args.workload)
        return decode_arm(args, w, args.workload)
    w = WORKLOADS[args.workload]
    if args.impl == "reference":
        return reference_arm(args, w, args.workload)
    return gpu_arm(args, w, args.workload)


if __name__ == "__main__":
    sys.exit(main())
