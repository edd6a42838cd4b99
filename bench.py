#!/usr/bin/env python
"""Benchmark of the frame-wise Gated DeltaNet layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl gdn|reference]

One step = one gdn_frame_forward over the 720p 60 s clip (B1 H20 D128 T961 N880, 22x40 latent
grid, synthetic seeded bf16 inputs resident in HBM). Prints one JSON line (rank 0).

* value: whole-job tokens*heads/s = (units all ranks processed) / (max over ranks of the
  device time of K steps, CUDA events on the launching stream).
* e2e: the same metric through the C ABI's host-buffer entry point with pinned HOST buffers:
  every step copies q, k, v, gamma, beta host->device and out and the final state back.
* roofline: the dominant kernel (largest share of the timed region, timed live with CUDA
  events the library records around each of its launches) against the measured HBM copy
  bandwidth; traffic from the committed ncu summary when the kernel sources still match it.
* cpu_baseline: the fp64 oracle on a bounded sample of the same workload (rank 0, N = 1).
* --impl reference: the oracle itself as the reference arm (host cores, bounded samples).
* --backward: one step = one gdn_frame_backward (the gradients for a seeded d_out) instead of
  the forward; no e2e leg.
* --rope: one step = gdn_rope_3d of the clip's q and k in place; no e2e or CPU-baseline leg.

Multi-GPU (torchrun): every rank processes its own clip (independent problems, no collective
on the data path), so scaling is weak.
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
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "GDN layer tokens·heads/sec and % of roofline (720p 60 s config, 1 B200)"
METRIC_BWD = "GDN layer backward tokens·heads/sec (720p 60 s config, 1 B200)"
METRIC_ROPE = "3D RoPE of q and k, tokens·heads/sec (720p 60 s config, 1 B200)"
METRIC_ROPE_FUSED = "GDN layer with fused 3D RoPE of q and k, tokens·heads/sec (720p 60 s config, 1 B200)"
METRIC_SOFTMAX = "chunk-causal softmax attention tokens·heads/sec and % of bf16 tensor peak (1 B200)"
UNIT = "tokens*heads/s"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0


def args_parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="gdn", choices=["gdn", "reference"])
    ap.add_argument("--workload", default="720p")
    ap.add_argument("--frames", type=int, default=0,
                    help="truncate the clip to its first FRAMES frames (small profiling cases)")
    ap.add_argument("--heads", type=int, default=0,
                    help="override the workload's head count (scaling studies)")
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--fp8", action="store_true",
                    help="E4M3 q, k, v with per-(frame, head) scales (gdn_frame_forward_fp8)")
    ap.add_argument("--backward", action="store_true",
                    help="time gdn_frame_backward (the training pass) instead of the forward")
    ap.add_argument("--backward-saved", action="store_true",
                    help="with --backward: time gdn_frame_backward_saved, reading the A_t, B_t, "
                         "S_t that one gdn_frame_forward_train call kept (outside the timed region)")
    ap.add_argument("--rope", action="store_true",
                    help="time gdn_rope_3d on the clip's q and k (in place) instead of the forward")
    ap.add_argument("--rope-fused", action="store_true",
                    help="time gdn_frame_forward_rope (the forward with the 3D RoPE of q and k "
                         "fused into its kernels) instead of the forward")
    ap.add_argument("--no-workloads", action="store_true",
                    help="skip the other configurations' records (480p, stream, LA, fp8, "
                         "backward, RoPE) that the default 720p run adds to its line")
    ap.add_argument("--shard", default="none", choices=["none", "heads"],
                    help="under torchrun: 'heads' splits one clip's heads over the ranks "
                         "(strong scaling) instead of one clip per rank (weak scaling)")
    ap.add_argument("--forward-mode", type=int, default=0,
                    help="gdn_set_forward_mode: 0 auto, 1 three kernels, 2 fused, 3 chunked")
    a = ap.parse_args()
    a.backward = a.backward or a.backward_saved
    return a


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


def tensor_peak():
    """Dense bf16 tensor peak in TFLOP/s: the measured burst figure (a kernel timed alone), else
    the recipe's fallback."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["bf16_tflops"]), "measured dense bf16 (cuBLAS, burst)"
    except (OSError, KeyError, ValueError):
        return FALLBACK_BF16_TFLOPS, "fallback dense bf16"


def softmax_flops(B, H, T, N, D, F):
    """Algorithmic flops of chunk-causal softmax attention: 2*D for a query-key score and 2*D
    for its share of P V, over every visible (query, key) pair."""
    pairs = sum(N * min(T, (t // F + 1) * F) * N for t in range(T))
    return B * H * 4 * D * pairs


def algorithmic_bytes(w, fp8=False):
    """Bytes the layer must move per call: Q, K, V read (bf16, or E4M3 plus three f32 scales per
    frame-head) and O written (bf16), gamma and beta, the fp32 state written, and read when the
    call starts from a carried state."""
    fh = w.B * w.H * w.T
    state = w.B * w.H * w.D * w.D * 4
    if w.kind == "la":
        return fh * (4 * w.N * w.D * 2) + state + w.B * w.H * w.D * 4
    qkv = fh * (3 * w.N * w.D + 3 * 4) if fp8 else fh * 3 * w.N * w.D * 2
    return (qkv + fh * w.N * w.D * 2 + w.B * w.T * w.H * 2 * 4 + state
            + (state if w.kind == "stream" else 0))


def backward_bytes(w):
    """Bytes the backward must move per call: Q, K, V, dO read and dQ, dK, dV written (bf16),
    gamma and beta read, d_gamma and d_beta written, the fp32 S_0 read and dS_0 written."""
    fh = w.B * w.H * w.T
    state = w.B * w.H * w.D * w.D * 4
    return fh * 7 * w.N * w.D * 2 + w.B * w.T * w.H * 4 * 4 + 2 * state


def rope_bytes(w):
    """Bytes of the 3D RoPE prologue per call: q and k read and written (bf16)."""
    return w.B * w.H * w.T * 4 * w.N * w.D * 2


def kernel_bytes(name, w, fp8=False):
    """Algorithmic bytes per launch of each kernel of the forward (the bytes its stage must
    move in the three-kernel design)."""
    fh = w.B * w.H * w.T
    nd2 = w.N * w.D * 2
    if fp8:
        if name == "gdn_stats_kernel":     # read K, V (E4M3); write A_t (bf16) and B_t (f32)
            return fh * (2 * w.N * w.D + w.D * w.D * 6 + 8)
        if name == "gdn_output_kernel":    # read Q (E4M3), S_t; write O (bf16)
            return fh * (w.N * w.D + nd2 + w.D * w.D * 2 + 4)
        if name == "gdn_fused_kernel":
            return algorithmic_bytes(w, True)
    dd = w.D * w.D
    if name == "gdn_rope_kernel":        # one tensor read and written
        return fh * 2 * nd2
    if name == "gdn_bwd_token_kernel_dkdv":  # read V, K, G_t, W'_t; write dK, dV
        return fh * (4 * nd2 + 2 * dd * 2)
    if name == "gdn_bwd_token_kernel_dqe":  # read dO, Q, S_t; write dQ and E_t (f32)
        return fh * (3 * nd2 + dd * 2 + dd * 4)
    if name.startswith("gdn_bwd_token_kernel_d"):  # read X tiles and frame matrices; write out
        terms = 2 if name.endswith("_dk") else 1
        return fh * ((terms + 1) * nd2 + terms * dd * 2)
    if name == "gdn_bwd_chain_kernel":   # read A_t, E_t, gamma, beta; write G_t (bf16), dS_0
        return fh * (dd * 2 + dd * 4 + dd * 2 + 8) + w.B * w.H * dd * 4
    if name == "gdn_bwd_frame_kernel":   # read S_{t-1}, G_t, A_t, B_t; write W'_t, dgamma, dbeta
        return fh * (dd * 2 * 3 + dd * 4 + dd * 2 + 16)
    if name == "gdn_stats_kernel":       # read K, V; write A_t (bf16) and B_t (f32)
        return fh * (2 * nd2 + dd * 2 + dd * 4)
    if name == "gdn_chain_kernel":       # read A_t, B_t, gamma, beta; write S_t (bf16), S_T
        return fh * (dd * 2 + dd * 4 + dd * 2 + 8) + w.B * w.H * dd * 4
    if name == "gdn_output_kernel":      # read Q, S_t (per block for LA); write O
        if w.kind == "la":
            nblk = -(-w.T // w.frames_per_block)
            return fh * 2 * nd2 + w.B * w.H * nblk * (w.D + 1) * w.D * 2
        return fh * (2 * nd2 + dd * 2)
    if name in ("gdn_fused_kernel", "gdn_step_kernel"):  # the whole path in one launch
        return algorithmic_bytes(w)
    if w.kind == "la":
        nblk = -(-w.T // w.frames_per_block)
        sums = w.B * w.H * nblk * (w.D + 1) * w.D
        if name == "gdn_stats_kernel_la":   # read K, V; write the per-block f32 sums
            return fh * 2 * nd2 + sums * 4
        if name == "gdn_la_scan_kernel":    # read the sums; write bf16 block states, (S, z)
            return sums * (4 + 2) + w.B * w.H * (w.D + 1) * w.D * 4
    return None


def per_launch_bytes(name, w, fp8, backward, steps, launches):
    """Algorithmic bytes per launch: the kernel's bytes per step over its launches per step. The
    backward's statistics kernel makes two full passes per step, (k, v) and (q, dO); its
    segmented kernels split one pass over several launches."""
    kb = kernel_bytes(name, w, fp8)
    if not kb or launches < 1:
        return None
    # (the RoPE step rotates q and k: two launches of one full pass each)
    passes = 2 if ((backward and name == "gdn_stats_kernel") or name == "gdn_rope_kernel") else 1
    return kb * passes * steps / launches


# Sources each kernel is built from: an ncu traffic figure stays valid while these are unchanged.
KERNEL_SOURCES = {
    "gdn_fused_kernel": ["fused_kernel.cuh", "chain_kernel.cuh", "stats_kernel.cuh",
                         "output_kernel.cuh", "rope_kernel.cuh", "common.cuh", "ptx.cuh"],
    "gdn_step_kernel": ["step_kernel.cuh", "common.cuh", "ptx.cuh"],
    "gdn_stats_kernel": ["stats_kernel.cuh", "rope_kernel.cuh", "common.cuh", "ptx.cuh"],
    "gdn_stats_kernel_la": ["stats_kernel.cuh", "rope_kernel.cuh", "common.cuh", "ptx.cuh"],
    "gdn_output_kernel": ["output_kernel.cuh", "rope_kernel.cuh", "common.cuh", "ptx.cuh"],
    "gdn_rope_kernel": ["rope_kernel.cuh", "common.cuh", "ptx.cuh"],
    "gdn_softmax_kernel": ["softmax_kernel.cuh", "common.cuh", "ptx.cuh"],
    "gdn_chain_kernel": ["chain_kernel.cuh", "common.cuh", "ptx.cuh"],
    "gdn_scan_kernel": ["scan_kernel.cuh", "common.cuh", "ptx.cuh"],
    "gdn_bwd_chain_kernel": ["bwd_chain_kernel.cuh", "common.cuh", "ptx.cuh"],
    "gdn_bwd_frame_kernel": ["bwd_frame_kernel.cuh", "common.cuh", "ptx.cuh"],
    "gdn_bwd_token_kernel_dq": ["bwd_token_kernel.cuh", "common.cuh", "ptx.cuh"],
    "gdn_bwd_token_kernel_dv": ["bwd_token_kernel.cuh", "common.cuh", "ptx.cuh"],
    "gdn_bwd_token_kernel_dk": ["bwd_token_kernel.cuh", "common.cuh", "ptx.cuh"],
    "gdn_bwd_token_kernel_dkdv": ["bwd_token_kernel.cuh", "common.cuh", "ptx.cuh"],
    "gdn_bwd_token_kernel_dqe": ["bwd_token_kernel.cuh", "common.cuh", "ptx.cuh"],
}


def source_digest(kernel=None):
    """sha256 prefix of the kernel's source files (all of csrc/ when the kernel is unknown)."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "frame_wise_gated_deltanet_b200", "csrc")
    files = KERNEL_SOURCES.get(kernel) or sorted(os.listdir(csrc))
    for f in files:
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(f.encode() + fh.read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel, workload):
    """DRAM bytes per launch of `kernel` from profiles/traffic.json, if it was taken on the
    kernel's current sources and on this workload; else None."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            t = json.load(f)
        entries = t["kernels"][kernel]
        for e in entries if isinstance(entries, list) else [entries]:
            if e.get("source_digest") == source_digest(kernel) and e.get("workload") == workload:
                return float(e["dram_bytes_per_launch"])
        return None
    except (OSError, KeyError, ValueError, TypeError):
        return None


class ClockSampler:
    """nvidia-smi clock/throttle samples of one GPU while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_uuid):
        self.uuid = gpu_uuid
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.uuid, "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        self.t0 = time.time()

    def stop(self):
        self.t1 = time.time()
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.1)
        self.proc.terminate()
        self.proc.wait()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        # the sampler ran from just before to just after the timed region; keep loaded samples
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        smax = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i] == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None, "reasons": reasons,
                "samples": len(rows)}


def dist_setup():
    import torch
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x, world, device="cuda"):
    """Largest value of x over all ranks (the job's time is its slowest rank's)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank, ms_local, world, device="cuda"):
    """Whole-job throughput: every rank processed units_per_rank units; the job took the slowest
    rank's device time. Returns (units per second, max ms)."""
    ms = max_over_ranks(ms_local, world, device)
    return units_per_rank * world / (ms * 1e-3), ms


def oracle_sample_rate(w, heads, frames, seed=99, backward=False):
    """The fp64 oracle on a bounded sample of workload `w` (`heads` heads, `frames` frames, same
    token count and head dim), forward or backward. Returns (tokens*heads/s, seconds, threads)."""
    import numpy as np
    import gdn_inputs
    import oracle
    x = gdn_inputs.clip_inputs(1, heads, frames, w.N, w.D, w.gamma_range, w.beta_range, seed=seed)
    f = lambda t: t.float().numpy()
    args = [f(x["q"]), f(x["k"]), f(x["v"]), f(x["gamma"]), f(x["beta"])]
    if backward:
        c = gdn_inputs.cotangents(1, heads, frames, w.N, w.D, seed=seed + 1)
    t0 = time.perf_counter()
    if backward:
        oracle.gdn_frame_backward(*args, None, f(c["d_out"]), None, w.key_scale)
    else:
        oracle.gdn_frame_forward(*args, None, w.key_scale)
    dt = time.perf_counter() - t0
    try:
        import threadpoolctl
        threads = max(i.get("num_threads", 1) for i in threadpoolctl.threadpool_info())
    except Exception:  # noqa: BLE001
        threads = os.cpu_count()
    return heads * frames * w.N / dt, dt, threads


def host_info():
    """The host's usable cores (affinity mask) and CPU model, for the CPU baseline's record."""
    cores = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()
    model = ""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"host_cores": cores, "cpu_model": model}


def run_reference(a, w):
    """The oracle as the reference arm: each step is a bounded sample (1 head x 192 frames)."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    heads, frames = 1, 192
    for _ in range(a.warmup):
        oracle_sample_rate(w, heads, frames)
    rates, secs, threads = [], 0.0, 1
    for _ in range(a.steps):
        r, dt, threads = oracle_sample_rate(w, heads, frames)
        rates.append(r)
        secs += dt
    units = a.steps * heads * frames * w.N
    value = units / secs
    sample = f"{heads} head x {frames} frames of the {w.name} clip (N={w.N}, D={w.D}) per step"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": world, "steps": a.steps, "warmup": a.warmup,
        "ms_per_step": secs / a.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(w),
        "cpu_baseline": dict({"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                              "sample": sample}, **host_info()),
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))


def workload_config(w, shard=False, world=1):
    what = {"stream": "streaming step", "la": "block-causal LA clip"}.get(w.kind, "GDN clip")
    par = ("one clip's heads split over %d GPUs (contiguous head ranges, no collective)" % world
           if shard else "independent clip per GPU")
    return {"workload": f"{w.name} {what}: B{w.B} H{w.H} D{w.D} T{w.T} N{w.N} ({w.grid} grid)",
            "B": w.B, "H": w.H, "D": w.D, "T": w.T, "N": w.N, "key_scale": w.key_scale,
            "gamma_range": list(w.gamma_range), "beta_range": list(w.beta_range),
            "l2": "inputs (%.1f GB of q,k,v) larger than the 126 MB L2; no flush"
                  % (3 * w.B * w.T * w.N * w.H * w.D * 2 / 1e9),
            "parallelism": par}


def main():
    a = args_parse()
    import dataclasses
    import gdn_inputs
    w = gdn_inputs.WORKLOADS[a.workload]
    if a.frames > 0:
        w = dataclasses.replace(w, T=a.frames, name=f"{w.name}[:{a.frames}]")
    if a.heads > 0:
        w = dataclasses.replace(w, H=a.heads, name=f"{w.name}[H={a.heads}]")
    if a.impl == "reference":
        run_reference(a, w)
        return

    import torch
    from frame_wise_gated_deltanet_b200 import _lib, api

    world, rank, local = dist_setup()
    dev = torch.device("cuda", local)
    # --shard heads: the ranks split one clip's heads (strong scaling; per-rank byte counts use
    # the rank's own heads); otherwise every rank runs its own clip (weak scaling)
    shard = a.shard == "heads" and world > 1
    if a.shard == "heads" and (w.kind != "gdn" or a.fp8 or a.backward or a.rope or a.rope_fused):
        raise ValueError("--shard heads applies to the bf16 forward of a GDN clip")
    w_rank = w
    if shard:
        from frame_wise_gated_deltanet_b200.parallel import head_range
        h0, h1 = head_range(w.H, world, rank)
        if h1 == h0:
            raise ValueError(f"--shard heads: rank {rank} of {world} would own no head of {w.H}")
        w_rank = dataclasses.replace(w, H=h1 - h0, name=f"{w.name}[heads {h0}:{h1}]")
    if _lib.LIB.gdn_set_forward_mode(a.forward_mode) != 0:
        raise ValueError(f"invalid --forward-mode {a.forward_mode}")
    stream = torch.cuda.current_stream(dev)
    if w.kind == "stream":
        # one streaming step per bench step: a new frame for every stream, state in place
        g = gdn_inputs.workload_inputs(w, device=dev, step=0)
        q, k, v = (g[n][:, 0].contiguous() for n in ("q", "k", "v"))
        gam, bet = g["gamma"][:, 0].contiguous(), g["beta"][:, 0].contiguous()
        st = gdn_inputs.workload_inputs(w, device=dev)["state"].contiguous()
        out = torch.empty_like(q)
        g = {"q": q, "k": k, "v": v, "gamma": gam, "beta": bet}

        def step():
            api.gdn_frame_step(q, k, v, gam, bet, st, out, st, key_scale=w.key_scale,
                               stream=stream)
    elif w.kind == "la":
        # block-causal linear attention over the clip
        g = gdn_inputs.workload_inputs(w, device=dev)
        q, k, v = g["q"], g["k"], g["v"]
        out = torch.empty_like(q)
        st = torch.empty((w.B, w.H, w.D, w.D), dtype=torch.float32, device=dev)
        zt = torch.empty((w.B, w.H, w.D), dtype=torch.float32, device=dev)

        def step():
            api.gdn_block_causal_la(q, k, v, w.frames_per_block, out=out, state_out=st,
                                    z_out=zt, stream=stream)
    elif a.fp8:
        # E4M3 q, k, v with one absmax scale per (batch, frame, head)
        g = gdn_inputs.workload_inputs(w, device=dev)
        f8 = {}
        for n in ("q", "k", "v"):
            f8[n], f8["s" + n] = gdn_inputs.quantize_e4m3(g[n])
        out = torch.empty_like(g["q"])
        del g["q"], g["k"], g["v"]
        gam, bet = g["gamma"], g["beta"]
        st = torch.empty((w.B, w.H, w.D, w.D), dtype=torch.float32, device=dev)

        def step():
            api.gdn_frame_forward_fp8(f8["q"], f8["k"], f8["v"], f8["sq"], f8["sk"], f8["sv"],
                                      gam, bet, None, out, st, key_scale=w.key_scale,
                                      stream=stream)
    elif w.kind == "softmax":
        # chunk-causal softmax attention of the hybrid blocks over the clip's tokens
        g = gdn_inputs.workload_inputs(w, device=dev)
        q, k, v = g["q"], g["k"], g["v"]
        out = torch.empty_like(q)
        st = None

        def step():
            api.gdn_softmax_attention(q, k, v, w.frames_per_block, out=out, stream=stream)
    elif a.rope_fused:
        # the forward with the 3D RoPE of q and k fused into its statistics and output kernels
        g = gdn_inputs.workload_inputs(w, device=dev)
        q, k, v, gam, bet = g["q"], g["k"], g["v"], g["gamma"], g["beta"]
        gh, gw = (int(x) for x in w.grid.split("x"))
        out = torch.empty_like(q)
        st = torch.empty((w.B, w.H, w.D, w.D), dtype=torch.float32, device=dev)

        def step():
            api.gdn_frame_forward_rope(q, k, v, gam, bet, gh, gw, out=out, state_out=st,
                                       key_scale=w.key_scale, stream=stream)
    elif a.rope:
        # the 3D RoPE prologue of the clip's q and k, in place (22 x 40 latent grid at 720p)
        g = gdn_inputs.workload_inputs(w, device=dev)
        q, k = g["q"], g["k"]
        gh, gw = (int(x) for x in w.grid.split("x"))
        out = st = None

        def step():
            api.gdn_rope_3d(q, gh, gw, out=q, stream=stream)
            api.gdn_rope_3d(k, gh, gw, out=k, stream=stream)
    elif a.backward:
        # the training pass: gradients of the clip for seeded cotangents of the output
        g = gdn_inputs.workload_inputs(w, device=dev)
        q, k, v, gam, bet = g["q"], g["k"], g["v"], g["gamma"], g["beta"]
        d_out = gdn_inputs.cotangents(w.B, w.H, w.T, w.N, w.D, seed=w.seed + 50,
                                      device=dev)["d_out"]
        out = st = None

        if a.backward_saved:
            _, _, saved = api.gdn_frame_forward_train(q, k, v, gam, bet, key_scale=w.key_scale,
                                                      stream=stream)

            def step():
                api.gdn_frame_backward_saved(q, k, v, gam, bet, saved, d_out,
                                             key_scale=w.key_scale, stream=stream)
        else:
            def step():
                api.gdn_frame_backward(q, k, v, gam, bet, d_out, key_scale=w.key_scale,
                                       stream=stream)
    else:
        g = gdn_inputs.workload_inputs(w, device=dev)
        if shard:
            # this rank's heads of the one clip, as a column-parallel projection hands them over
            from frame_wise_gated_deltanet_b200.parallel import shard_heads
            g = {n: (None if t is None else
                     shard_heads(t, world, rank, {5: 3, 3: 2, 4: 1}[t.dim()]))
                 for n, t in g.items()}
            torch.cuda.empty_cache()
        q, k, v, gam, bet = g["q"], g["k"], g["v"], g["gamma"], g["beta"]
        out = torch.empty_like(q)
        st = torch.empty((w_rank.B, w_rank.H, w.D, w.D), dtype=torch.float32, device=dev)

        def step():
            api.gdn_frame_forward(q, k, v, gam, bet, None, out, st, key_scale=w.key_scale,
                                  stream=stream)

    for _ in range(max(a.warmup, 3)):
        step()
    torch.cuda.synchronize()
    # status checks are collective, so that every rank stops together
    if max_over_ranks(float(api.gdn_sync_status() != 0), world) > 0:
        raise RuntimeError("device status error during warm-up")

    # per-launch events the library records around each kernel (created before arming)
    n_ev = 2 * 16 * a.steps  # at most 16 launches per step
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(n_ev)]
    for e in evs:
        e.record(stream)
    import ctypes
    handles = (ctypes.c_void_p * n_ev)(*[e.cuda_event for e in evs])
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    props = torch.cuda.get_device_properties(dev)
    sampler = ClockSampler("GPU-" + str(props.uuid))

    torch.cuda.synchronize()
    barrier(world)
    _lib.LIB.gdn_profile_arm(handles, n_ev)
    sampler.start()
    t_start.record(stream)
    for _ in range(a.steps):
        step()
    t_end.record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    launches = _lib.LIB.gdn_profile_count()
    names = [_lib.LIB.gdn_profile_kernel(i).decode() for i in range(launches)]
    _lib.LIB.gdn_profile_arm(None, 0)
    barrier(world)
    status = api.gdn_sync_status()
    if max_over_ranks(float(status != 0), world) > 0:
        raise RuntimeError(f"device status {status} after the timed region (this rank)")

    ms_local = t_start.elapsed_time(t_end)
    if shard:  # one clip over all ranks: its units once, in the slowest rank's time
        ms = max_over_ranks(ms_local, world)
        value = w.tokens_heads * a.steps / (ms * 1e-3)
    else:
        value, ms = job_throughput(w.tokens_heads * a.steps, ms_local, world)
    w_all, w = w, w_rank  # per-rank byte accounting below
    per_kernel = {}
    for i, n in enumerate(names):
        d = evs[2 * i].elapsed_time(evs[2 * i + 1])
        tot, cnt = per_kernel.get(n, (0.0, 0))
        per_kernel[n] = (tot + d, cnt + 1)
    dom = max(per_kernel, key=lambda n: per_kernel[n][0])
    dom_ms = per_kernel[dom][0] / per_kernel[dom][1]
    hbm, peak_kind = peaks()
    kb = per_launch_bytes(dom, w, a.fp8, a.backward, a.steps, per_kernel[dom][1])
    achieved = kb / (dom_ms * 1e-3) / 1e9 if kb else None
    sm_flops = (softmax_flops(w.B, w.H, w.T, w.N, w.D, w.frames_per_block)
                if w.kind == "softmax" else None)
    path_bytes = (4 * w.B * w.T * w.N * w.H * w.D * 2 if w.kind == "softmax" else
                  rope_bytes(w) if a.rope else
                  backward_bytes(w) if a.backward else algorithmic_bytes(w, a.fp8))
    path_gbs = path_bytes / (ms / a.steps * 1e-3) / 1e9

    # ---------------------------------------------------------------- end to end, host buffers
    e2e = None
    if not a.no_e2e:
        e2e = (measure_e2e(a, w, g, out, st, stream, world, dev)
               if w.kind == "gdn" and not a.fp8 and not a.backward and not a.rope
               and not a.rope_fused else None)
        if shard and e2e and e2e.get("ms_per_step"):
            # the ranks' copies and computes cover one clip: its units in the slowest rank's time
            e2e["value"] = w_all.tokens_heads / (e2e["ms_per_step"] * 1e-3)

    workloads = None
    if (not a.no_workloads and world == 1 and w.kind == "gdn" and w.name == "720p" and not a.fp8
            and not a.backward and not a.rope and not a.rope_fused):
        sampler2 = ClockSampler("GPU-" + str(props.uuid))
        sampler2.start()
        workloads = measure_workloads(dev, stream, g)
        workloads["clocks"] = sampler2.stop()

    line = {
        "metric": (METRIC_ROPE if a.rope else METRIC_BWD if a.backward else
                   METRIC_ROPE_FUSED if a.rope_fused else METRIC),
        "value": value, "unit": UNIT,
        "n_gpus": world, "steps": a.steps,
        "warmup": a.warmup, "ms_per_step": ms / a.steps, "higher_is_better": True,
        "scaling": "strong" if shard else "weak", "vs_baseline": None,
        "dtype": "e4m3 q/k/v, bf16 out" if a.fp8 else "bf16", "data": "synthetic",
        "config": dict(workload_config(w_all, shard, world),
                       **({"backward": "saved states (gdn_frame_backward_saved)"
                           if a.backward_saved else "recomputed forward (gdn_frame_backward)"}
                          if a.backward else {})),
        "roofline": {
            "bound": "hbm", "kernel": dom, "achieved": achieved, "peak": hbm, "unit": "GB/s",
            "frac": (achieved / hbm) if achieved else None,
            "peak_source": f"{peak_kind} HBM copy bandwidth",
            "traffic": ncu_traffic(dom, w.name + ("+fp8" if a.fp8 else "")
                                   + ("+bwd" if a.backward else "")
                                   + ("+saved" if a.backward_saved else "")
                                   + ("+rope" if a.rope_fused else "")),
            "algorithmic_bytes_per_launch": kb, "ms_per_launch": dom_ms,
            "path": {"algorithmic_bytes_per_step": path_bytes, "achieved_gbs": path_gbs,
                     "frac": path_gbs / hbm},
        },
        "kernels": {n: {"launches": c, "ms_total": t, "share": t / sum(x[0] for x in per_kernel.values())}
                    for n, (t, c) in per_kernel.items()},
        "gpu_launches": launches,
        "clocks": clocks,
        "e2e": e2e,
    }
    if workloads is not None:
        line["workloads"] = workloads
    if sm_flops:
        # a contraction: measured against the dense bf16 tensor peak
        tp, tp_kind = tensor_peak()
        fpl = sm_flops * a.steps / per_kernel[dom][1]
        ktf = fpl / (dom_ms * 1e-3) / 1e12
        ptf = sm_flops / (ms / a.steps * 1e-3) / 1e12
        line["metric"] = METRIC_SOFTMAX
        line["roofline"] = {"bound": "tensor", "kernel": dom, "achieved": ktf, "peak": tp,
                            "unit": "TFLOP/s", "frac": ktf / tp, "peak_source": tp_kind,
                            "traffic": ncu_traffic(dom, w.name),
                            "algorithmic_flops_per_launch": fpl, "ms_per_launch": dom_ms,
                            "path": {"algorithmic_flops_per_step": sm_flops,
                                     "achieved_tflops": ptf, "frac": ptf / tp}}
    if (rank == 0 and world == 1 and not a.no_cpu_baseline and w.kind == "gdn" and not a.fp8
            and not a.rope and not a.rope_fused):
        heads = 1 if a.backward else 4
        rate, secs, threads = oracle_sample_rate(w, heads, w.T, backward=a.backward)
        line["cpu_baseline"] = dict({"value": rate, "unit": UNIT, "cores": threads,
                                     "kind": "oracle",
                                     "sample": f"{heads} head(s) x {w.T} frames of the {w.name} "
                                               f"clip shape (N={w.N}, D={w.D}), "
                                               f"{'backward' if a.backward else 'forward'}, "
                                               f"{secs:.1f} s of fp64 numpy"}, **host_info())
    if rank == 0:
        print(json.dumps(line))
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def timed(step, steps, stream, max_launches_per_step=16):
    """Run step() `steps` times between two CUDA events on `stream`, with the library's per-launch
    events armed. Returns (ms for all steps, {kernel: (ms total, launches)}, launches)."""
    import ctypes
    import torch
    from frame_wise_gated_deltanet_b200 import _lib
    n_ev = 2 * max_launches_per_step * steps
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(n_ev)]
    for e in evs:
        e.record(stream)  # creates the event
    handles = (ctypes.c_void_p * n_ev)(*[e.cuda_event for e in evs])
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    _lib.LIB.gdn_profile_arm(handles, n_ev)
    t0.record(stream)
    for _ in range(steps):
        step()
    t1.record(stream)
    torch.cuda.synchronize()
    launches = _lib.LIB.gdn_profile_count()
    names = [_lib.LIB.gdn_profile_kernel(i).decode() for i in range(launches)]
    _lib.LIB.gdn_profile_arm(None, 0)
    per_kernel = {}
    for i, n in enumerate(names):
        d = evs[2 * i].elapsed_time(evs[2 * i + 1])
        tot, cnt = per_kernel.get(n, (0.0, 0))
        per_kernel[n] = (tot + d, cnt + 1)
    return t0.elapsed_time(t1), per_kernel, launches


def rotating(copies):
    """A callable returning the next of `copies` on each call (inputs of a workload smaller than
    L2 rotate over enough copies that each step reads data no earlier step left in L2)."""
    state = {"i": -1}

    def nxt():
        state["i"] = (state["i"] + 1) % len(copies)
        return copies[state["i"]]
    return nxt


L2_BYTES = 126 * 1024 * 1024


def n_copies(bytes_per_step):
    """Copies of a workload's inputs so that the ones a step reads were last read two L2 sizes
    of traffic ago (1 when one copy is already larger than twice the L2)."""
    return max(1, -(-2 * L2_BYTES // max(bytes_per_step, 1)) + 1) if bytes_per_step < 2 * L2_BYTES else 1


def workload_record(label, w, step, stream, path_bytes, kernel_bytes_fn, units_per_step,
                    warmup=3, target_ms=400.0, max_steps=400, flops_per_step=None,
                    tensor_peak=None, l2_note="", launches_per_step=16):
    """Time one extra workload of the run: warm-up, then about target_ms of steps. Returns its
    record: ms per step, tokens*heads/s, the dominant kernel with its roofline fraction against
    the measured peak, and the whole path's fraction."""
    import torch
    from frame_wise_gated_deltanet_b200 import api
    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    if api.gdn_sync_status() != 0:
        raise RuntimeError(f"device status error in the {label} warm-up")
    ms1, _, _ = timed(step, 1, stream, launches_per_step)
    steps = int(max(3, min(max_steps, target_ms / max(ms1, 1e-3))))
    ms, per_kernel, launches = timed(step, steps, stream, launches_per_step)
    if api.gdn_sync_status() != 0:
        raise RuntimeError(f"device status error in the {label} timed region")
    hbm, peak_kind = peaks()
    dom = max(per_kernel, key=lambda n: per_kernel[n][0])
    dom_ms = per_kernel[dom][0] / per_kernel[dom][1]
    kb = kernel_bytes_fn(dom, per_kernel[dom][1], steps)
    step_ms = ms / steps
    rec = {
        "workload": w if isinstance(w, str) else workload_config(w)["workload"],
        "ms_per_step": step_ms,
        "tokens_heads_per_s": units_per_step / (step_ms * 1e-3),
        "steps": steps, "warmup": warmup,
        "gpu_launches": launches,
        "dominant_kernel": {"name": dom, "ms_per_launch": dom_ms,
                            "share": per_kernel[dom][0] / sum(t for t, _ in per_kernel.values())},
        "path": {"bound": "hbm", "algorithmic_bytes_per_step": path_bytes,
                 "achieved_gbs": path_bytes / (step_ms * 1e-3) / 1e9,
                 "peak_gbs": hbm, "frac": path_bytes / (step_ms * 1e-3) / 1e9 / hbm,
                 "peak_source": f"{peak_kind} HBM copy bandwidth"},
        "kernels": {n: {"launches": c, "ms_total": t} for n, (t, c) in per_kernel.items()},
        "l2": l2_note or "inputs larger than the 126 MB L2; no flush",
    }
    if kb:
        rec["dominant_kernel"].update(
            {"algorithmic_bytes_per_launch": kb, "achieved_gbs": kb / (dom_ms * 1e-3) / 1e9,
             "frac": kb / (dom_ms * 1e-3) / 1e9 / hbm})
    if flops_per_step and tensor_peak:
        tf = flops_per_step / (step_ms * 1e-3) / 1e12
        rec["path"] = {"bound": "tensor", "algorithmic_flops_per_step": flops_per_step,
                       "achieved_tflops": tf, "peak_tflops": tensor_peak[0],
                       "frac": tf / tensor_peak[0], "peak_source": tensor_peak[1]}
        fpl = flops_per_step * steps / per_kernel[dom][1]  # flops per launch of the kernel
        ktf = fpl / (dom_ms * 1e-3) / 1e12
        rec["dominant_kernel"].update({"algorithmic_flops_per_launch": fpl,
                                       "achieved_tflops": ktf, "frac": ktf / tensor_peak[0],
                                       "bound": "tensor"})
    return rec


def measure_workloads(dev, stream, g720=None):
    """The other configurations of the layer, timed in the same run as the contract line: the
    480p clip, the streaming workload (64 chained single-frame steps per step), the block-causal
    LA clip, and on the 720p clip the E4M3-input forward, the backward and the standalone 3D RoPE
    of q and k. Each record: ms per step, tokens*heads/s, the dominant kernel's and the path's
    fraction of the measured roofline."""
    import torch
    import gdn_inputs
    from frame_wise_gated_deltanet_b200 import api
    W = gdn_inputs.WORKLOADS
    recs = {}
    tok_bytes = lambda w: w.B * w.T * w.N * w.H * w.D * 2

    # ---- 480p clip (inputs smaller than L2: rotate over copies)
    w = W["480p"]
    base = gdn_inputs.workload_inputs(w, device=dev)
    inb = 3 * tok_bytes(w)
    nc = n_copies(inb)
    sets = []
    for _ in range(nc):
        c = {k: (None if v is None else v.clone()) for k, v in base.items()}
        sets.append((c, torch.empty_like(c["q"])))
    st = torch.empty((w.B, w.H, w.D, w.D), dtype=torch.float32, device=dev)
    nxt = rotating(sets)

    def step_480():
        c, o = nxt()
        api.gdn_frame_forward(c["q"], c["k"], c["v"], c["gamma"], c["beta"], None, o, st,
                              key_scale=w.key_scale, stream=stream)
    recs["480p"] = workload_record(
        "480p", w, step_480, stream, algorithmic_bytes(w),
        lambda n, l, s, w=w: per_launch_bytes(n, w, False, False, s, l), w.tokens_heads,
        l2_note=f"{nc} copies of the inputs ({inb / 1e6:.0f} MB of q,k,v each) rotated, so a "
                f"step's inputs were evicted from the 126 MB L2 by the steps before it")
    del base, sets

    # ---- streaming workload: one step = 64 chained gdn_frame_step calls, state in place
    w = W["stream"]
    frames = []
    for j in range(4):  # four distinct frames (216 MB of q,k,v each) cycled over the 64 calls
        x = gdn_inputs.workload_inputs(w, device=dev, step=j)
        frames.append({n: x[n][:, 0].contiguous() for n in ("q", "k", "v", "gamma", "beta")})
    state = gdn_inputs.workload_inputs(w, device=dev)["state"].contiguous()
    out_s = torch.empty_like(frames[0]["q"])

    def step_stream():
        for j in range(w.steps):
            f = frames[j % len(frames)]
            api.gdn_frame_step(f["q"], f["k"], f["v"], f["gamma"], f["beta"], state, out_s,
                               state, key_scale=w.key_scale, stream=stream)
    recs["stream"] = workload_record(
        "stream", f"streaming decode: {w.steps} chained gdn_frame_step calls of B{w.B} H{w.H} "
                  f"D{w.D} N{w.N} ({w.grid} grid), state in place",
        step_stream, stream, w.steps * algorithmic_bytes(w),
        lambda n, l, s, w=w: kernel_bytes(n, w), w.steps * w.tokens_heads,
        launches_per_step=w.steps + 4, target_ms=300.0)
    recs["stream"]["per_call_ms"] = recs["stream"]["ms_per_step"] / w.steps
    del frames, state, out_s

    # ---- block-causal LA clip
    w = W["la"]
    g = gdn_inputs.workload_inputs(w, device=dev)
    out_la = torch.empty_like(g["q"])
    st_la = torch.empty((w.B, w.H, w.D, w.D), dtype=torch.float32, device=dev)
    z_la = torch.empty((w.B, w.H, w.D), dtype=torch.float32, device=dev)

    def step_la():
        api.gdn_block_causal_la(g["q"], g["k"], g["v"], w.frames_per_block, out=out_la,
                                state_out=st_la, z_out=z_la, stream=stream)
    recs["la"] = workload_record(
        "la", w, step_la, stream, algorithmic_bytes(w),
        lambda n, l, s, w=w: per_launch_bytes(n, w, False, False, s, l), w.tokens_heads)
    del g, out_la

    # ---- 720p clip: fp8 inputs, backward, standalone 3D RoPE
    w = W["720p"]
    g = g720 if g720 is not None else gdn_inputs.workload_inputs(w, device=dev)
    f8 = {}
    for n in ("q", "k", "v"):
        f8[n], f8["s" + n] = gdn_inputs.quantize_e4m3(g[n])
    out8 = torch.empty_like(g["q"])
    st8 = torch.empty((w.B, w.H, w.D, w.D), dtype=torch.float32, device=dev)

    def step_fp8():
        api.gdn_frame_forward_fp8(f8["q"], f8["k"], f8["v"], f8["sq"], f8["sk"], f8["sv"],
                                  g["gamma"], g["beta"], None, out8, st8, key_scale=w.key_scale,
                                  stream=stream)
    recs["720p_fp8"] = workload_record(
        "720p_fp8", w.name + " clip, E4M3 q/k/v with per-(frame, head) scales", step_fp8,
        stream, algorithmic_bytes(w, True),
        lambda n, l, s, w=w: per_launch_bytes(n, w, True, False, s, l), w.tokens_heads,
        target_ms=150.0)
    del f8, out8

    d_out = gdn_inputs.cotangents(w.B, w.H, w.T, w.N, w.D, seed=w.seed + 50,
                                  device=dev)["d_out"]

    def step_bwd():
        api.gdn_frame_backward(g["q"], g["k"], g["v"], g["gamma"], g["beta"], d_out,
                               key_scale=w.key_scale, stream=stream)
    recs["720p_backward"] = workload_record(
        "720p_backward", w.name + " clip, gdn_frame_backward (dq, dk, dv, dgamma, dbeta, dS_0)",
        step_bwd, stream, backward_bytes(w),
        lambda n, l, s, w=w: per_launch_bytes(n, w, False, True, s, l), w.tokens_heads,
        target_ms=150.0)

    # the training pair: a forward that keeps A_t, B_t, S_t, and the backward that reads them
    _, _, saved = api.gdn_frame_forward_train(g["q"], g["k"], g["v"], g["gamma"], g["beta"],
                                              key_scale=w.key_scale, stream=stream)

    def step_bwd_saved():
        api.gdn_frame_backward_saved(g["q"], g["k"], g["v"], g["gamma"], g["beta"], saved,
                                     d_out, key_scale=w.key_scale, stream=stream)
    recs["720p_backward_saved"] = workload_record(
        "720p_backward_saved", w.name + " clip, gdn_frame_backward_saved (the backward reading "
                                        "the states gdn_frame_forward_train kept)",
        step_bwd_saved, stream, backward_bytes(w),
        lambda n, l, s, w=w: per_launch_bytes(n, w, False, False, s, l), w.tokens_heads,
        target_ms=150.0)
    out_t = torch.empty_like(g["q"])
    st_t = torch.empty((w.B, w.H, w.D, w.D), dtype=torch.float32, device=dev)

    def step_fwd_train():
        api.gdn_frame_forward_train(g["q"], g["k"], g["v"], g["gamma"], g["beta"], None, saved,
                                    out_t, st_t, key_scale=w.key_scale, stream=stream)
    recs["720p_forward_train"] = workload_record(
        "720p_forward_train", w.name + " clip, gdn_frame_forward_train (three kernels, A_t, B_t, "
                                       "S_t kept for the backward)",
        step_fwd_train, stream, algorithmic_bytes(w),
        lambda n, l, s, w=w: per_launch_bytes(n, w, False, False, s, l), w.tokens_heads,
        target_ms=150.0)
    del d_out, saved, out_t
    torch.cuda.empty_cache()

    gh, gw = (int(x) for x in w.grid.split("x"))
    qr, kr = torch.empty_like(g["q"]), torch.empty_like(g["k"])

    def step_rope():
        api.gdn_rope_3d(g["q"], gh, gw, out=qr, stream=stream)
        api.gdn_rope_3d(g["k"], gh, gw, out=kr, stream=stream)
    recs["720p_rope_standalone"] = workload_record(
        "720p_rope_standalone", w.name + " clip, gdn_rope_3d of q and k (out of place)",
        step_rope, stream, rope_bytes(w),
        lambda n, l, s, w=w: per_launch_bytes(n, w, False, False, s, l), w.tokens_heads,
        target_ms=150.0)
    del qr, kr
    torch.cuda.empty_cache()

    # ---- fused 3D RoPE prologue: the 720p forward with q and k rotated inside the kernels
    out_r = torch.empty_like(g["q"])
    st_r = torch.empty((w.B, w.H, w.D, w.D), dtype=torch.float32, device=dev)

    def step_rope_fused():
        api.gdn_frame_forward_rope(g["q"], g["k"], g["v"], g["gamma"], g["beta"], gh, gw,
                                   out=out_r, state_out=st_r, key_scale=w.key_scale,
                                   stream=stream)
    recs["720p_rope_fused"] = workload_record(
        "720p_rope_fused", w.name + " clip, gdn_frame_forward_rope (3D RoPE of q and k fused "
                                    "into the statistics and output kernels)",
        step_rope_fused, stream, algorithmic_bytes(w),
        lambda n, l, s, w=w: per_launch_bytes(n, w, False, False, s, l), w.tokens_heads,
        target_ms=150.0)
    del out_r
    if g720 is None:
        del g
    torch.cuda.empty_cache()

    # ---- chunk-causal softmax attention of the hybrid blocks (tensor-bound)
    for label in ("softmax_480p", "softmax_720p21"):
        ws = W[label]
        B, H, T, N, D, F = ws.B, ws.H, ws.T, ws.N, ws.D, ws.frames_per_block
        x = gdn_inputs.workload_inputs(ws, device=dev)
        o = torch.empty_like(x["q"])

        def step_sm(x=x, o=o, F=F):
            api.gdn_softmax_attention(x["q"], x["k"], x["v"], F, out=o, stream=stream)
        fl = softmax_flops(B, H, T, N, D, F)
        inb = 4 * B * T * N * H * D * 2
        recs[label] = workload_record(
            label, f"chunk-causal softmax attention B{B} H{H} D{D} T{T} N{N}, chunks of {F} "
                   f"frames (q, k, v, out {inb / 1e6:.0f} MB)",
            step_sm, stream, inb, lambda n, l, s: None, B * H * T * N, target_ms=200.0,
            flops_per_step=fl, tensor_peak=tensor_peak(),
            l2_note="compute-bound: K and V are meant to be re-read from L2 by a head's query "
                    "tiles; no flush")
        del x, o
    return recs


def measure_e2e(a, w, g, out, st, stream, world, dev):
    """Throughput through the C ABI's host-buffer entry point (gdn_frame_forward_host) with pinned
    host inputs and outputs: every step copies q, k, v, gamma, beta in and out, state out."""
    import torch
    from frame_wise_gated_deltanet_b200 import api
    # every rank takes the same decision (a rank that skipped would leave the others waiting
    # in the collectives below)
    short = 0.0
    try:
        import psutil
        need = sum(t.numel() * t.element_size() for t in (g["q"], g["k"], g["v"], out))
        short = 1.0 if psutil.virtual_memory().available < 1.5 * need * world else 0.0
    except ImportError:
        pass
    if max_over_ranks(short, world) > 0:
        return {"value": None, "unit": UNIT, "reason": "not enough host memory to pin"}
    host = {n: torch.empty(g[n].shape, dtype=g[n].dtype, pin_memory=True)
            for n in ("q", "k", "v", "gamma", "beta")}
    for n in host:
        host[n].copy_(g[n])
    out_h = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
    st_h = torch.empty(st.shape, dtype=st.dtype, pin_memory=True)

    def e2e_step():
        api.gdn_frame_forward_host(host["q"], host["k"], host["v"], host["gamma"], host["beta"],
                                   None, out_h, st_h, key_scale=w.key_scale, stream=stream,
                                   device=dev)

    e2e_step()
    torch.cuda.synchronize()
    if max_over_ranks(float(api.gdn_sync_status(stream) != 0), world) > 0:
        raise RuntimeError("device status error in the end-to-end leg")
    steps = max(1, a.e2e_steps)
    s0 = torch.cuda.Event(enable_timing=True)
    s1 = torch.cuda.Event(enable_timing=True)
    barrier(world)
    s0.record(stream)
    for _ in range(steps):
        e2e_step()
    s1.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(s0.elapsed_time(s1), world)
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = out_h.numel() * out_h.element_size() + st_h.numel() * st_h.element_size()
    return {"value": w.tokens_heads * world * steps / (ms * 1e-3), "unit": UNIT,
            "steps": steps, "ms_per_step": ms / steps, "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "api": "gdn_frame_forward_host (pinned host buffers, "
            "copies in, compute and copies out overlapped by frame segments)"}


if __name__ == "__main__":
    main()
