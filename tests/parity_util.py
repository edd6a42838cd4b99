"""Helpers of the GPU parity tests for whole-tensor comparisons at full workload sizes.

The oracle is run unchanged, one independent (batch, head) slice per call, on a pool of host
threads (numpy's matrix products release the GIL; each thread's BLAS is limited to one thread so
the slices run side by side). Errors are accumulated as sums of squares over every slice, so the
relative Frobenius error is the one of the whole output tensor of the workload.
"""
from __future__ import annotations

import json
import math
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import torch


def f32(t: torch.Tensor) -> np.ndarray:
    """A device or host tensor as a float32 numpy array (exact for bf16 and f32 values)."""
    return t.detach().to(torch.float32).cpu().numpy()


class RelF:
    """Relative Frobenius error ||got - ref|| / ||ref|| accumulated over slices, with the worst
    slice kept for the record."""

    def __init__(self):
        self.num = 0.0
        self.den = 0.0
        self.worst = 0.0
        self.worst_at = None

    def add(self, got, ref, where=None):
        got = np.asarray(got, dtype=np.float64)
        ref = np.asarray(ref, dtype=np.float64)
        n = float(np.sum((got - ref) ** 2))
        d = float(np.sum(ref ** 2))
        self.num += n
        self.den += d
        r = math.sqrt(n / max(d, 1e-300))
        if r >= self.worst:
            self.worst, self.worst_at = r, where

    def merge(self, other: "RelF"):
        self.num += other.num
        self.den += other.den
        if other.worst >= self.worst:
            self.worst, self.worst_at = other.worst, other.worst_at

    @property
    def value(self) -> float:
        return math.sqrt(self.num / max(self.den, 1e-300))


def workers(bytes_per_task: float) -> int:
    """Threads for the oracle: the host's cores, bounded so that the tasks in flight fit in about
    half of the available host memory."""
    cores = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()
    n = max(1, min(16, cores or 1))
    try:
        import psutil
        avail = psutil.virtual_memory().available
        n = max(1, min(n, int(0.5 * avail // max(bytes_per_task, 1.0))))
    except ImportError:
        pass
    return n


def pool_map(fn, items, bytes_per_task: float):
    """[fn(x) for x in items] on a thread pool, BLAS limited to one thread per worker."""
    items = list(items)
    try:
        from threadpoolctl import threadpool_limits
        limit = threadpool_limits(1)
    except ImportError:
        limit = None
    try:
        with ThreadPoolExecutor(workers(bytes_per_task)) as ex:
            return list(ex.map(fn, items))
    finally:
        if limit is not None:
            limit.restore_original_limits()


def log(name: str, **errors):
    """Append the measured errors of a full-size parity test to $GDN_PARITY_LOG (JSON lines), if
    set, so that a run's achieved errors can be recorded."""
    path = os.environ.get("GDN_PARITY_LOG")
    if not path:
        return
    rec = {"test": name}
    for k, v in errors.items():
        if isinstance(v, RelF):
            rec[k] = {"relF": v.value, "worst_slice": v.worst, "worst_at": str(v.worst_at)}
        else:
            rec[k] = v
    with open(path, "a") as f:
        f.write(json.dumps(rec) + "\n")
