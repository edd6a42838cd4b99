"""gdn_frame_forward_noalloc, the entry point for callers that must not allocate device memory
(for example code running inside a server or framework that owns every device allocation
through its own pool, or a real-time loop that cannot afford the device-wide synchronisation a
growing workspace implies). It runs the regular forward's kernels on a fixed scratch array the
library reserves on each GPU, so its results must match the fp64 oracle and gdn_frame_forward.

This file is collected last on purpose, and passes both alone in a fresh process and after the
other GPU tests.
"""
import math
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

import gdn_inputs
import oracle

pytestmark = pytest.mark.gpu

O_TOL = 1e-2
S_TOL = 5e-3
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _np(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def _relf(a, b):
    a = a if isinstance(a, np.ndarray) else _np(a)
    b = b if isinstance(b, np.ndarray) else _np(b)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def _noalloc(lib, x, out, st, B, H, T, N, D, ks):
    s = x["state"]
    return lib.gdn_frame_forward_noalloc(
        x["q"].data_ptr(), x["k"].data_ptr(), x["v"].data_ptr(), x["gamma"].data_ptr(),
        x["beta"].data_ptr(), None if s is None else s.data_ptr(), out.data_ptr(), st.data_ptr(),
        B, H, T, N, D, ks, torch.cuda.current_stream().cuda_stream)


# Problems run back to back on the one shared scratch: D = 128 first fills every byte of the
# per-frame state tiles, so the later D = 96 call (state tiles padded from 96 to 128) and the
# D = 64 call (its own tile size) must write, not inherit, whatever they read back.
CASES = [
    # (B, H, T, N, D, seed, state std)
    (1, 4, 12, 300, 128, 21, 0.2),
    (1, 4, 12, 300, 128, 22, 0.0),
    (2, 3, 7, 129, 96, 23, 0.3),
    (1, 5, 9, 200, 64, 24, 0.1),
    (1, 2, 6, 77, 96, 25, 0.0),
]


def test_noalloc_matches_oracle_and_forward_on_calls_in_a_row():
    from frame_wise_gated_deltanet_b200 import _lib, api
    lib = _lib.LIB
    runs = []
    for B, H, T, N, D, seed, std in CASES:
        x = gdn_inputs.clip_inputs(B, H, T, N, D, seed=seed, state_std=std)
        g = {k: (None if v is None else v.cuda()) for k, v in x.items()}
        ks = 1.0 / math.sqrt(D * N)
        out = torch.empty_like(g["q"])
        st = torch.empty((B, H, D, D), device="cuda")
        runs.append((x, g, out, st, ks, (B, H, T, N, D)))
    for x, g, out, st, ks, dims in runs:  # calls in a row on the shared scratch
        assert _noalloc(lib, g, out, st, *dims, ks) == 0
    assert api.gdn_sync_status() == 0
    for x, g, out, st, ks, dims in runs:
        o_ref, s_ref = oracle.gdn_frame_forward(
            _np(x["q"]), _np(x["k"]), _np(x["v"]), _np(x["gamma"]), _np(x["beta"]),
            None if x["state"] is None else _np(x["state"]), ks)
        eo, es = _relf(out, o_ref), _relf(st, s_ref)
        assert eo <= O_TOL and es <= S_TOL, f"{dims}: O err {eo:.2e}, S err {es:.2e}"
        ro, rs = api.gdn_frame_forward(g["q"], g["k"], g["v"], g["gamma"], g["beta"], g["state"],
                                       key_scale=ks)
        torch.cuda.synchronize()
        assert _relf(out, ro) <= O_TOL and _relf(st, rs) <= S_TOL, dims


_CHILD = r"""
import math, sys, torch
sys.path.insert(0, sys.argv[1])
import gdn_inputs
from frame_wise_gated_deltanet_b200 import _lib, api
lib = _lib.LIB
B, H, T, N, D = 1, 4, 96, 256, 128            # three-kernel workspace: 384 x 128 KiB = 48 MiB
x = gdn_inputs.clip_inputs(B, H, T, N, D, seed=31, device="cuda")
out = torch.empty_like(x["q"]); st = torch.empty((B, H, D, D), device="cuda")
ks = 1.0 / math.sqrt(D * N)
assert api.gdn_sync_status() == 0             # loads the library's module (and its scratch)
torch.cuda.synchronize()
free0 = torch.cuda.mem_get_info()[0]
for _ in range(2):
    assert lib.gdn_frame_forward_noalloc(
        x["q"].data_ptr(), x["k"].data_ptr(), x["v"].data_ptr(), x["gamma"].data_ptr(),
        x["beta"].data_ptr(), None, out.data_ptr(), st.data_ptr(), B, H, T, N, D, ks,
        torch.cuda.current_stream().cuda_stream) == 0
assert api.gdn_sync_status() == 0
free1 = torch.cuda.mem_get_info()[0]
# the regular entry point on the same problem (three-kernel path, into the same outputs) grows
# its cached workspace: the measurement sees it
assert lib.gdn_set_forward_mode(1) == 0
api.gdn_frame_forward(x["q"], x["k"], x["v"], x["gamma"], x["beta"], None, out, st, key_scale=ks)
assert api.gdn_sync_status() == 0
free2 = torch.cuda.mem_get_info()[0]
print(free0 - free1, free1 - free2)
"""


def test_noalloc_allocates_nothing_in_a_fresh_process():
    """In a fresh process, after the library's module is loaded: two allocation-free calls leave
    the device's free memory unchanged (within a few MiB the driver may take for launch
    resources), while one gdn_frame_forward of the same problem takes its 48 MiB workspace."""
    r = subprocess.run([sys.executable, "-c", _CHILD, ROOT], capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr
    used_noalloc, used_forward = (int(v) for v in r.stdout.split()[-2:])
    mib = 1 << 20
    assert used_noalloc <= 4 * mib, f"noalloc calls took {used_noalloc / mib:.1f} MiB"
    assert used_forward >= 40 * mib, f"forward took only {used_forward / mib:.1f} MiB"


def test_noalloc_rejects_problems_beyond_its_scratch():
    from frame_wise_gated_deltanet_b200 import _lib
    lib = _lib.LIB
    # the 720p clip needs 2.5 GB of scratch; the check happens on the host before any launch
    p = 1 << 20
    rc = lib.gdn_frame_forward_noalloc(p, 2 * p, 3 * p, 4 * p, 5 * p, None, 6 * p, None,
                                       1, 20, 961, 880, 128, 0.003, None)
    assert rc == 7
    assert b"64 MiB" in lib.gdn_status_string(7)
