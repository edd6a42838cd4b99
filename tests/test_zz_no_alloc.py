"""gdn_frame_forward_noalloc, the entry point for callers that must not allocate device memory
(for example code running inside a server or framework that owns every device allocation
through its own pool, or a real-time loop that cannot afford the device-wide synchronisation a
growing workspace implies). It runs the regular forward's kernels on a fixed scratch array the
library reserves on each GPU, so its results must match gdn_frame_forward.

This file is collected last on purpose, and passes both alone in a fresh process and after the
other GPU tests.
"""
import math

import numpy as np
import pytest
import torch

import gdn_inputs

pytestmark = pytest.mark.gpu

O_TOL = 1e-2
S_TOL = 5e-3


def _relf(a, b):
    a = a.detach().float().cpu().numpy().astype(np.float64)
    b = b.detach().float().cpu().numpy().astype(np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def _noalloc(lib, x, out, st, B, H, T, N, D, ks):
    s = x["state"]
    return lib.gdn_frame_forward_noalloc(
        x["q"].data_ptr(), x["k"].data_ptr(), x["v"].data_ptr(), x["gamma"].data_ptr(),
        x["beta"].data_ptr(), None if s is None else s.data_ptr(), out.data_ptr(), st.data_ptr(),
        B, H, T, N, D, ks, torch.cuda.current_stream().cuda_stream)


def test_noalloc_matches_forward_on_two_calls_in_a_row():
    from frame_wise_gated_deltanet_b200 import _lib, api
    lib = _lib.LIB
    B, H, T, N, D = 1, 4, 12, 300, 128
    ks = 1.0 / math.sqrt(D * N)
    # two different problems: the second call must not depend on what the first left behind
    xs = []
    for seed, std in ((21, 0.2), (22, 0.0)):
        x = gdn_inputs.clip_inputs(B, H, T, N, D, seed=seed, state_std=std)
        xs.append({k: (None if v is None else v.cuda()) for k, v in x.items()})
    refs = [api.gdn_frame_forward(x["q"], x["k"], x["v"], x["gamma"], x["beta"], x["state"],
                                  key_scale=ks) for x in xs]
    outs = [(torch.empty_like(x["q"]), torch.empty((B, H, D, D), device="cuda")) for x in xs]
    for x, (o, s) in zip(xs, outs):  # two calls in a row
        assert _noalloc(lib, x, o, s, B, H, T, N, D, ks) == 0
    assert api.gdn_sync_status() == 0
    for (ro, rs), (o, s) in zip(refs, outs):
        assert _relf(o, ro) <= O_TOL
        assert _relf(s, rs) <= S_TOL


def test_noalloc_rejects_problems_beyond_its_scratch():
    from frame_wise_gated_deltanet_b200 import _lib
    lib = _lib.LIB
    # the 720p clip needs 2.5 GB of scratch; the check happens on the host before any launch
    p = 1 << 20
    rc = lib.gdn_frame_forward_noalloc(p, 2 * p, 3 * p, 4 * p, 5 * p, None, 6 * p, None,
                                       1, 20, 961, 880, 128, 0.003, None)
    assert rc == 7
    assert b"64 MiB" in lib.gdn_status_string(7)
