"""Failure detection on the GPU without a fault: a bounded device-side wait that runs out.

The fused forward's chain waits for the statistics of every frame. The test hook
GDN_TEST_WITHHOLD_FRAME makes the statistics role skip publishing one frame of head 0, i.e. the
flag the chain waits on is never set. With a short wait limit the kernel must give up, unwind
and report GDN_ERR_TIMEOUT through gdn_sync_status; afterwards the CUDA context must still be
usable (a three-kernel forward on the same inputs matches the oracle). Runs in a child process
because the library reads its environment once.
"""
import os
import subprocess
import sys
import textwrap

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = textwrap.dedent("""
    import math, sys
    import numpy as np, torch
    sys.path.insert(0, {root!r})
    import gdn_inputs, oracle
    from frame_wise_gated_deltanet_b200 import _lib, api
    B, H, T, N, D = 1, 2, 8, 64, 64
    x = gdn_inputs.clip_inputs(B, H, T, N, D, seed=77)
    g = {{k: (None if v is None else v.cuda()) for k, v in x.items()}}
    ks = 1.0 / math.sqrt(D * N)
    assert _lib.LIB.gdn_set_forward_mode(2) == 0
    api.gdn_frame_forward(g["q"], g["k"], g["v"], g["gamma"], g["beta"], key_scale=ks)
    status = api.gdn_sync_status()
    print("fused status", status)
    assert status == 6, status
    assert api.gdn_sync_status() == 0  # the status word was cleared
    assert _lib.LIB.gdn_set_forward_mode(1) == 0
    out, st = api.gdn_frame_forward(g["q"], g["k"], g["v"], g["gamma"], g["beta"], key_scale=ks)
    assert api.gdn_sync_status() == 0
    f64 = lambda t: t.float().cpu().numpy().astype(np.float64)
    o_ref, s_ref = oracle.gdn_frame_forward(f64(x["q"]), f64(x["k"]), f64(x["v"]),
                                            f64(x["gamma"]), f64(x["beta"]), None, ks)
    eo = np.linalg.norm(f64(out) - o_ref) / np.linalg.norm(o_ref)
    assert eo <= 1e-2, eo
    print("OK")
""")


def test_withheld_flag_times_out_and_context_survives():
    env = dict(os.environ, GDN_TEST_WITHHOLD_FRAME="3", GDN_WAIT_LIMIT_MS="300")
    r = subprocess.run([sys.executable, "-c", CHILD.format(root=ROOT)], env=env,
                       capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and "OK" in r.stdout, r.stdout + r.stderr
