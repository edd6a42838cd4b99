"""GPU parity of gdn_rope_3d (through the C ABI) against the fp64 oracle's 3D RoPE.

Bar: every element within 2^-8 of the oracle's value, relative, plus 1e-5 of the input's largest
magnitude. The kernel rotates in f32 with angles computed in double precision and rounds to
bf16 once (2^-9 relative); the absolute term covers results that cancel to near zero."""
import numpy as np
import pytest
import torch

import gdn_inputs
import oracle

pytestmark = pytest.mark.gpu


def api():
    from frame_wise_gated_deltanet_b200 import api as a
    return a


def f64(t):
    return t.detach().to(torch.float32).cpu().numpy().astype(np.float64)


def check(got, x, ref):
    g, r = f64(got), ref
    bound = 2.0 ** -8 * np.abs(r) + 1e-5 * float(np.abs(f64(x)).max())
    bad = np.abs(g - r) > bound
    assert not bad.any(), f"{int(bad.sum())} elements off, max err {float(np.abs(g - r).max()):.3e}"


SHAPES = [
    # (B, T, H, D, grid_h, grid_w, base, t_offset)
    (1, 3, 2, 128, 4, 5, 10000.0, 0),
    (2, 2, 3, 64, 3, 3, 10000.0, 7),
    (1, 4, 1, 8, 2, 2, 100.0, 0),        # smallest head dim: 4 / 2 / 2
    (1, 2, 2, 96, 1, 7, 500.0, 300),     # one grid row
    (1, 1, 4, 120, 6, 1, 10000.0, 960),  # one grid column, a late frame
]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "B%dT%dH%dD%d_g%dx%d_t%d" % (s[:6] + (s[7],)))
def test_rope_matches_oracle(shape):
    B, T, H, D, gh, gw, base, toff = shape
    x = gdn_inputs.clip_inputs(B, H, T, gh * gw, D, seed=60 + D)["q"]
    ref = oracle.rope_3d(f64(x), gh, gw, base, toff)
    got = api().gdn_rope_3d(x.cuda(), gh, gw, base, toff)
    assert api().gdn_sync_status() == 0
    check(got, x, ref)


def test_rope_in_place():
    x = gdn_inputs.clip_inputs(1, 2, 3, 20, 128, seed=70)["k"].cuda()
    ref = api().gdn_rope_3d(x, 4, 5, t_offset=2)
    y = x.clone()
    out = api().gdn_rope_3d(y, 4, 5, t_offset=2, out=y)
    assert out.data_ptr() == y.data_ptr()
    assert torch.equal(y, ref)


def test_rope_720p_sampled_frames():
    """The 720p clip's q (B1 T961 N880 H20 D128, 22 x 40 grid) in one call; the oracle recomputes
    three frames, including the last, with t_offset set to their frame index."""
    w = gdn_inputs.WORKLOADS["720p"]
    x = gdn_inputs.workload_inputs(w, device="cuda")["q"]
    got = api().gdn_rope_3d(x, 22, 40)
    assert api().gdn_sync_status() == 0
    for t in (0, 481, w.T - 1):
        xs = x[:, t:t + 1]
        ref = oracle.rope_3d(f64(xs), 22, 40, 10000.0, t)
        check(got[:, t:t + 1], xs, ref)
