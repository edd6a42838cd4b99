"""GPU parity of the 3D RoPE (through the C ABI) against the fp64 oracle.

gdn_rope_3d (the standalone pass): every element within 2^-8 of the oracle's value, relative,
plus 1e-5 of the input's largest magnitude. The kernel rotates in f32 with angles computed in
double precision and rounds to bf16 once (2^-9 relative); the absolute term covers results that
cancel to near zero.

gdn_frame_forward_rope (the rotation fused into the layer's kernels): against the oracle's
rope_3d of q and k followed by the oracle's forward, with the layer's bars (relative Frobenius
error of the output <= 1e-2, of the final state <= 5e-3); the rotated operands carry one more
bf16 rounding (2^-9 relative per element), which the sums over tokens average down.
"""
import math
import os

import numpy as np
import pytest
import torch

import gdn_inputs
import oracle

from tests import parity_util as pu

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


def test_rope_720p_sampled_frames_and_norms():
    """The 720p clip's q (B1 T961 N880 H20 D128, 22 x 40 grid) in one call; the oracle recomputes
    eight frames, including the first and the last, with t_offset set to their frame index. Over
    the whole tensor, each pair's rotation preserves its length (checked per token and head: the
    norms of the rotated and the original rows agree to the bf16 rounding)."""
    w = gdn_inputs.WORKLOADS["720p"]
    x = gdn_inputs.workload_inputs(w, device="cuda")["q"]
    got = api().gdn_rope_3d(x, 22, 40)
    assert api().gdn_sync_status() == 0
    for t in (0, 1, 97, 300, 481, 700, 959, w.T - 1):
        xs = x[:, t:t + 1]
        ref = oracle.rope_3d(f64(xs), 22, 40, 10000.0, t)
        check(got[:, t:t + 1], xs, ref)
    for t0 in range(0, w.T, 64):  # every frame, in slices of 64 frames
        a = x[:, t0:t0 + 64].float().norm(dim=-1)
        b = got[:, t0:t0 + 64].float().norm(dim=-1)
        assert float(((b - a).abs() / a.clamp_min(1e-6)).max()) <= 2.0 ** -7


# ------------------------------------------------------------ the prologue fused into the layer

O_TOL = 1e-2
S_TOL = 5e-3


@pytest.fixture
def forward_mode(request):
    """gdn_set_forward_mode(mode) for one test (1 three kernels, 2 fused, 3 chunked with chunks
    of 3 frames)."""
    from frame_wise_gated_deltanet_b200 import _lib
    assert _lib.LIB.gdn_set_forward_mode(request.param) == 0
    old = os.environ.get("GDN_CHUNK_LEN")
    os.environ["GDN_CHUNK_LEN"] = "3"
    try:
        yield request.param
    finally:
        _lib.LIB.gdn_set_forward_mode(0)
        if old is None:
            os.environ.pop("GDN_CHUNK_LEN", None)
        else:
            os.environ["GDN_CHUNK_LEN"] = old


def relf(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


FWD_SHAPES = [
    # (B, H, T, grid_h, grid_w, D, base, t_offset, with_state)
    (1, 2, 5, 10, 20, 128, 10000.0, 0, True),    # N = 200: two tiles, the second ragged
    (2, 3, 4, 3, 43, 112, 10000.0, 17, False),   # N = 129: a one-token tail; padded head dim
    (1, 3, 6, 15, 26, 64, 10000.0, 0, True),     # the 480p grid; 64-dim operand tiles
    (1, 1, 3, 1, 1, 128, 500.0, 5, True),        # one token per frame
    (1, 2, 20, 4, 8, 32, 10000.0, 0, False),     # many frames, small head dim
    (1, 2, 7, 11, 12, 96, 10000.0, 950, True),   # late frames of a resumed clip
    # grids past the kernels' 32 KB shared-memory copy of the table's grid-row and grid-column
    # entries (256 bytes per grid row and per grid column): read from the table in global memory
    (1, 2, 3, 2, 150, 128, 10000.0, 0, True),
    (1, 2, 3, 1, 320, 64, 10000.0, 3, False),
]


@pytest.mark.parametrize("forward_mode", [1, 2, 3], indirect=True, ids=["split", "fused", "chunked"])
@pytest.mark.parametrize("shape", FWD_SHAPES, ids=lambda s: "B%dH%dT%d_g%dx%d_D%d_t%d" % (s[:6] + (s[7],)))
def test_forward_rope_matches_oracle(shape, forward_mode):
    B, H, T, gh, gw, D, base, toff, with_state = shape
    N = gh * gw
    x = gdn_inputs.clip_inputs(B, H, T, N, D, seed=1200 + N + D, state_std=0.3 if with_state else 0.0)
    ks = 1.0 / math.sqrt(D * N)
    g = {k: (None if v is None else v.cuda()) for k, v in x.items()}
    out, st = api().gdn_frame_forward_rope(g["q"], g["k"], g["v"], g["gamma"], g["beta"], gh, gw,
                                           base, toff, state_in=g["state"], key_scale=ks)
    assert api().gdn_sync_status() == 0
    qr = oracle.rope_3d(f64(x["q"]), gh, gw, base, toff)
    kr = oracle.rope_3d(f64(x["k"]), gh, gw, base, toff)
    o_ref, s_ref = oracle.gdn_frame_forward(qr, kr, f64(x["v"]), f64(x["gamma"]), f64(x["beta"]),
                                            None if x["state"] is None else f64(x["state"]), ks)
    eo, es = relf(f64(out), o_ref), relf(f64(st), s_ref)
    assert eo <= O_TOL and es <= S_TOL, f"O err {eo:.2e}, S err {es:.2e}"


@pytest.mark.parametrize("forward_mode", [1, 2], indirect=True, ids=["split", "fused"])
def test_forward_rope_equals_rope_then_forward(forward_mode):
    """The fused prologue rotates exactly as the standalone pass does (same table, same f32
    arithmetic, same bf16 rounding), so it equals gdn_rope_3d of q and k followed by
    gdn_frame_forward on the same path, up to the f32 contraction order of the rotation."""
    B, H, T, gh, gw, D = 1, 3, 9, 13, 17, 128
    x = gdn_inputs.clip_inputs(B, H, T, gh * gw, D, seed=1300, state_std=0.2, device="cuda")
    a = api()
    out, st = a.gdn_frame_forward_rope(x["q"], x["k"], x["v"], x["gamma"], x["beta"], gh, gw,
                                       t_offset=4, state_in=x["state"])
    qr = a.gdn_rope_3d(x["q"], gh, gw, t_offset=4)
    kr = a.gdn_rope_3d(x["k"], gh, gw, t_offset=4)
    o2, s2 = a.gdn_frame_forward(qr, kr, x["v"], x["gamma"], x["beta"], x["state"])
    torch.cuda.synchronize()
    assert a.gdn_sync_status() == 0
    assert relf(f64(out), f64(o2)) <= 2e-3 and relf(f64(st), f64(s2)) <= 2e-4


def test_forward_rope_720p_all_heads():
    """The 720p clip (22 x 40 grid) through the fused prologue in the benchmark's launch
    configuration; the oracle rotates q and k and recomputes every head over all 961 frames."""
    w = gdn_inputs.WORKLOADS["720p"]
    g = gdn_inputs.workload_inputs(w, device="cuda")
    out, st = api().gdn_frame_forward_rope(g["q"], g["k"], g["v"], g["gamma"], g["beta"], 22, 40,
                                           key_scale=w.key_scale)
    assert api().gdn_sync_status() == 0

    def one(h):
        sl = lambda t: pu.f32(t[:, :, :, h:h + 1])
        qr = oracle.rope_3d(sl(g["q"]), 22, 40)
        kr = oracle.rope_3d(sl(g["k"]), 22, 40)
        o_ref, s_ref = oracle.gdn_frame_forward(qr, kr, sl(g["v"]), pu.f32(g["gamma"][:, :, h:h + 1]),
                                                pu.f32(g["beta"][:, :, h:h + 1]), None, w.key_scale)
        del qr, kr
        eo, es = pu.RelF(), pu.RelF()
        eo.add(sl(out), o_ref, h)
        es.add(pu.f32(st[:, h:h + 1]), s_ref, h)
        return eo, es

    eo, es = pu.RelF(), pu.RelF()
    for a, b in pu.pool_map(one, range(w.H), bytes_per_task=8e9):
        eo.merge(a)
        es.merge(b)
    pu.log("rope_720p_all_heads", out=eo, state=es)
    assert eo.value <= O_TOL and es.value <= S_TOL, (
        f"O err {eo.value:.2e} (worst head {eo.worst_at}: {eo.worst:.2e}), S err {es.value:.2e}")
