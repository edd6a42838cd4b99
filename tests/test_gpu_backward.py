"""GPU parity of gdn_frame_backward (through the C ABI) against the fp64 oracle's backward, on
the same seeded inputs and cotangents.

Tolerances (relative Frobenius error): dq, dk, dv <= 1e-2; d_gamma, d_beta <= 2e-2;
d_state_in <= 5e-3. The kernels keep S_t, G_t = dL/dS_t and W'_t as bf16 operands (relative
rounding <= 2^-9 per element) and round dq, dk, dv to bf16, so about 2.5e-3 is expected; a
numpy model of exactly those roundings gives 1.6e-3 .. 3.7e-3 on these shapes. The scalar
gradients are sums of products of two rounded factors; d_state_in only carries the rounding of
the chain's bf16 operand, like the forward's final state.
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

GRAD_TOL = 1e-2
SCALAR_TOL = 2e-2
STATE_TOL = 5e-3


def api():
    from frame_wise_gated_deltanet_b200 import api as a
    return a


def f64(t):
    return t.detach().to(torch.float32).cpu().numpy().astype(np.float64)


def relf(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


SHAPES = [
    # (B, H, T, N, D, with_state)
    (1, 2, 5, 200, 128, True),
    (2, 1, 3, 96, 96, False),      # padded head dim, fewer tokens than one tile
    (1, 2, 1, 130, 128, True),     # one frame, ragged tail of two tokens
    (1, 1, 40, 64, 128, True),     # long chain
    (1, 3, 7, 300, 72, True),      # smallest supported head dim class, three tiles
    (2, 2, 4, 128, 120, False),    # exactly one tile
]


def check_against_oracle(x, c, got, ks, b_sl=slice(None), h_sl=slice(None)):
    """got = (dq, dk, dv, d_gamma, d_beta, d_state_in) from the GPU; compares the (batch, head)
    slices b_sl, h_sl (heads are independent) with the oracle on the same slices."""
    sl5 = lambda t: None if t is None else f64(t[b_sl, :, :, h_sl])
    sl3 = lambda t: f64(t[b_sl, :, h_sl])
    sl4 = lambda t: None if t is None else f64(t[b_sl, h_sl])
    ref = oracle.gdn_frame_backward(sl5(x["q"]), sl5(x["k"]), sl5(x["v"]), sl3(x["gamma"]),
                                    sl3(x["beta"]), sl4(x["state"]), sl5(c["d_out"]),
                                    sl4(c["d_state"]), ks)
    names = ["dq", "dk", "dv", "d_gamma", "d_beta", "d_state_in"]
    tols = [GRAD_TOL] * 3 + [SCALAR_TOL] * 2 + [STATE_TOL]
    gots = [sl5(got[0]), sl5(got[1]), sl5(got[2]), sl3(got[3]), sl3(got[4]), sl4(got[5])]
    errs = {n: relf(g, r) for n, g, r in zip(names, gots, ref)}
    for n, tol in zip(names, tols):
        assert np.all(np.isfinite(gots[names.index(n)])), f"{n} not finite"
        assert errs[n] <= tol, f"{n}: rel err {errs[n]:.2e} > {tol:.0e} (all: {errs})"
    return errs


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "B%dH%dT%dN%dD%d%s" % (s[:5] + ("s" if s[5] else "",)))
def test_backward_matches_oracle(shape):
    B, H, T, N, D, with_state = shape
    x = gdn_inputs.clip_inputs(B, H, T, N, D, gamma_range=(0.9, 0.999), beta_range=(0.05, 0.95),
                               seed=700 + T + D, state_std=0.3 if with_state else 0.0)
    c = gdn_inputs.cotangents(B, H, T, N, D, seed=800 + T + D, state_std=1.0 if with_state else 0.0)
    ks = 1.0 / math.sqrt(D * N)
    g = {k: (None if v is None else v.cuda()) for k, v in x.items()}
    gc = {k: (None if v is None else v.cuda()) for k, v in c.items()}
    got = api().gdn_frame_backward(g["q"], g["k"], g["v"], g["gamma"], g["beta"], gc["d_out"],
                                   state_in=g["state"], d_state_out=gc["d_state"], key_scale=ks)
    assert api().gdn_sync_status() == 0
    check_against_oracle(x, c, got, ks)


SEGMENTED = [
    # (B, H, T, N, D, with_state, frames per segment of the reverse chain)
    (1, 2, 10, 150, 128, True, 3),   # segments of 4, 4 and 2 frames
    (2, 1, 7, 64, 96, False, 2),     # a segment ending at frame 0 after carried ones
    (1, 3, 5, 200, 128, True, 1),    # one frame per segment
]


@pytest.mark.parametrize("shape", SEGMENTED, ids=lambda s: "B%dH%dT%dN%dD%d%s_seg%d" % (s[:5] + ("s" if s[5] else "", s[6])))
def test_backward_segmented_chain_matches_oracle(shape):
    """The reverse state chain in several launches (G carried in f32 between them), with each
    segment's per-frame and dk/dv passes on the second stream beside the next segment."""
    B, H, T, N, D, with_state, seg = shape
    old = os.environ.get("GDN_BWD_SEGMENT_FRAMES")
    os.environ["GDN_BWD_SEGMENT_FRAMES"] = str(seg)
    try:
        x = gdn_inputs.clip_inputs(B, H, T, N, D, seed=750 + T + seg,
                                   state_std=0.3 if with_state else 0.0)
        c = gdn_inputs.cotangents(B, H, T, N, D, seed=850 + T + seg,
                                  state_std=1.0 if with_state else 0.0)
        ks = 1.0 / math.sqrt(D * N)
        g = {k: (None if v is None else v.cuda()) for k, v in x.items()}
        gc = {k: (None if v is None else v.cuda()) for k, v in c.items()}
        got = api().gdn_frame_backward(g["q"], g["k"], g["v"], g["gamma"], g["beta"],
                                       gc["d_out"], state_in=g["state"],
                                       d_state_out=gc["d_state"], key_scale=ks)
        assert api().gdn_sync_status() == 0
    finally:
        if old is None:
            os.environ.pop("GDN_BWD_SEGMENT_FRAMES", None)
        else:
            os.environ["GDN_BWD_SEGMENT_FRAMES"] = old
    check_against_oracle(x, c, got, ks)


def test_backward_zero_cotangents_give_zero_gradients():
    """Linearity in the cotangents, at the ends: zero d_out and no d_state_out give exactly zero
    gradients (every kernel of the path multiplies or sums zeros only)."""
    B, H, T, N, D = 1, 2, 6, 140, 128
    x = gdn_inputs.clip_inputs(B, H, T, N, D, seed=901, state_std=0.3, device="cuda")
    zero = torch.zeros_like(x["q"])
    got = api().gdn_frame_backward(x["q"], x["k"], x["v"], x["gamma"], x["beta"], zero,
                                   state_in=x["state"])
    assert api().gdn_sync_status() == 0
    for t in got:
        assert float(t.abs().max()) == 0.0


def test_backward_state_gradient_aliases_its_cotangent():
    """d_state_in may be the memory of d_state_out (each element is read before it is written by
    the same thread): the result equals the one into separate memory."""
    B, H, T, N, D = 1, 2, 4, 100, 128
    x = gdn_inputs.clip_inputs(B, H, T, N, D, seed=902, state_std=0.3, device="cuda")
    c = gdn_inputs.cotangents(B, H, T, N, D, seed=903, state_std=1.0, device="cuda")
    a = api()
    ref = a.gdn_frame_backward(x["q"], x["k"], x["v"], x["gamma"], x["beta"], c["d_out"],
                               state_in=x["state"], d_state_out=c["d_state"])
    ds = c["d_state"].clone()
    from frame_wise_gated_deltanet_b200 import _lib
    outs = [torch.empty_like(x["q"]) for _ in range(3)] + [torch.empty_like(x["gamma"]) for _ in range(2)]
    with torch.cuda.device(x["q"].device):
        _lib.check("gdn_frame_backward", _lib.LIB.gdn_frame_backward(
            x["q"].data_ptr(), x["k"].data_ptr(), x["v"].data_ptr(), x["gamma"].data_ptr(),
            x["beta"].data_ptr(), x["state"].data_ptr(), c["d_out"].data_ptr(), ds.data_ptr(),
            outs[0].data_ptr(), outs[1].data_ptr(), outs[2].data_ptr(), outs[3].data_ptr(),
            outs[4].data_ptr(), ds.data_ptr(), B, H, T, N, D, 1.0 / math.sqrt(D * N),
            torch.cuda.current_stream().cuda_stream))
    assert a.gdn_sync_status() == 0
    assert torch.equal(ds, ref[5])
    for o, r in zip(outs, ref[:5]):
        assert torch.equal(o, r)


def test_backward_720p_all_heads():
    """The full 720p clip (B1 H20 T961 N880 D128) with random cotangents, one backward call in
    the launch configuration the benchmark times; the oracle recomputes the gradients of every
    head over all 961 frames (heads are independent), and the errors are those of the whole
    gradient tensors."""
    w = gdn_inputs.WORKLOADS["720p"]
    x = gdn_inputs.workload_inputs(w, device="cuda")
    c = gdn_inputs.cotangents(w.B, w.H, w.T, w.N, w.D, seed=904, state_std=1.0, device="cuda")
    got = api().gdn_frame_backward(x["q"], x["k"], x["v"], x["gamma"], x["beta"], c["d_out"],
                                   state_in=x["state"], d_state_out=c["d_state"],
                                   key_scale=w.key_scale)
    assert api().gdn_sync_status() == 0
    names = ["dq", "dk", "dv", "d_gamma", "d_beta", "d_state_in"]
    tols = [GRAD_TOL] * 3 + [SCALAR_TOL] * 2 + [STATE_TOL]

    def one(h):
        sl5 = lambda t: None if t is None else pu.f32(t[:, :, :, h:h + 1])
        sl3 = lambda t: pu.f32(t[:, :, h:h + 1])
        sl4 = lambda t: None if t is None else pu.f32(t[:, h:h + 1])
        ref = oracle.gdn_frame_backward(sl5(x["q"]), sl5(x["k"]), sl5(x["v"]), sl3(x["gamma"]),
                                        sl3(x["beta"]), sl4(x["state"]), sl5(c["d_out"]),
                                        sl4(c["d_state"]), w.key_scale)
        gots = [sl5(got[0]), sl5(got[1]), sl5(got[2]), sl3(got[3]), sl3(got[4]), sl4(got[5])]
        errs = []
        for g_, r in zip(gots, ref):
            assert np.all(np.isfinite(g_))
            e = pu.RelF()
            e.add(g_, r, h)
            errs.append(e)
        return errs

    total = [pu.RelF() for _ in names]
    for errs in pu.pool_map(one, range(w.H), bytes_per_task=9e9):
        for t, e in zip(total, errs):
            t.merge(e)
    pu.log("backward_720p_all_heads", **dict(zip(names, total)))
    for n, t, tol in zip(names, total, tols):
        assert t.value <= tol, f"{n}: rel err {t.value:.2e} > {tol:.0e} (worst head {t.worst_at})"


def test_backward_in_a_cuda_graph():
    """After one uncaptured call (which sizes the workspace and creates the internal stream), the
    backward can be captured in a CUDA graph: the fork to the internal stream and the join back
    are event nodes of the graph. Replays give the uncaptured call's result bit for bit."""
    B, H, T, N, D = 1, 2, 9, 100, 128
    x = gdn_inputs.clip_inputs(B, H, T, N, D, seed=905, state_std=0.3, device="cuda")
    c = gdn_inputs.cotangents(B, H, T, N, D, seed=906, state_std=1.0, device="cuda")
    a = api()
    old = os.environ.get("GDN_BWD_SEGMENT_FRAMES")
    os.environ["GDN_BWD_SEGMENT_FRAMES"] = "3"  # three segments: the second stream is used
    try:
        ref = a.gdn_frame_backward(x["q"], x["k"], x["v"], x["gamma"], x["beta"], c["d_out"],
                                   state_in=x["state"], d_state_out=c["d_state"])
        torch.cuda.synchronize()
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(s):
            with torch.cuda.graph(g, stream=s):
                got = a.gdn_frame_backward(x["q"], x["k"], x["v"], x["gamma"], x["beta"],
                                           c["d_out"], state_in=x["state"],
                                           d_state_out=c["d_state"], stream=s)
        for _ in range(2):
            g.replay()
        torch.cuda.synchronize()
        assert a.gdn_sync_status() == 0
    finally:
        if old is None:
            os.environ.pop("GDN_BWD_SEGMENT_FRAMES", None)
        else:
            os.environ["GDN_BWD_SEGMENT_FRAMES"] = old
    for r, o in zip(ref, got):
        assert torch.equal(r, o)


# --------------------------------------------------------------------------- training pair


@pytest.mark.parametrize("shape", SHAPES[:4], ids=lambda s: "B%dH%dT%dN%dD%d%s" % (s[:5] + ("s" if s[5] else "",)))
def test_training_pair_matches_oracle(shape):
    """gdn_frame_forward_train (the forward that keeps A_t, B_t, S_t) and
    gdn_frame_backward_saved (the backward that reads them instead of recomputing) against the
    oracle's forward and backward."""
    B, H, T, N, D, with_state = shape
    x = gdn_inputs.clip_inputs(B, H, T, N, D, gamma_range=(0.9, 0.999), beta_range=(0.05, 0.95),
                               seed=710 + T + D, state_std=0.3 if with_state else 0.0)
    c = gdn_inputs.cotangents(B, H, T, N, D, seed=810 + T + D, state_std=1.0 if with_state else 0.0)
    ks = 1.0 / math.sqrt(D * N)
    g = {k: (None if v is None else v.cuda()) for k, v in x.items()}
    gc = {k: (None if v is None else v.cuda()) for k, v in c.items()}
    a = api()
    out, st, saved = a.gdn_frame_forward_train(g["q"], g["k"], g["v"], g["gamma"], g["beta"],
                                               g["state"], key_scale=ks)
    got = a.gdn_frame_backward_saved(g["q"], g["k"], g["v"], g["gamma"], g["beta"], saved,
                                     gc["d_out"], state_in=g["state"],
                                     d_state_out=gc["d_state"], key_scale=ks)
    assert a.gdn_sync_status() == 0
    o_ref, s_ref = oracle.gdn_frame_forward(f64(x["q"]), f64(x["k"]), f64(x["v"]), f64(x["gamma"]),
                                            f64(x["beta"]), None if x["state"] is None else f64(x["state"]), ks)
    assert relf(f64(out), o_ref) <= 1e-2 and relf(f64(st), s_ref) <= 5e-3
    check_against_oracle(x, c, got, ks)


@pytest.mark.parametrize("shape", SEGMENTED, ids=lambda s: "B%dH%dT%dN%dD%d%s_seg%d" % (s[:5] + ("s" if s[5] else "", s[6])))
def test_training_pair_segmented_matches_oracle(shape):
    """The backward with saved states in segments of frames: each segment's dQ/E pass runs
    before its part of the reverse chain (from the clip's end), the per-frame and dk/dv passes
    of every segment after it; against the oracle."""
    B, H, T, N, D, with_state, seg = shape
    old = os.environ.get("GDN_BWD_SEGMENT_FRAMES")
    os.environ["GDN_BWD_SEGMENT_FRAMES"] = str(seg)
    try:
        x = gdn_inputs.clip_inputs(B, H, T, N, D, seed=760 + T + seg,
                                   state_std=0.3 if with_state else 0.0)
        c = gdn_inputs.cotangents(B, H, T, N, D, seed=860 + T + seg,
                                  state_std=1.0 if with_state else 0.0)
        ks = 1.0 / math.sqrt(D * N)
        g = {k: (None if v is None else v.cuda()) for k, v in x.items()}
        gc = {k: (None if v is None else v.cuda()) for k, v in c.items()}
        a = api()
        _, _, saved = a.gdn_frame_forward_train(g["q"], g["k"], g["v"], g["gamma"], g["beta"],
                                                g["state"], key_scale=ks)
        got = a.gdn_frame_backward_saved(g["q"], g["k"], g["v"], g["gamma"], g["beta"], saved,
                                         gc["d_out"], state_in=g["state"],
                                         d_state_out=gc["d_state"], key_scale=ks)
        assert a.gdn_sync_status() == 0
    finally:
        if old is None:
            os.environ.pop("GDN_BWD_SEGMENT_FRAMES", None)
        else:
            os.environ["GDN_BWD_SEGMENT_FRAMES"] = old
    check_against_oracle(x, c, got, ks)


def test_training_pair_equals_recomputing_backward_on_720p():
    """On the 720p clip the saved states are those the recomputing backward builds (the same
    statistics and chain kernels), and the saved path's dQ/E pass issues the same products in the
    same order as the separate dq and E passes, so both backwards agree bit for bit; the forward
    that saves them equals the three-kernel forward bit for bit."""
    from frame_wise_gated_deltanet_b200 import _lib
    w = gdn_inputs.WORKLOADS["720p"]
    x = gdn_inputs.workload_inputs(w, device="cuda")
    c = gdn_inputs.cotangents(w.B, w.H, w.T, w.N, w.D, seed=904, state_std=1.0, device="cuda")
    a = api()
    out, st, saved = a.gdn_frame_forward_train(x["q"], x["k"], x["v"], x["gamma"], x["beta"])
    got = a.gdn_frame_backward_saved(x["q"], x["k"], x["v"], x["gamma"], x["beta"], saved,
                                     c["d_out"], d_state_out=c["d_state"])
    assert a.gdn_sync_status() == 0
    del saved
    ref = a.gdn_frame_backward(x["q"], x["k"], x["v"], x["gamma"], x["beta"], c["d_out"],
                               d_state_out=c["d_state"])
    try:
        assert _lib.LIB.gdn_set_forward_mode(1) == 0
        o3, s3 = a.gdn_frame_forward(x["q"], x["k"], x["v"], x["gamma"], x["beta"])
    finally:
        _lib.LIB.gdn_set_forward_mode(0)
    assert a.gdn_sync_status() == 0
    assert torch.equal(out, o3) and torch.equal(st, s3)
    for r, o in zip(ref, got):
        assert torch.equal(r, o)
