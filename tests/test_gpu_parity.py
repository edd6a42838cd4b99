"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle, element by element,
on the same seeded inputs.

Tolerances: relative Frobenius error of the output <= 1e-2 and of the final state <= 5e-3
(the bars the layer's definition sets for bf16 Q/K/V/O with an fp32 state); the per-frame
statistics A (stored bf16) <= 5e-3 and B (stored f32) <= 1e-5.
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

O_TOL = 1e-2
S_TOL = 5e-3


def api():
    from frame_wise_gated_deltanet_b200 import api as a
    return a


def f64(t):
    return t.detach().to(torch.float32).cpu().numpy().astype(np.float64)


def relf(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def to_cuda(d):
    return {k: (None if v is None else v.cuda()) for k, v in d.items()}


SHAPES = [
    # (B, H, T, N, D, with_state)
    (1, 2, 8, 16, 32, False),     # the tiny workload's shape
    (1, 3, 5, 200, 64, True),
    (2, 2, 4, 300, 128, False),
    (1, 1, 3, 1, 128, True),      # one token per frame
    (1, 2, 2, 128, 128, False),   # exactly one tile
    (1, 2, 3, 129, 112, True),    # ragged tail of one token
    (1, 1, 1, 880, 128, False),   # one frame
    (2, 1, 6, 77, 48, True),
    (1, 2, 20, 33, 128, True),    # many frames
    (3, 5, 2, 64, 8, False),      # smallest head dim
]


@pytest.fixture
def forward_mode(request):
    """Run a test with gdn_set_forward_mode(mode) (1 = three kernels, 2 = fused persistent,
    3 = chunked with chunks of 3 frames)."""
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


@pytest.mark.parametrize("forward_mode", [1, 2, 3], indirect=True, ids=["split", "fused", "chunked"])
@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "B%dH%dT%dN%dD%d%s" % (s[:5] + ("s" if s[5] else "",)))
def test_forward_matches_oracle(shape, forward_mode):
    B, H, T, N, D, with_state = shape
    x = gdn_inputs.clip_inputs(B, H, T, N, D, seed=100 + D + N, state_std=0.3 if with_state else 0.0)
    ks = 1.0 / math.sqrt(D * N)
    g = to_cuda(x)
    out, st = api().gdn_frame_forward(g["q"], g["k"], g["v"], g["gamma"], g["beta"], g["state"],
                                      key_scale=ks)
    assert api().gdn_sync_status() == 0
    o_ref, s_ref = oracle.gdn_frame_forward(f64(x["q"]), f64(x["k"]), f64(x["v"]), f64(x["gamma"]),
                                            f64(x["beta"]),
                                            None if x["state"] is None else f64(x["state"]), ks)
    eo, es = relf(f64(out), o_ref), relf(f64(st), s_ref)
    assert eo <= O_TOL and es <= S_TOL, f"O err {eo:.2e}, S err {es:.2e}"


@pytest.mark.parametrize("shape", [(1, 2, 3, 200, 128), (2, 3, 2, 77, 64), (1, 1, 2, 16, 32),
                                   (1, 2, 2, 390, 112), (1, 1, 1, 1, 128)])
def test_frame_stats_match_oracle(shape):
    B, H, T, N, D = shape
    x = gdn_inputs.clip_inputs(B, H, T, N, D, seed=7 + N)
    ks = 1.0 / math.sqrt(D * N)
    A, Bm = api().gdn_frame_stats(x["k"].cuda(), x["v"].cuda(), key_scale=ks)
    A, Bm = f64(A), f64(Bm)
    k, v = f64(x["k"]), f64(x["v"])
    for b in range(B):
        for h in range(H):
            for t in range(T):
                Ar, Br = oracle.frame_statistics(k[b, t, :, h], v[b, t, :, h], ks)
                assert relf(A[b, h, t], Ar) <= 5e-3
                assert relf(Bm[b, h, t], Br) <= 1e-5


def test_tiny_workload():
    w = gdn_inputs.WORKLOADS["tiny"]
    x = gdn_inputs.workload_inputs(w)
    g = to_cuda(x)
    out, st = api().gdn_frame_forward(g["q"], g["k"], g["v"], g["gamma"], g["beta"], None,
                                      key_scale=w.key_scale)
    o_ref, s_ref = oracle.gdn_frame_forward(f64(x["q"]), f64(x["k"]), f64(x["v"]), f64(x["gamma"]),
                                            f64(x["beta"]), None, w.key_scale)
    assert relf(f64(out), o_ref) <= O_TOL
    assert relf(f64(st), s_ref) <= S_TOL


def test_480p_workload_full():
    """The 480p clip in the benchmark's launch configuration, every head against the oracle."""
    w = gdn_inputs.WORKLOADS["480p"]
    x = gdn_inputs.workload_inputs(w)
    g = to_cuda(x)
    out, st = api().gdn_frame_forward(g["q"], g["k"], g["v"], g["gamma"], g["beta"], None,
                                      key_scale=w.key_scale)
    assert api().gdn_sync_status() == 0
    o_ref, s_ref = oracle.gdn_frame_forward(f64(x["q"]), f64(x["k"]), f64(x["v"]), f64(x["gamma"]),
                                            f64(x["beta"]), None, w.key_scale)
    eo, es = relf(f64(out), o_ref), relf(f64(st), s_ref)
    pu.log("480p_full", out={"relF": eo}, state={"relF": es})
    assert eo <= O_TOL
    assert es <= S_TOL


def _head_slice(t, b, h):
    """[B,T,N,H,D] -> [1,T,N,1,D] float64 numpy for one (b, h), copied from the device."""
    return f64(t[b:b + 1, :, :, h:h + 1, :].contiguous())


def test_720p_workload_all_heads():
    """The full 60 s 720p clip in the benchmark's launch configuration. The oracle recomputes
    every head over all 961 frames; the errors are those of the whole output tensor and of the
    whole final state."""
    w = gdn_inputs.WORKLOADS["720p"]
    g = gdn_inputs.workload_inputs(w, device="cuda")
    out, st = api().gdn_frame_forward(g["q"], g["k"], g["v"], g["gamma"], g["beta"], None,
                                      key_scale=w.key_scale)
    assert api().gdn_sync_status() == 0

    def one(h):
        sl = lambda t: pu.f32(t[:, :, :, h:h + 1])
        o_ref, s_ref = oracle.gdn_frame_forward(
            sl(g["q"]), sl(g["k"]), sl(g["v"]), pu.f32(g["gamma"][:, :, h:h + 1]),
            pu.f32(g["beta"][:, :, h:h + 1]), None, w.key_scale)
        eo, es = pu.RelF(), pu.RelF()
        eo.add(sl(out), o_ref, h)
        es.add(pu.f32(st[:, h:h + 1]), s_ref, h)
        return eo, es

    eo, es = pu.RelF(), pu.RelF()
    for a, b in pu.pool_map(one, range(w.H), bytes_per_task=5e9):
        eo.merge(a)
        es.merge(b)
    pu.log("720p_all_heads", out=eo, state=es)
    assert eo.value <= O_TOL and es.value <= S_TOL, (
        f"O err {eo.value:.2e} (worst head {eo.worst_at}: {eo.worst:.2e}), "
        f"S err {es.value:.2e} (worst head {es.worst_at}: {es.worst:.2e})")


def test_stream_workload_all_streams():
    """64 chained single-frame steps of all 16 streams x 20 heads, state updated in place; the
    oracle follows every (stream, head) through all steps. The output error is over all 64
    steps' outputs concatenated, the state error over the state after the 64th step."""
    w = gdn_inputs.WORKLOADS["stream"]
    state = gdn_inputs.workload_inputs(w, device="cuda")["state"].contiguous()
    ref_state = pu.f32(state).astype(np.float64)
    eo = pu.RelF()
    for j in range(w.steps):
        x = gdn_inputs.workload_inputs(w, device="cuda", step=j)
        q, k, v = (x[n][:, 0].contiguous() for n in ("q", "k", "v"))
        gam, bet = x["gamma"][:, 0].contiguous(), x["beta"][:, 0].contiguous()
        out, _ = api().gdn_frame_step(q, k, v, gam, bet, state, state_out=state,
                                      key_scale=w.key_scale)
        qh, kh, vh, oh = pu.f32(q), pu.f32(k), pu.f32(v), pu.f32(out)
        gh, bh = pu.f32(gam), pu.f32(bet)

        def one(i):
            b, h = divmod(i, w.H)
            o_ref, s_ref = oracle.gdn_frame_step(
                qh[b:b + 1, :, h:h + 1], kh[b:b + 1, :, h:h + 1], vh[b:b + 1, :, h:h + 1],
                gh[b:b + 1, h:h + 1], bh[b:b + 1, h:h + 1], ref_state[b:b + 1, h:h + 1],
                w.key_scale)
            ref_state[b, h] = s_ref[0, 0]  # each task owns its own (b, h) slice
            e = pu.RelF()
            e.add(oh[b:b + 1, :, h:h + 1], o_ref, (j, b, h))
            return e

        for e in pu.pool_map(one, range(w.B * w.H), bytes_per_task=5e7):
            eo.merge(e)
    assert api().gdn_sync_status() == 0
    es = pu.RelF()
    es.add(pu.f32(state), ref_state, "all")
    pu.log("stream_all_streams", out=eo, state=es)
    assert eo.value <= O_TOL and es.value <= S_TOL, (
        f"O err {eo.value:.2e} (worst {eo.worst_at}: {eo.worst:.2e}), S err {es.value:.2e}")


@pytest.mark.parametrize("forward_mode", [1, 2, 3], indirect=True, ids=["split", "fused", "chunked"])
def test_480p_workload_all_paths(forward_mode):
    w = gdn_inputs.WORKLOADS["480p"]
    x = gdn_inputs.workload_inputs(w)
    g = to_cuda(x)
    out, st = api().gdn_frame_forward(g["q"], g["k"], g["v"], g["gamma"], g["beta"], None,
                                      key_scale=w.key_scale)
    assert api().gdn_sync_status() == 0
    o_ref, s_ref = oracle.gdn_frame_forward(f64(x["q"]), f64(x["k"]), f64(x["v"]), f64(x["gamma"]),
                                            f64(x["beta"]), None, w.key_scale)
    assert relf(f64(out), o_ref) <= O_TOL
    assert relf(f64(st), s_ref) <= S_TOL


@pytest.mark.parametrize("forward_mode", [1, 2, 3], indirect=True, ids=["split", "fused", "chunked"])
def test_forward_in_a_cuda_graph(forward_mode):
    """After one uncaptured call (which sizes the workspace), the forward can be captured in a
    CUDA graph on every path (the fused path's cooperative launch and its flag memset become
    graph nodes) and its replays give the uncaptured call's result bit for bit."""
    B, H, T, N, D = 1, 3, 11, 150, 128
    x = gdn_inputs.clip_inputs(B, H, T, N, D, seed=1910, state_std=0.3, device="cuda")
    a = api()
    ref_o, ref_s = a.gdn_frame_forward(x["q"], x["k"], x["v"], x["gamma"], x["beta"], x["state"])
    torch.cuda.synchronize()
    out = torch.empty_like(ref_o)
    st = torch.empty_like(ref_s)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            a.gdn_frame_forward(x["q"], x["k"], x["v"], x["gamma"], x["beta"], x["state"], out,
                                st, stream=s)
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    assert a.gdn_sync_status() == 0
    assert torch.equal(out, ref_o) and torch.equal(st, ref_s)


def test_fused_and_split_paths_agree_on_720p():
    """Both forward paths on the full 720p clip: same kernels' arithmetic, so they agree to the
    rounding of the bf16 copies of S (identical in practice)."""
    from frame_wise_gated_deltanet_b200 import _lib
    w = gdn_inputs.WORKLOADS["720p"]
    g = gdn_inputs.workload_inputs(w, device="cuda")
    res = {}
    try:
        for mode in (1, 2):
            assert _lib.LIB.gdn_set_forward_mode(mode) == 0
            res[mode] = api().gdn_frame_forward(g["q"], g["k"], g["v"], g["gamma"], g["beta"],
                                                None, key_scale=w.key_scale)
            assert api().gdn_sync_status() == 0
    finally:
        _lib.LIB.gdn_set_forward_mode(0)
    assert torch.equal(res[1][1], res[2][1])
    assert torch.equal(res[1][0], res[2][0])


# --------------------------------------------------------------------------- chunked forward


def _launched(fn):
    """Names of the library's kernel launches made by fn()."""
    from frame_wise_gated_deltanet_b200 import _lib
    import ctypes
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(64)]
    for e in evs:
        e.record()  # creates the event
    handles = (ctypes.c_void_p * len(evs))(*[e.cuda_event for e in evs])
    _lib.LIB.gdn_profile_arm(handles, len(evs))
    try:
        fn()
        torch.cuda.synchronize()
        return [_lib.LIB.gdn_profile_kernel(i).decode()
                for i in range(_lib.LIB.gdn_profile_count())]
    finally:
        _lib.LIB.gdn_profile_arm(None, 0)


@pytest.mark.parametrize("case", [
    # (B, H, T, N, D, L, with_state)
    (1, 2, 37, 100, 128, 8, True),    # ragged last chunk (5 frames)
    (1, 2, 37, 100, 128, 1, True),    # one frame per chunk: 36 scan steps
    (1, 2, 37, 100, 128, 36, False),  # two chunks, the second of one frame
    (1, 2, 37, 100, 128, 37, True),   # one chunk: the plain chain
    (2, 3, 29, 64, 64, 4, True),
    (1, 1, 50, 17, 8, 7, False),
    (1, 2, 24, 130, 112, 5, True),
    (1, 1, 33, 40, 48, 2, True),
])
def test_chunked_forward_matches_oracle(case):
    """Chunked forward (per-chunk composition of the frame maps, inter-chunk scan, per-chunk
    replay) for several chunk lengths, against the oracle."""
    from frame_wise_gated_deltanet_b200 import _lib
    B, H, T, N, D, L, with_state = case
    x = gdn_inputs.clip_inputs(B, H, T, N, D, seed=700 + L + D, state_std=0.5 if with_state else 0.0)
    ks = 1.0 / math.sqrt(D * N)
    g = to_cuda(x)
    old = os.environ.get("GDN_CHUNK_LEN")
    os.environ["GDN_CHUNK_LEN"] = str(L)
    try:
        assert _lib.LIB.gdn_set_forward_mode(3) == 0
        res = {}
        names = _launched(lambda: res.update(r=api().gdn_frame_forward(
            g["q"], g["k"], g["v"], g["gamma"], g["beta"], g["state"], key_scale=ks)))
        out, st = res["r"]
        assert api().gdn_sync_status() == 0
    finally:
        _lib.LIB.gdn_set_forward_mode(0)
        if old is None:
            os.environ.pop("GDN_CHUNK_LEN", None)
        else:
            os.environ["GDN_CHUNK_LEN"] = old
    if L < T:
        assert "gdn_scan_kernel" in names and "gdn_chain_kernel_compose" in names, names
    o_ref, s_ref = oracle.gdn_frame_forward(f64(x["q"]), f64(x["k"]), f64(x["v"]), f64(x["gamma"]),
                                            f64(x["beta"]),
                                            None if x["state"] is None else f64(x["state"]), ks)
    eo, es = relf(f64(out), o_ref), relf(f64(st), s_ref)
    assert eo <= O_TOL and es <= S_TOL, f"O err {eo:.2e}, S err {es:.2e}"


def test_few_heads_long_clip_uses_chunked_path():
    """Two heads over the 961 frames of the 720p clip (the per-GPU slice of the 720p layer under
    10-way head sharding): the chain, not HBM, bounds the other paths, so the automatic choice
    is the chunked forward; the oracle recomputes both heads over all frames."""
    w = gdn_inputs.WORKLOADS["720p_2h"]
    x = gdn_inputs.workload_inputs(w, device="cuda")
    H = w.H
    res = {}
    names = _launched(lambda: res.update(r=api().gdn_frame_forward(
        x["q"], x["k"], x["v"], x["gamma"], x["beta"], None, key_scale=w.key_scale)))
    out, st = res["r"]
    assert api().gdn_sync_status() == 0
    assert "gdn_scan_kernel" in names, names
    for h in range(H):
        o_ref, s_ref = oracle.gdn_frame_forward(
            _head_slice(x["q"], 0, h), _head_slice(x["k"], 0, h), _head_slice(x["v"], 0, h),
            f64(x["gamma"][:, :, h:h + 1]), f64(x["beta"][:, :, h:h + 1]), None, w.key_scale)
        eo = relf(_head_slice(out, 0, h), o_ref)
        es = relf(f64(st[0, h]), s_ref[0, 0])
        assert eo <= O_TOL and es <= S_TOL, f"head {h}: O err {eo:.2e}, S err {es:.2e}"


@pytest.mark.parametrize("forward_mode", [1, 2, 3], indirect=True, ids=["split", "fused", "chunked"])
def test_forward_state_in_place(forward_mode):
    """state_out may be state_in: every path reads the start state before any CTA writes the
    final one (the chunked replay reads the scan's copy)."""
    B, H, T, N, D = 1, 2, 17, 64, 128
    x = gdn_inputs.clip_inputs(B, H, T, N, D, seed=41, state_std=0.4)
    ks = 1.0 / math.sqrt(D * N)
    g = to_cuda(x)
    st = g["state"].clone()
    out, st2 = api().gdn_frame_forward(g["q"], g["k"], g["v"], g["gamma"], g["beta"], st,
                                       state_out=st, key_scale=ks)
    assert api().gdn_sync_status() == 0 and st2 is st
    o_ref, s_ref = oracle.gdn_frame_forward(f64(x["q"]), f64(x["k"]), f64(x["v"]), f64(x["gamma"]),
                                            f64(x["beta"]), f64(x["state"]), ks)
    eo, es = relf(f64(out), o_ref), relf(f64(st), s_ref)
    assert eo <= O_TOL and es <= S_TOL, f"O err {eo:.2e}, S err {es:.2e}"


@pytest.mark.parametrize("case", [
    # (B, H, T, N, D, segment frames, with_state)
    (2, 3, 13, 50, 64, 4, True),     # ragged last segment, two batches
    (1, 2, 30, 100, 128, 7, True),
    (1, 2, 9, 33, 128, 0, False),    # automatic segment size: one segment
    (3, 1, 5, 20, 32, 1, True),      # one frame per segment
])
def test_forward_host_matches_oracle(case):
    """gdn_frame_forward_host: pinned host tensors streamed through the GPU in segments."""
    B, H, T, N, D, seg, with_state = case
    x = gdn_inputs.clip_inputs(B, H, T, N, D, seed=900 + T, state_std=0.3 if with_state else 0.0)
    ks = 1.0 / math.sqrt(D * N)
    pin = {k: (None if t is None else t.pin_memory()) for k, t in x.items()}
    old = os.environ.get("GDN_HOST_SEGMENT_FRAMES")
    os.environ["GDN_HOST_SEGMENT_FRAMES"] = str(seg)
    try:
        out, st = api().gdn_frame_forward_host(pin["q"], pin["k"], pin["v"], pin["gamma"],
                                               pin["beta"], pin["state"], key_scale=ks)
        assert api().gdn_sync_status() == 0
    finally:
        if old is None:
            os.environ.pop("GDN_HOST_SEGMENT_FRAMES", None)
        else:
            os.environ["GDN_HOST_SEGMENT_FRAMES"] = old
    assert not out.is_cuda and not st.is_cuda
    o_ref, s_ref = oracle.gdn_frame_forward(f64(x["q"]), f64(x["k"]), f64(x["v"]), f64(x["gamma"]),
                                            f64(x["beta"]),
                                            None if x["state"] is None else f64(x["state"]), ks)
    eo, es = relf(f64(out), o_ref), relf(f64(st), s_ref)
    assert eo <= O_TOL and es <= S_TOL, f"O err {eo:.2e}, S err {es:.2e}"
    # the device entry point on the same inputs: the same recurrence split at segment bounds,
    # possibly through another path (the whole clip and a segment may pick different kernels),
    # so they agree to rounding, not bit for bit
    g = to_cuda(x)
    od, sd = api().gdn_frame_forward(g["q"], g["k"], g["v"], g["gamma"], g["beta"], g["state"],
                                     key_scale=ks)
    torch.cuda.synchronize()
    assert relf(f64(out), f64(od)) <= 3e-3 and relf(f64(st), f64(sd)) <= 3e-4


# --------------------------------------------------------------------------- fp8 inputs


def _fp8_clip(B, H, T, N, D, seed, with_state):
    x = gdn_inputs.clip_inputs(B, H, T, N, D, seed=seed, state_std=0.3 if with_state else 0.0)
    q8, sq = gdn_inputs.quantize_e4m3(x["q"])
    k8, sk = gdn_inputs.quantize_e4m3(x["k"])
    v8, sv = gdn_inputs.quantize_e4m3(x["v"])
    return dict(q8=q8, k8=k8, v8=v8, sq=sq, sk=sk, sv=sv, gamma=x["gamma"], beta=x["beta"],
                state=x["state"])


def _fp8_oracle(c, ks):
    return oracle.gdn_frame_forward_fp8(c["q8"].cpu().numpy(), c["k8"].cpu().numpy(),
                                        c["v8"].cpu().numpy(), f64(c["sq"]), f64(c["sk"]),
                                        f64(c["sv"]), f64(c["gamma"]), f64(c["beta"]),
                                        None if c["state"] is None else f64(c["state"]), ks)


FP8_SHAPES = [
    # (B, H, T, N, D, with_state)
    (1, 2, 5, 200, 128, True),
    (2, 3, 4, 129, 112, False),   # ragged tail, padded head dim
    (1, 1, 3, 64, 80, True),
    (1, 2, 20, 33, 96, True),
    (1, 1, 1, 880, 128, False),   # one frame
]


@pytest.mark.parametrize("forward_mode", [1, 2, 3], indirect=True, ids=["split", "fused", "chunked"])
@pytest.mark.parametrize("shape", FP8_SHAPES, ids=lambda s: "B%dH%dT%dN%dD%d%s" % (s[:5] + ("s" if s[5] else "",)))
def test_fp8_forward_matches_oracle(shape, forward_mode):
    """E4M3 q, k, v with per-(frame, head) scales against the oracle on the decoded values."""
    B, H, T, N, D, with_state = shape
    c = _fp8_clip(B, H, T, N, D, seed=600 + N + D, with_state=with_state)
    ks = 1.0 / math.sqrt(D * N)
    g = to_cuda(c)
    out, st = api().gdn_frame_forward_fp8(g["q8"], g["k8"], g["v8"], g["sq"], g["sk"], g["sv"],
                                          g["gamma"], g["beta"], g["state"], key_scale=ks)
    assert api().gdn_sync_status() == 0
    o_ref, s_ref = _fp8_oracle(c, ks)
    eo, es = relf(f64(out), o_ref), relf(f64(st), s_ref)
    assert eo <= O_TOL and es <= S_TOL, f"O err {eo:.2e}, S err {es:.2e}"


def test_fp8_720p_all_heads():
    """The 720p clip quantised to E4M3 (per frame and head), in the launch configuration of the
    benchmark's fp8 line; the oracle recomputes every head over all 961 frames."""
    w = gdn_inputs.WORKLOADS["720p"]
    x = gdn_inputs.workload_inputs(w, device="cuda")
    c = {}
    for n in ("q", "k", "v"):
        c[n + "8"], c["s" + n] = gdn_inputs.quantize_e4m3(x[n])
    del x["q"], x["k"], x["v"]
    out, st = api().gdn_frame_forward_fp8(c["q8"], c["k8"], c["v8"], c["sq"], c["sk"], c["sv"],
                                          x["gamma"], x["beta"], None, key_scale=w.key_scale)
    assert api().gdn_sync_status() == 0

    def one(h):
        sl = lambda t: t[:, :, :, h:h + 1].contiguous().cpu().numpy()
        sc = lambda t: pu.f32(t[:, :, h:h + 1])
        o_ref, s_ref = oracle.gdn_frame_forward_fp8(
            sl(c["q8"]), sl(c["k8"]), sl(c["v8"]), sc(c["sq"]), sc(c["sk"]), sc(c["sv"]),
            sc(x["gamma"]), sc(x["beta"]), None, w.key_scale)
        eo, es = pu.RelF(), pu.RelF()
        eo.add(pu.f32(out[:, :, :, h:h + 1]), o_ref, h)
        es.add(pu.f32(st[:, h:h + 1]), s_ref, h)
        return eo, es

    eo, es = pu.RelF(), pu.RelF()
    for a, b in pu.pool_map(one, range(w.H), bytes_per_task=7e9):
        eo.merge(a)
        es.merge(b)
    pu.log("fp8_720p_all_heads", out=eo, state=es)
    assert eo.value <= O_TOL and es.value <= S_TOL, (
        f"O err {eo.value:.2e} (worst head {eo.worst_at}: {eo.worst:.2e}), S err {es.value:.2e}")


STEP_SHAPES = [
    # (B, H, N, D, with_state)
    (2, 3, 100, 128, True),
    (1, 2, 257, 112, True),     # padded head dim, ragged tokens
    (3, 1, 880, 128, False),    # S_0 = 0
    (2, 2, 16, 72, True),
]


@pytest.mark.parametrize("forward_mode", [1, 0], indirect=True, ids=["split", "fused"])
@pytest.mark.parametrize("shape", STEP_SHAPES, ids=lambda s: "B%dH%dN%dD%d%s" % (s[:4] + ("s" if s[4] else "",)))
def test_step_matches_oracle(shape, forward_mode):
    """gdn_frame_step (fused one-pass kernel for D > 64, or the three kernels), state in place."""
    B, H, N, D, with_state = shape
    x = gdn_inputs.clip_inputs(B, H, 1, N, D, seed=500 + N + D, state_std=0.2 if with_state else 0.0)
    ks = 1.0 / math.sqrt(D * N)
    q, k, v = (x[n][:, 0].contiguous().cuda() for n in ("q", "k", "v"))
    gam, bet = x["gamma"][:, 0].contiguous().cuda(), x["beta"][:, 0].contiguous().cuda()
    state = x["state"].cuda() if with_state else torch.zeros((B, H, D, D), device="cuda")
    out, st = api().gdn_frame_step(q, k, v, gam, bet, state if with_state else None,
                                   state_out=state, key_scale=ks)
    assert api().gdn_sync_status() == 0
    o_ref, s_ref = oracle.gdn_frame_step(f64(x["q"][:, 0]), f64(x["k"][:, 0]), f64(x["v"][:, 0]),
                                         f64(x["gamma"][:, 0]), f64(x["beta"][:, 0]),
                                         f64(x["state"]) if with_state else None, ks)
    assert relf(f64(out), o_ref) <= O_TOL
    assert relf(f64(st), s_ref) <= S_TOL


def test_step_paths_agree_on_stream_workload():
    """The fused step and the three-kernel step on the full streaming workload (B16 H20 N880)."""
    from frame_wise_gated_deltanet_b200 import _lib
    w = gdn_inputs.WORKLOADS["stream"]
    x = gdn_inputs.workload_inputs(w, device="cuda", step=0)
    q, k, v = (x[n][:, 0].contiguous() for n in ("q", "k", "v"))
    gam, bet = x["gamma"][:, 0].contiguous(), x["beta"][:, 0].contiguous()
    s0 = gdn_inputs.workload_inputs(w, device="cuda")["state"]
    res = {}
    try:
        for mode in (1, 0):
            assert _lib.LIB.gdn_set_forward_mode(mode) == 0
            res[mode] = api().gdn_frame_step(q, k, v, gam, bet, s0, key_scale=w.key_scale)
            assert api().gdn_sync_status() == 0
    finally:
        _lib.LIB.gdn_set_forward_mode(0)
    assert relf(f64(res[0][0]), f64(res[1][0])) <= 2e-3
    assert relf(f64(res[0][1]), f64(res[1][1])) <= 1e-5


def test_split_resume_on_gpu():
    """forward(T) equals forward(T1) then forward(T - T1) through the carried state."""
    B, H, T, N, D = 1, 2, 9, 150, 128
    x = to_cuda(gdn_inputs.clip_inputs(B, H, T, N, D, seed=5))
    ks = 1.0 / math.sqrt(D * N)
    out, st = api().gdn_frame_forward(x["q"], x["k"], x["v"], x["gamma"], x["beta"], key_scale=ks)
    T1 = 4
    sl = lambda t, a, b: t[:, a:b].contiguous()
    o1, s1 = api().gdn_frame_forward(sl(x["q"], 0, T1), sl(x["k"], 0, T1), sl(x["v"], 0, T1),
                                     sl(x["gamma"], 0, T1), sl(x["beta"], 0, T1), key_scale=ks)
    o2, s2 = api().gdn_frame_forward(sl(x["q"], T1, T), sl(x["k"], T1, T), sl(x["v"], T1, T),
                                     sl(x["gamma"], T1, T), sl(x["beta"], T1, T), s1, key_scale=ks)
    torch.cuda.synchronize()
    # the bf16 copy of S used by the output GEMM is rounded from the same fp32 state, so the
    # two paths agree to fp32 rounding of the state
    assert relf(f64(torch.cat([o1, o2], 1)), f64(out)) <= 1e-3
    assert relf(f64(s2), f64(st)) <= 1e-5


def test_deterministic():
    B, H, T, N, D = 1, 4, 6, 333, 128
    x = to_cuda(gdn_inputs.clip_inputs(B, H, T, N, D, seed=9))
    a = api().gdn_frame_forward(x["q"], x["k"], x["v"], x["gamma"], x["beta"])
    b = api().gdn_frame_forward(x["q"], x["k"], x["v"], x["gamma"], x["beta"])
    torch.cuda.synchronize()
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_invalid_sizes_rejected_on_gpu():
    from frame_wise_gated_deltanet_b200 import _lib
    q = torch.zeros((1, 2, 16, 2, 32), dtype=torch.bfloat16, device="cuda")
    g = torch.zeros((1, 2, 2), dtype=torch.float32, device="cuda")
    o = torch.empty_like(q)
    f = _lib.LIB.gdn_frame_forward
    assert f(q.data_ptr(), q.data_ptr(), q.data_ptr(), g.data_ptr(), g.data_ptr(), None,
             o.data_ptr(), None, 1, 2, 0, 16, 32, 0.1, None) == 1  # T = 0 (empty clip)
    assert f(q.data_ptr(), q.data_ptr(), q.data_ptr(), g.data_ptr(), g.data_ptr(), None,
             o.data_ptr(), None, 1, 2, 2, 0, 32, 0.1, None) == 1  # N = 0 (empty frames)


# --------------------------------------------------------------------------- block-causal LA

LA_SHAPES = [
    # (B, H, T, N, D, F, with_state)
    (1, 2, 7, 50, 112, 3, True),    # partial last block, carried (S, z)
    (1, 1, 4, 16, 32, 2, False),
    (1, 2, 5, 129, 64, 1, False),   # frame-causal special case
    (2, 1, 6, 200, 120, 6, True),   # one block = whole clip
    (1, 1, 3, 1, 8, 2, False),
]


def _la_inputs(B, H, T, N, D, with_state, seed):
    x = gdn_inputs.clip_inputs(B, H, T, N, D, seed=seed)
    s = z = None
    if with_state:
        gen = torch.Generator().manual_seed(seed + 1)
        s = torch.randn((B, H, D, D), generator=gen) * 5.0
        z = torch.rand((B, H, D), generator=gen) * 50.0 + 1.0
    return x["q"], x["k"], x["v"], s, z


@pytest.mark.parametrize("shape", LA_SHAPES, ids=lambda s: "B%dH%dT%dN%dD%dF%d%s" % (s[:6] + ("s" if s[6] else "",)))
def test_la_matches_oracle(shape):
    B, H, T, N, D, F, with_state = shape
    q, k, v, s, z = _la_inputs(B, H, T, N, D, with_state, seed=300 + N)
    cu = lambda t: None if t is None else t.cuda()
    out, so, zo = api().gdn_block_causal_la(cu(q), cu(k), cu(v), F, cu(s), cu(z))
    assert api().gdn_sync_status() == 0
    o_ref, s_ref, z_ref = oracle.la_block_causal(f64(q), f64(k), f64(v),
                                                 None if s is None else f64(s),
                                                 None if z is None else f64(z), F)
    assert relf(f64(out), o_ref) <= O_TOL
    assert relf(f64(so), s_ref) <= S_TOL
    assert relf(f64(zo), z_ref) <= S_TOL


def test_la_workload_all_heads():
    """The block-causal LA workload (B2 H20 D112 T81 N390, blocks of 3 frames): the oracle
    recomputes every (batch, head); errors over the whole output, state and normaliser."""
    w = gdn_inputs.WORKLOADS["la"]
    g = gdn_inputs.workload_inputs(w, device="cuda")
    out, so, zo = api().gdn_block_causal_la(g["q"], g["k"], g["v"], w.frames_per_block)
    assert api().gdn_sync_status() == 0

    def one(i):
        b, h = divmod(i, w.H)
        sl = lambda t: pu.f32(t[b:b + 1, :, :, h:h + 1])
        o_ref, s_ref, z_ref = oracle.la_block_causal(sl(g["q"]), sl(g["k"]), sl(g["v"]), None,
                                                     None, w.frames_per_block)
        e = [pu.RelF(), pu.RelF(), pu.RelF()]
        e[0].add(sl(out), o_ref, (b, h))
        e[1].add(pu.f32(so[b:b + 1, h:h + 1]), s_ref, (b, h))
        e[2].add(pu.f32(zo[b:b + 1, h:h + 1]), z_ref, (b, h))
        return e

    eo, es, ez = pu.RelF(), pu.RelF(), pu.RelF()
    for a in pu.pool_map(one, range(w.B * w.H), bytes_per_task=5e8):
        eo.merge(a[0])
        es.merge(a[1])
        ez.merge(a[2])
    pu.log("la_all_heads", out=eo, state=es, z=ez)
    assert eo.value <= O_TOL and es.value <= S_TOL and ez.value <= S_TOL, (
        f"O {eo.value:.2e}, S {es.value:.2e}, z {ez.value:.2e}")
