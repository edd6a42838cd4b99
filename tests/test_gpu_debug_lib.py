"""The debug library (libgdn_debug.so: the same sources with device-side checks of every copy's
shared-memory range, alignment, size and TMA coordinates, and of every MMA operand address) on
small ragged problems of every entry point: the results match the fp64 oracle at the usual bars
and no check fired. This is the stand-in for a memory checker, which cannot run on this hardware
pool.
"""
import math
import os

import numpy as np
import pytest
import torch

import gdn_inputs
import oracle

pytestmark = pytest.mark.gpu

O_TOL = 1e-2
S_TOL = 5e-3


def f64(t):
    return t.detach().to(torch.float32).cpu().numpy().astype(np.float64)


def relf(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


@pytest.fixture(scope="module")
def dbg():
    """The binding pointed at the debug library for this module's tests."""
    from frame_wise_gated_deltanet_b200 import _lib, api, build
    build.build(debug=True)
    lib = _lib.load(_lib.DEBUG_LIB_PATH)
    assert lib.gdn_debug_checks() == 1
    old = api.LIB
    api.LIB = lib
    try:
        yield api, lib
    finally:
        api.LIB = old


def no_violation(lib):
    import ctypes
    site, value = ctypes.c_int(0), ctypes.c_longlong(0)
    r = lib.gdn_debug_report(ctypes.byref(site), ctypes.byref(value))
    assert r == 0, f"debug check fired: site {site.value}, value {value.value}"


@pytest.mark.parametrize("mode", [1, 2, 3], ids=["split", "fused", "chunked"])
@pytest.mark.parametrize("shape", [(1, 2, 7, 129, 112, True), (2, 1, 5, 77, 64, False),
                                   (1, 3, 9, 300, 128, True)],
                         ids=lambda s: "B%dH%dT%dN%dD%d" % s[:5])
def test_forward_paths_under_checks(dbg, shape, mode):
    api, lib = dbg
    B, H, T, N, D, st = shape
    x = gdn_inputs.clip_inputs(B, H, T, N, D, seed=2000 + N, state_std=0.3 if st else 0.0)
    g = {k: (None if v is None else v.cuda()) for k, v in x.items()}
    old = os.environ.get("GDN_CHUNK_LEN")
    os.environ["GDN_CHUNK_LEN"] = "3"
    try:
        assert lib.gdn_set_forward_mode(mode) == 0
        out, s = api.gdn_frame_forward(g["q"], g["k"], g["v"], g["gamma"], g["beta"], g["state"])
        assert api.gdn_sync_status() == 0
    finally:
        lib.gdn_set_forward_mode(0)
        if old is None:
            os.environ.pop("GDN_CHUNK_LEN", None)
        else:
            os.environ["GDN_CHUNK_LEN"] = old
    no_violation(lib)
    ks = 1.0 / math.sqrt(D * N)
    o_ref, s_ref = oracle.gdn_frame_forward(f64(x["q"]), f64(x["k"]), f64(x["v"]), f64(x["gamma"]),
                                            f64(x["beta"]), None if x["state"] is None else f64(x["state"]), ks)
    assert relf(f64(out), o_ref) <= O_TOL and relf(f64(s), s_ref) <= S_TOL


def test_other_entry_points_under_checks(dbg):
    api, lib = dbg
    # streaming step (fused step kernel), in place
    y = gdn_inputs.clip_inputs(2, 2, 1, 100, 128, seed=2100, state_std=0.1)
    q, k, v = (y[n][:, 0].contiguous().cuda() for n in ("q", "k", "v"))
    gm, bt = y["gamma"][:, 0].contiguous().cuda(), y["beta"][:, 0].contiguous().cuda()
    st = y["state"].cuda()
    o, _ = api.gdn_frame_step(q, k, v, gm, bt, st, state_out=st)
    assert api.gdn_sync_status() == 0
    ks = 1.0 / math.sqrt(128 * 100)
    o_ref, s_ref = oracle.gdn_frame_step(f64(y["q"][:, 0]), f64(y["k"][:, 0]), f64(y["v"][:, 0]),
                                         f64(y["gamma"][:, 0]), f64(y["beta"][:, 0]),
                                         f64(y["state"]), ks)
    assert relf(f64(o), o_ref) <= O_TOL and relf(f64(st), s_ref) <= S_TOL
    no_violation(lib)

    # block-causal LA with a partial last block
    z = gdn_inputs.clip_inputs(1, 2, 7, 50, 112, seed=2101)
    o3, s3, z3 = api.gdn_block_causal_la(z["q"].cuda(), z["k"].cuda(), z["v"].cuda(), 3)
    assert api.gdn_sync_status() == 0
    r3 = oracle.la_block_causal(f64(z["q"]), f64(z["k"]), f64(z["v"]), None, None, 3)
    assert relf(f64(o3), r3[0]) <= O_TOL and relf(f64(s3), r3[1]) <= S_TOL
    no_violation(lib)

    # fp8 inputs
    e = gdn_inputs.clip_inputs(1, 2, 5, 100, 128, seed=2102)
    q8, sq = gdn_inputs.quantize_e4m3(e["q"])
    k8, sk = gdn_inputs.quantize_e4m3(e["k"])
    v8, sv = gdn_inputs.quantize_e4m3(e["v"])
    o5, s5 = api.gdn_frame_forward_fp8(*(t.cuda() for t in (q8, k8, v8, sq, sk, sv, e["gamma"],
                                                             e["beta"])))
    assert api.gdn_sync_status() == 0
    r5 = oracle.gdn_frame_forward_fp8(q8.numpy(), k8.numpy(), v8.numpy(), f64(sq), f64(sk), f64(sv),
                                      f64(e["gamma"]), f64(e["beta"]), None,
                                      1.0 / math.sqrt(128 * 100))
    assert relf(f64(o5), r5[0]) <= O_TOL and relf(f64(s5), r5[1]) <= S_TOL
    no_violation(lib)

    # fused 3D RoPE prologue, and the standalone pass
    r = gdn_inputs.clip_inputs(1, 2, 4, 130, 128, seed=2103)
    gr = {n: r[n].cuda() for n in ("q", "k", "v", "gamma", "beta")}
    o6, s6 = api.gdn_frame_forward_rope(gr["q"], gr["k"], gr["v"], gr["gamma"], gr["beta"], 10, 13)
    rq = api.gdn_rope_3d(gr["q"], 10, 13, t_offset=3)
    assert api.gdn_sync_status() == 0
    qr = oracle.rope_3d(f64(r["q"]), 10, 13)
    kr = oracle.rope_3d(f64(r["k"]), 10, 13)
    r6 = oracle.gdn_frame_forward(qr, kr, f64(r["v"]), f64(r["gamma"]), f64(r["beta"]), None,
                                  1.0 / math.sqrt(128 * 130))
    assert relf(f64(o6), r6[0]) <= O_TOL and relf(f64(s6), r6[1]) <= S_TOL
    assert relf(f64(rq), oracle.rope_3d(f64(r["q"]), 10, 13, 10000.0, 3)) <= 5e-3
    no_violation(lib)

    # softmax attention, chunk-causal with a ragged clip
    a = gdn_inputs.clip_inputs(1, 2, 5, 70, 128, seed=2104)
    o7 = api.gdn_softmax_attention(a["q"].cuda(), a["k"].cuda(), a["v"].cuda(), 2)
    assert api.gdn_sync_status() == 0
    r7 = oracle.softmax_attention_chunk_causal(f64(a["q"]), f64(a["k"]), f64(a["v"]), 2)
    assert relf(f64(o7), r7) <= O_TOL
    no_violation(lib)


def test_backward_under_checks(dbg):
    api, lib = dbg
    B, H, T, N, D = 1, 2, 6, 90, 128
    x = gdn_inputs.clip_inputs(B, H, T, N, D, seed=2110, state_std=0.2)
    c = gdn_inputs.cotangents(B, H, T, N, D, seed=2111, state_std=1.0)
    old = os.environ.get("GDN_BWD_SEGMENT_FRAMES")
    os.environ["GDN_BWD_SEGMENT_FRAMES"] = "2"
    try:
        got = api.gdn_frame_backward(*(x[n].cuda() for n in ("q", "k", "v", "gamma", "beta")),
                                     c["d_out"].cuda(), state_in=x["state"].cuda(),
                                     d_state_out=c["d_state"].cuda())
        assert api.gdn_sync_status() == 0
    finally:
        if old is None:
            os.environ.pop("GDN_BWD_SEGMENT_FRAMES", None)
        else:
            os.environ["GDN_BWD_SEGMENT_FRAMES"] = old
    no_violation(lib)
    refs = oracle.gdn_frame_backward(*(f64(x[n]) for n in ("q", "k", "v", "gamma", "beta", "state")),
                                     f64(c["d_out"]), f64(c["d_state"]), 1.0 / math.sqrt(D * N))
    for got_t, ref, tol in zip(got, refs, (1e-2, 1e-2, 1e-2, 2e-2, 2e-2, 5e-3)):
        assert relf(f64(got_t), ref) <= tol
