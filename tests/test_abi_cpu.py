"""The C-ABI library loads without a GPU, exports every symbol include/gdn.h declares, and its
host-side argument checks answer before any CUDA call (CPU only; no compute calls)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gdn.h")


def _declared_symbols():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(gdn_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    from frame_wise_gated_deltanet_b200 import build
    build.build()
    from frame_wise_gated_deltanet_b200 import _lib
    return _lib.LIB


def test_header_declares_the_entry_points():
    syms = _declared_symbols()
    for s in ("gdn_frame_forward", "gdn_frame_forward_host", "gdn_frame_step", "gdn_frame_stats",
              "gdn_block_causal_la", "gdn_status_string", "gdn_sync_status",
              "gdn_release_workspace"):
        assert s in syms


def test_every_declared_symbol_is_exported(lib):
    from frame_wise_gated_deltanet_b200 import _lib
    syms = _declared_symbols()
    for s in syms:
        assert hasattr(lib, s), f"libgdn.so does not export {s}"
        assert s in _lib.SIGNATURES, f"binding has no signature for {s}"
    assert set(_lib.SIGNATURES) == set(syms)


def test_status_strings(lib):
    for code in range(7):
        assert lib.gdn_status_string(code)
    assert lib.gdn_version() >= 100


def test_workspace_sizes(lib):
    # 720p clip: per frame-head A (bf16) + B (f32) + S (bf16) = 128 KiB, plus for the chunked
    # forward (chunks of >= 4 frames) one 128 KiB record of composed maps per chunk boundary
    # and one 64 KiB f32 start state per chunk
    split = 1 * 20 * 961 * 128 * 128 * (2 + 4 + 2)
    n = lib.gdn_workspace_bytes(1, 20, 961, 880, 128)
    assert n >= split
    assert n < split + 20 * 241 * (128 + 64) * 1024 + 4096
    assert lib.gdn_la_workspace_bytes(2, 20, 81, 112) >= 2 * 20 * 81 * 113 * 112 * 6
    assert lib.gdn_workspace_bytes(0, 1, 1, 1, 8) == 0


P = 4096  # a fake, 16-byte aligned "device address"; never dereferenced by these calls


def _fwd(lib, q=P, k=P + 0x10000, v=P + 0x20000, g=P + 0x30000, b=P + 0x31000, si=None,
         out=P + 0x40000, so=None, B=1, H=2, T=3, N=16, D=32, ks=0.1):
    return lib.gdn_frame_forward(q, k, v, g, b, si, out, so, B, H, T, N, D, ks, None)


def test_forward_rejects_bad_arguments_on_the_host(lib):
    assert _fwd(lib, q=None) == 1
    assert _fwd(lib, g=None) == 1
    assert _fwd(lib, B=0) == 1
    assert _fwd(lib, N=0) == 1
    assert _fwd(lib, D=36) == 2     # not a multiple of 8
    assert _fwd(lib, D=136) == 2    # above 128
    assert _fwd(lib, ks=-0.5) == 1
    assert _fwd(lib, ks=float("nan")) == 1
    assert _fwd(lib, ks=float("inf")) == 1
    assert _fwd(lib, q=P + 8) == 3  # misaligned
    assert _fwd(lib, out=P + 0x10000) == 1  # out overlaps k


def _fwd_host(lib, q=P, k=P + 0x10000, v=P + 0x20000, g=P + 0x30000, b=P + 0x31000, si=None,
              out=P + 0x40000, so=None, B=1, H=2, T=3, N=16, D=32, ks=0.1):
    return lib.gdn_frame_forward_host(q, k, v, g, b, si, out, so, B, H, T, N, D, ks, None)


def test_forward_host_rejects_bad_arguments_on_the_host(lib):
    assert _fwd_host(lib, v=None) == 1
    assert _fwd_host(lib, out=None) == 1
    assert _fwd_host(lib, T=0) == 1
    assert _fwd_host(lib, D=20) == 2
    assert _fwd_host(lib, ks=-1.0) == 1
    assert _fwd_host(lib, out=P + 0x20000) == 1   # out overlaps v
    # host buffers need no 16-byte alignment; without a GPU the call then fails loudly
    import torch
    if not torch.cuda.is_available():
        assert _fwd_host(lib, q=P + 2) == 5


def test_forward_fp8_rejects_bad_arguments_on_the_host(lib):
    f = lib.gdn_frame_forward_fp8
    args = lambda D=128, qs=P + 0x50000, ks=0.1: (P, P + 0x10000, P + 0x20000, qs, P + 0x51000,
                                                  P + 0x52000, P + 0x30000, P + 0x31000, None,
                                                  P + 0x40000, None, 1, 2, 3, 16, D, ks, None)
    assert f(*args(qs=None)) == 1
    assert f(*args(D=64)) == 2      # fp8 path: 64 < D <= 128
    assert f(*args(D=120)) == 2     # D % 16 != 0
    assert f(*args(ks=-1.0)) == 1
    import torch
    if not torch.cuda.is_available():
        assert f(*args()) == 5


def test_valid_call_without_gpu_fails_loudly(lib):
    # Arguments pass the host checks, then the library needs a CUDA device: no CPU fallback.
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    assert _fwd(lib) == 5


def test_la_rejects_bad_arguments_on_the_host(lib):
    f = lib.gdn_block_causal_la
    assert f(P, P + 0x10000, P + 0x20000, None, None, P + 0x40000, None, None, 1, 1, 4, 8, 128,
             2, None) == 2  # D = 128 leaves no column for the normaliser
    assert f(P, P + 0x10000, P + 0x20000, None, None, P + 0x40000, None, None, 1, 1, 4, 8, 32,
             0, None) == 1  # frames_per_block < 1


def test_binding_refuses_cpu_tensors():
    import torch
    from frame_wise_gated_deltanet_b200 import api
    q = torch.zeros((1, 2, 16, 2, 32), dtype=torch.bfloat16)
    g = torch.zeros((1, 2, 2), dtype=torch.float32)
    with pytest.raises(ValueError):
        api.gdn_frame_forward(q, q, q, g, g)


def test_backward_rejects_bad_arguments_on_the_host(lib):
    f = lib.gdn_frame_backward
    # q, k, v, gamma, beta, state_in, d_out, d_state_out, dq, dk, dv, d_gamma, d_beta, d_state_in
    def args(D=128, dq=P + 0x60000, dgam=P + 0x90000, ks=0.1, q=P, dsi=None, si=None):
        return (q, P + 0x10000, P + 0x20000, P + 0x30000, P + 0x31000, si, P + 0x40000, None,
                dq, P + 0x70000, P + 0x80000, dgam, P + 0x91000, dsi, 1, 2, 3, 16, D, ks, None)
    assert f(*args(q=None)) == 1
    assert f(*args(D=64)) == 2            # backward: 64 < D <= 128
    assert f(*args(D=100)) == 2           # D % 8 != 0
    assert f(*args(ks=float("nan"))) == 1
    assert f(*args(dq=P + 0x60008)) == 3  # misaligned
    assert f(*args(dq=P + 0x10000)) == 1  # dq overlaps k
    assert f(*args(dgam=P + 0x31000)) == 1  # d_gamma overlaps beta
    assert f(*args(si=P + 0xA0000, dsi=P + 0xA0000)) == 1  # d_state_in overlaps state_in
    import torch
    if not torch.cuda.is_available():
        assert f(*args()) == 5
    assert lib.gdn_backward_workspace_bytes(1, 20, 961, 880, 128) > 19220 * 250_000


def test_backward_binding_refuses_cpu_tensors():
    import torch
    from frame_wise_gated_deltanet_b200 import api
    q = torch.zeros((1, 2, 16, 2, 128), dtype=torch.bfloat16)
    g = torch.zeros((1, 2, 2), dtype=torch.float32)
    with pytest.raises(ValueError):
        api.gdn_frame_backward(q, q, q, g, g, q)


def test_rope_rejects_bad_arguments_on_the_host(lib):
    f = lib.gdn_rope_3d
    args = lambda D=128, gh=2, gw=8, base=10000.0, toff=0, y=P + 0x40000: (
        P, y, 1, 3, 16, 2, D, gh, gw, base, toff, None)
    assert f(*args(D=100)) == 2          # D % 8 != 0
    assert f(*args(gh=3)) == 1           # grid_h * grid_w != N
    assert f(*args(base=1.0)) == 1
    assert f(*args(toff=-1)) == 1
    assert f(*args(y=P + 0x10)) == 1     # partial overlap with x
    assert f(*args(y=P + 0x40008)) == 3  # misaligned
    import torch
    if not torch.cuda.is_available():
        assert f(*args()) == 5
        assert f(*args(y=P)) == 5        # in place passes the host checks


def test_zero_key_scale_selects_the_default_in_the_library(lib):
    """key_scale == 0 is the documented request for the layer's 1/sqrt(D*N): the host checks
    accept it (and the call then needs a GPU), and the header states the convention."""
    import torch
    text = open(HEADER).read()
    assert "0 selects the pages' key scale" in text and "1/sqrt(D*N)" in text
    if not torch.cuda.is_available():
        assert _fwd(lib, ks=0.0) == 5
        assert _fwd_host(lib, ks=0.0) == 5


def test_binding_holds_no_key_scale_arithmetic():
    """The Python binding passes key_scale through (None as 0); the default scale is computed
    in the library."""
    src = open(os.path.join(ROOT, "frame_wise_gated_deltanet_b200", "api.py")).read()
    for pattern in ("math.", "np.sqrt", "torch.sqrt", "rsqrt", "** 0.5", "** -0.5", "import math"):
        assert pattern not in src, pattern


def test_forward_rope_rejects_bad_arguments_on_the_host(lib):
    f = lib.gdn_frame_forward_rope

    def args(D=32, gh=4, gw=4, base=10000.0, toff=0, ks=0.1, q=P):
        return (q, P + 0x10000, P + 0x20000, P + 0x30000, P + 0x31000, None, P + 0x40000, None,
                1, 2, 3, 16, D, ks, gh, gw, base, toff, None)
    assert f(*args(q=None)) == 1
    assert f(*args(D=36)) == 2           # not a multiple of 8
    assert f(*args(gh=3)) == 1           # grid_h * grid_w != N
    assert f(*args(base=1.0)) == 1
    assert f(*args(base=float("nan"))) == 1
    assert f(*args(toff=-1)) == 1
    assert f(*args(ks=-1.0)) == 1
    assert f(*args(q=P + 8)) == 3        # misaligned
    import torch
    if not torch.cuda.is_available():
        assert f(*args()) == 5


def test_softmax_attention_rejects_bad_arguments_on_the_host(lib):
    f = lib.gdn_softmax_attention

    def args(D=64, F=2, scale=0.0, out=P + 0x40000, q=P):
        return (q, P + 0x10000, P + 0x20000, out, 1, 2, 3, 16, D, F, scale, None)
    assert f(*args(q=None)) == 1
    assert f(*args(F=0)) == 1            # frames_per_chunk < 1
    assert f(*args(D=36)) == 2           # not a multiple of 8
    assert f(*args(D=136)) == 2          # above 128
    assert f(*args(scale=-1.0)) == 1
    assert f(*args(scale=float("inf"))) == 1
    assert f(*args(out=P + 0x10000)) == 1  # out overlaps k
    assert f(*args(out=P + 0x40008)) == 3  # misaligned
    import torch
    if not torch.cuda.is_available():
        assert f(*args()) == 5


def test_debug_library_builds_and_exports_the_same_symbols(lib):
    """libgdn_debug.so (the device-side checks) exports every declared symbol and says it has
    the checks; the release library compiles them out."""
    from frame_wise_gated_deltanet_b200 import _lib, build
    build.build(debug=True)
    dbg = _lib.load(_lib.DEBUG_LIB_PATH)
    for s in _declared_symbols():
        assert hasattr(dbg, s), f"libgdn_debug.so does not export {s}"
    assert dbg.gdn_debug_checks() == 1
    assert lib.gdn_debug_checks() == 0


def test_training_pair_rejects_bad_arguments_on_the_host(lib):
    f = lib.gdn_frame_forward_train
    S = P + 0x100000  # 256-byte aligned fake "saved" buffer

    def fa(D=128, saved=S, q=P):
        return (q, P + 0x10000, P + 0x20000, P + 0x30000, P + 0x31000, None, P + 0x40000, None,
                saved, 1, 2, 3, 16, D, 0.0, None)
    assert f(*fa(saved=None)) == 1
    assert f(*fa(D=64)) == 2             # the pair needs 64 < D <= 128
    assert f(*fa(saved=S + 16)) == 3     # saved must be 256-byte aligned
    assert f(*fa(saved=P + 0x20000)) == 1  # saved overlaps v
    assert lib.gdn_train_saved_bytes(1, 2, 3, 16, 64) == 0
    assert lib.gdn_train_saved_bytes(1, 20, 961, 880, 128) == lib.gdn_workspace_bytes(1, 20, 961, 880, 128) or \
        lib.gdn_train_saved_bytes(1, 20, 961, 880, 128) >= 19220 * 128 * 1024
    b = lib.gdn_frame_backward_saved

    def ba(saved=S, dq=P + 0x60000):
        return (P, P + 0x10000, P + 0x20000, P + 0x30000, P + 0x31000, None, saved, P + 0x40000,
                None, dq, P + 0x70000, P + 0x80000, P + 0x90000, P + 0x91000, None,
                1, 2, 3, 16, 128, 0.0, None)
    assert b(*ba(saved=None)) == 1
    assert b(*ba(saved=S + 8)) == 3
    assert b(*ba(dq=P + 0x10000)) == 1   # dq overlaps k
    import torch
    if not torch.cuda.is_available():
        assert f(*fa()) == 5
        assert b(*ba()) == 5
