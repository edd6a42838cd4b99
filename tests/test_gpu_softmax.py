"""GPU parity of gdn_softmax_attention (through the C ABI) against the fp64 oracle's chunk-causal
softmax attention, element by element on the same seeded inputs.

Bars: relative Frobenius error of the output <= 1e-2 (the layer's output bar), and every element
within 2^-6 of the oracle's value, relative, plus 2e-2 of the output's rms. The kernel rounds P to
bf16 for the second product (2^-9 relative per weight), takes 2^x with the hardware's approximate
exponential (about 2 ulp of f32) and rounds O to bf16 once (2^-9 relative); a wrong mask or a lost
rescale moves elements by the output's rms or more.
"""
import math

import numpy as np
import pytest
import torch

import gdn_inputs
import oracle

from tests import parity_util as pu

pytestmark = pytest.mark.gpu

O_TOL = 1e-2


def api():
    from frame_wise_gated_deltanet_b200 import api as a
    return a


def f64(t):
    return t.detach().to(torch.float32).cpu().numpy().astype(np.float64)


def check(got, ref):
    g = np.asarray(got, dtype=np.float64)
    rms = math.sqrt(float(np.mean(ref ** 2)))
    e = float(np.linalg.norm(g - ref) / max(np.linalg.norm(ref), 1e-300))
    bound = 2.0 ** -6 * np.abs(ref) + 2e-2 * rms
    worst = float(np.max(np.abs(g - ref) / bound))
    assert e <= O_TOL and worst <= 1.0, f"relF {e:.2e}, worst element at {worst:.2f} of its bound"
    return e, worst


CASES = [
    # (B, H, T, N, D, F)
    (1, 2, 4, 50, 64, 1),      # frame-causal, 200 tokens: a ragged second query tile
    (1, 2, 6, 100, 128, 2),    # chunks of two frames: tiles straddle chunk ends
    (2, 1, 5, 77, 128, 5),     # one chunk: fully bidirectional
    (1, 3, 7, 40, 64, 3),      # a partial last chunk
    (1, 1, 3, 129, 112, 2),    # padded head dim
    (1, 2, 2, 16, 32, 1),      # tiny
    (1, 1, 1, 1, 128, 1),      # a single token
    (1, 1, 9, 300, 128, 4),    # 22 query tiles over up to 22 key tiles (online rescaling)
    (2, 2, 3, 64, 96, 9),      # F > T: bidirectional
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "B%dH%dT%dN%dD%dF%d" % c)
def test_softmax_attention_matches_oracle(case):
    B, H, T, N, D, F = case
    x = gdn_inputs.clip_inputs(B, H, T, N, D, seed=1400 + N + D + F)
    out = api().gdn_softmax_attention(x["q"].cuda(), x["k"].cuda(), x["v"].cuda(), F)
    assert api().gdn_sync_status() == 0
    ref = oracle.softmax_attention_chunk_causal(f64(x["q"]), f64(x["k"]), f64(x["v"]), F)
    check(f64(out), ref)


def test_softmax_attention_explicit_scale():
    """A scale other than 1/sqrt(D) (a sharper softmax: larger score spread, more rescaling)."""
    B, H, T, N, D, F = 1, 2, 4, 90, 128, 2
    x = gdn_inputs.clip_inputs(B, H, T, N, D, seed=1450)
    out = api().gdn_softmax_attention(x["q"].cuda(), x["k"].cuda(), x["v"].cuda(), F, scale=0.3)
    assert api().gdn_sync_status() == 0
    ref = oracle.softmax_attention_chunk_causal(f64(x["q"]), f64(x["k"]), f64(x["v"]), F, 0.3)
    check(f64(out), ref)


def test_softmax_attention_deterministic():
    x = gdn_inputs.clip_inputs(1, 2, 5, 200, 128, seed=1460, device="cuda")
    a = api().gdn_softmax_attention(x["q"], x["k"], x["v"], 2)
    b = api().gdn_softmax_attention(x["q"], x["k"], x["v"], 2)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


@pytest.mark.parametrize("name", ["softmax_480p", "softmax_720p21"])
def test_softmax_attention_bench_workloads_all_heads(name):
    """The benchmark's softmax workloads (the 480p clip's shape and 21 frames of the 720p grid,
    chunks of 3 frames) in their launch configuration; the oracle recomputes every head, and the
    errors are those of the whole output tensor."""
    w = gdn_inputs.WORKLOADS[name]
    H, F = w.H, w.frames_per_block
    x = gdn_inputs.workload_inputs(w, device="cuda")
    out = api().gdn_softmax_attention(x["q"], x["k"], x["v"], F)
    assert api().gdn_sync_status() == 0

    def one(h):
        sl = lambda t: pu.f32(t[:, :, :, h:h + 1])
        ref = oracle.softmax_attention_chunk_causal(sl(x["q"]), sl(x["k"]), sl(x["v"]), F)
        e = pu.RelF()
        g = sl(out)
        e.add(g, ref, h)
        rms = math.sqrt(float(np.mean(ref ** 2)))
        worst = float(np.max(np.abs(g - ref) / (2.0 ** -6 * np.abs(ref) + 2e-2 * rms)))
        return e, worst

    tot = pu.RelF()
    worst = 0.0
    for e, wst in pu.pool_map(one, range(H), bytes_per_task=4e9):
        tot.merge(e)
        worst = max(worst, wst)
    pu.log(name + "_all_heads", out=tot, worst_element_of_bound=worst)
    assert tot.value <= O_TOL and worst <= 1.0, f"relF {tot.value:.2e}, worst {worst:.2f}"
