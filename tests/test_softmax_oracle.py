"""Pins of the softmax-attention oracle (``oracle/softmax_oracle.py``), CPU only.

They check facts that do not come from the oracle:
* a hand-worked example;
* brute force per query with explicit loops on tiny inputs;
* the mask's invariants: chunk causality, bidirectionality inside a chunk, F >= T as full
  attention;
* the softmax's invariants: equal scores give the mean of the visible values, a per-query
  shift of every score changes nothing, and a large scale selects the highest-scoring key.

Planted mistakes in copies of the oracle each fail at least one pin.
"""
import math

import numpy as np
import pytest

import oracle


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def pin_hand_example(attn):
    """D = N = 1, two frames, one frame per chunk. Frame 0 sees only itself, so out_0 = v_0. Frame
    1 sees scores q_1 k_0 s = 0 and q_1 k_1 s = ln 3 (s = 1), so its weights are 1/4 and 3/4
    and out_1 = (v_0 + 3 v_1) / 4."""
    q = np.array([2.0, 1.0]).reshape(1, 2, 1, 1, 1)
    k = np.array([0.0, math.log(3.0)]).reshape(1, 2, 1, 1, 1)
    v = np.array([4.0, 8.0]).reshape(1, 2, 1, 1, 1)
    out = attn(q, k, v, 1, 1.0).ravel()
    assert abs(out[0] - 4.0) < 1e-12
    assert abs(out[1] - (4.0 + 3 * 8.0) / 4) < 1e-12


def _brute(q, k, v, F, scale):
    B, T, N, H, D = q.shape
    out = np.zeros(q.shape)
    for b in range(B):
        for h in range(H):
            for t in range(T):
                for n in range(N):
                    num = np.zeros(D)
                    den = 0.0
                    for t2 in range(T):
                        if t2 // F > t // F:
                            continue
                        for n2 in range(N):
                            e = math.exp(scale * float(np.dot(q[b, t, n, h], k[b, t2, n2, h])))
                            num += e * v[b, t2, n2, h]
                            den += e
                    out[b, t, n, h] = num / den
    return out


def pin_brute_force(attn):
    q, k, v = (_rand((2, 5, 3, 2, 4), s) for s in (1, 2, 3))
    for F in (1, 2, 3, 5, 7):
        got = attn(q, k, v, F, 0.5)
        assert np.allclose(got, _brute(q, k, v, F, 0.5), rtol=1e-12, atol=1e-12), F


def pin_default_scale(attn):
    q, k, v = (_rand((1, 3, 4, 1, 16), s) for s in (4, 5, 6))
    assert np.allclose(attn(q, k, v, 2, None), _brute(q, k, v, 2, 1.0 / 4.0), atol=1e-12)


def pin_chunk_causality(attn):
    """Changing the keys and values of later chunks changes no output of earlier chunks, and
    changes an earlier frame of the same chunk (bidirectional inside a chunk)."""
    q, k, v = (_rand((1, 6, 3, 1, 4), s) for s in (7, 8, 9))
    F = 2
    base = attn(q, k, v, F, 0.5)
    k2, v2 = k.copy(), v.copy()
    k2[:, 4:] += 1.0
    v2[:, 4:] -= 2.0
    other = attn(q, k2, v2, F, 0.5)
    assert np.array_equal(base[:, :4], other[:, :4])
    assert not np.allclose(base[:, 4:], other[:, 4:])
    k3 = k.copy()
    k3[:, 3] += 1.0  # frame 3, chunk 1: frame 2's output must change
    assert not np.allclose(attn(q, k3, v, F, 0.5)[:, 2], base[:, 2])


def pin_full_attention(attn):
    """F >= T is one chunk, full softmax attention over the clip per head."""
    q, k, v = (_rand((2, 3, 4, 2, 8), s) for s in (10, 11, 12))
    for b in range(2):
        for h in range(2):
            Q = q[b, :, :, h].reshape(-1, 8)
            K = k[b, :, :, h].reshape(-1, 8)
            V = v[b, :, :, h].reshape(-1, 8)
            w = np.exp(Q @ K.T * 0.3)
            ref = (w / w.sum(1, keepdims=True)) @ V
            for F in (3, 4, 100):
                got = attn(q, k, v, F, 0.3)[b, :, :, h].reshape(-1, 8)
                assert np.allclose(got, ref, atol=1e-12)


def pin_equal_scores_give_the_mean(attn):
    """q = 0: every visible key has the same score, so the output is the mean of the visible
    values (all frames of chunks up to the query's chunk)."""
    _, k, v = (_rand((1, 5, 2, 1, 3), s) for s in (13, 14, 15))
    q = np.zeros(k.shape)
    out = attn(q, k, v, 2, 1.0)
    for t in range(5):
        t_end = min((t // 2 + 1) * 2, 5)
        mean = v[0, :t_end, :, 0].reshape(-1, 3).mean(0)
        for n in range(2):
            assert np.allclose(out[0, t, n, 0], mean, atol=1e-12)


def pin_score_shift_invariance(attn):
    """Adding the same vector u to every key shifts each query's scores by one constant
    (q . u * scale), which the softmax ignores."""
    q, k, v = (_rand((1, 4, 3, 2, 5), s) for s in (16, 17, 18))
    u = _rand((5,), 19)
    assert np.allclose(attn(q, k, v, 2, 0.7), attn(q, k + u, v, 2, 0.7), atol=1e-11)


def pin_large_scale_selects_the_max(attn):
    """With a very large scale the softmax becomes a one-hot choice of the highest-scoring
    visible key."""
    q, k, v = (_rand((1, 3, 2, 1, 4), s) for s in (20, 21, 22))
    out = attn(q, k, v, 1, 1e6)
    for t in range(3):
        for n in range(2):
            keys = k[0, :t + 1, :, 0].reshape(-1, 4)
            vals = v[0, :t + 1, :, 0].reshape(-1, 4)
            best = int(np.argmax(keys @ q[0, t, n, 0]))
            assert np.allclose(out[0, t, n, 0], vals[best], atol=1e-9)


PINS = [pin_hand_example, pin_brute_force, pin_default_scale, pin_chunk_causality,
        pin_full_attention, pin_equal_scores_give_the_mean, pin_score_shift_invariance,
        pin_large_scale_selects_the_max]


@pytest.mark.parametrize("pin", PINS, ids=lambda p: p.__name__)
def test_softmax_oracle_pin(pin):
    pin(oracle.softmax_attention_chunk_causal)


def _variant(mistake):
    """The oracle with one planted mistake."""
    def attn(q, k, v, F, scale=None):
        q, k, v = (np.asarray(x, float) for x in (q, k, v))
        B, T, N, H, D = q.shape
        s = (1.0 / D if mistake == "scale_1_over_D" else 1.0 / math.sqrt(D)) if scale is None else scale
        if mistake == "scale_dropped":
            s = 1.0
        out = np.zeros(q.shape)
        for b in range(B):
            for h in range(H):
                for t0 in range(0, T, F):
                    t1 = min(t0 + F, T)
                    kend = {"keys_up_to_chunk_start": t0 if t0 > 0 else t1,
                            "frame_causal": None}.get(mistake, t1)
                    Q = q[b, t0:t1, :, h].reshape(-1, D)
                    if mistake == "frame_causal":
                        rows = []
                        for t in range(t0, t1):
                            Kt = k[b, :t + 1, :, h].reshape(-1, D)
                            Vt = v[b, :t + 1, :, h].reshape(-1, D)
                            sc = q[b, t, :, h] @ Kt.T * s
                            w = np.exp(sc - sc.max(1, keepdims=True))
                            rows.append((w / w.sum(1, keepdims=True)) @ Vt)
                        out[b, t0:t1, :, h] = np.stack(rows)
                        continue
                    K = k[b, :kend, :, h].reshape(-1, D)
                    V = v[b, :kend, :, h].reshape(-1, D)
                    sc = Q @ K.T * s
                    w = np.exp(sc - sc.max(1, keepdims=True))
                    axis = 0 if mistake == "softmax_over_queries" else 1
                    with np.errstate(all="ignore"):  # a mutant may divide 0 by 0
                        w = w / w.sum(axis, keepdims=True)
                    out[b, t0:t1, :, h] = (w @ V).reshape(t1 - t0, N, D)
        return out
    return attn


MISTAKES = ["scale_dropped", "scale_1_over_D", "keys_up_to_chunk_start", "frame_causal",
            "softmax_over_queries"]


@pytest.mark.parametrize("mistake", MISTAKES)
def test_softmax_mutant_is_caught(mistake):
    attn = _variant(mistake)
    failed = []
    for pin in PINS:
        try:
            pin(attn)
        except (AssertionError, FloatingPointError, ValueError):
            failed.append(pin.__name__)
    assert failed, f"mutant {mistake} passes every pin"


def test_unmutated_variant_passes():
    attn = _variant("none")
    for pin in PINS:
        pin(attn)
