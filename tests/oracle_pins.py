"""Pins for the fp64 oracle: checks against facts that do not come from the oracle.

Each ``pin_*`` function takes an implementation namespace ``impl`` (an object
with ``gdn_frame_forward``, ``gdn_frame_step``, ``la_block_causal``,
``frame_statistics``, ``e4m3_decode``, ``gdn_frame_forward_fp8`` and ``gdn_frame_backward``
attributes,
the same signatures as ``oracle.gdn_oracle``)
and raises ``AssertionError`` if the implementation disagrees with:

* the hand-worked examples under ``tests/golden/``;
* closed forms (single frame from S_0 = 0; beta = 0 pure decay);
* special cases that reduce to a textbook routine (N = 1 is the token-wise
  gated delta rule in residual form; block-causal LA equals brute-force
  quadratic block-causal attention);
* the E4M3 format's definition (landmark codes, ordering, spacing) and the
  scale algebra of the fp8 forward;
* exact invariants (delta-rule exactness for orthonormal keys; the consistent
  linear map is a fixed point; split/resume through the state; linearity in
  (V, S_0); causality across frames and bidirectionality inside a frame; the
  unrolled affine-map product form of the recurrence);
* for the backward: a hand-worked scalar example (``tests/golden/``), central differences of
  the forward, the exact dot-product (adjoint)
  identity of the map (V, S_0) -> (O, S_T), which is linear, the textbook gradients of
  unnormalised linear attention (one frame from a zero state), and linearity in the
  cotangents.

``tests/test_oracle_mutations.py`` plants plausible mistakes in copies of the
oracle and checks that each one fails at least one pin.
"""
from __future__ import annotations

import json
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")

_rng_seed = 12345


def _rng(extra=0):
    return np.random.default_rng(_rng_seed + extra)


def _rand_clip(B, T, N, H, D, rng, g=(0.9, 0.999), b=(0.1, 0.9)):
    q = rng.standard_normal((B, T, N, H, D))
    k = rng.standard_normal((B, T, N, H, D))
    v = rng.standard_normal((B, T, N, H, D))
    gamma = rng.uniform(*g, size=(B, T, H))
    beta = rng.uniform(*b, size=(B, T, H))
    return q, k, v, gamma, beta


def _close(a, b, tol=1e-10, what=""):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    assert a.shape == b.shape, f"{what}: shape {a.shape} vs {b.shape}"
    scale = max(1.0, float(np.max(np.abs(b))) if b.size else 1.0)
    err = float(np.max(np.abs(a - b))) if a.size else 0.0
    assert err <= tol * scale, f"{what}: max abs err {err:.3e} > {tol:.1e} * {scale:.3e}"


# --------------------------------------------------------------------------- GDN pins

def pin_hand_example(impl):
    """Exact rationals worked by hand from the definition (tests/golden/gdn_hand_example.json)."""
    with open(os.path.join(GOLDEN, "gdn_hand_example.json")) as f:
        g = json.load(f)
    q = np.array(g["q"], dtype=np.float64)[None, :, :, None, :]  # [1,T,N,1,D]
    k = np.array(g["k"], dtype=np.float64)[None, :, :, None, :]
    v = np.array(g["v"], dtype=np.float64)[None, :, :, None, :]
    gamma = np.array(g["gamma"])[None, :, None]
    beta = np.array(g["beta"])[None, :, None]
    out, st = impl.gdn_frame_forward(q, k, v, gamma, beta, None, g["key_scale"])
    _close(out[0, :, :, 0, :], g["expected_out"], 1e-14, "hand example O")
    _close(st[0, 0], g["expected_state_after_frame"][-1], 1e-14, "hand example S_T")
    # the state after frame 0 = state_out of the first frame alone
    _, st1 = impl.gdn_frame_forward(q[:, :1], k[:, :1], v[:, :1], gamma[:, :1], beta[:, :1],
                                    None, g["key_scale"])
    _close(st1[0, 0], g["expected_state_after_frame"][0], 1e-14, "hand example S_1")


def pin_single_frame_closed_form(impl):
    """S_0 = 0, one frame: S_1 = beta * s * V^T K and O = Q S_1^T (written as token sums)."""
    rng = _rng(1)
    B, T, N, H, D = 2, 1, 7, 3, 5
    q, k, v, gamma, beta = _rand_clip(B, T, N, H, D, rng)
    s = 0.37
    out, st = impl.gdn_frame_forward(q, k, v, gamma, beta, None, s)
    for b in range(B):
        for h in range(H):
            S1 = np.zeros((D, D))
            for i in range(N):
                S1 += np.outer(v[b, 0, i, h], k[b, 0, i, h])
            S1 *= beta[b, 0, h] * s
            _close(st[b, h], S1, 1e-12, "single frame S_1")
            for i in range(N):
                o = np.array([sum(S1[r, c] * q[b, 0, i, h, c] for c in range(D)) for r in range(D)])
                _close(out[b, 0, i, h], o, 1e-12, "single frame O")


def pin_pure_decay(impl):
    """beta = 0: S_T = (prod gamma) S_0 and O_t = (prod_{u<=t} gamma_u) Q_t S_0^T."""
    rng = _rng(2)
    B, T, N, H, D = 1, 6, 4, 2, 3
    q, k, v, gamma, _ = _rand_clip(B, T, N, H, D, rng)
    beta = np.zeros((B, T, H))
    S0 = rng.standard_normal((B, H, D, D))
    out, st = impl.gdn_frame_forward(q, k, v, gamma, beta, S0, 0.5)
    for h in range(H):
        p = 1.0
        for t in range(T):
            p *= gamma[0, t, h]
            _close(out[0, t, :, h], p * (q[0, t, :, h] @ S0[0, h].T), 1e-12, "decay O_t")
        _close(st[0, h], p * S0[0, h], 1e-12, "decay S_T")


def _tokenwise_gated_delta(qs, ks, vs, gs, bs, S0):
    """Textbook token-wise gated delta rule in residual form, one head:
    S <- gamma S + beta (v - gamma S k) k^T ; o = S q."""
    S = S0.copy()
    outs = []
    for q, k, v, g, b in zip(qs, ks, vs, gs, bs):
        pred = g * (S @ k)
        S = g * S + b * np.outer(v - pred, k)
        outs.append(S @ q)
    return np.array(outs), S


def pin_tokenwise_reduction(impl):
    """N = 1: one token per frame, so frame-wise GDN is the token-wise gated delta rule."""
    rng = _rng(3)
    B, T, N, H, D = 1, 9, 1, 2, 4
    q, k, v, gamma, beta = _rand_clip(B, T, N, H, D, rng)
    s = 0.6
    S0 = 0.3 * rng.standard_normal((B, H, D, D))
    out, st = impl.gdn_frame_forward(q, k, v, gamma, beta, S0, s)
    for h in range(H):
        o_ref, s_ref = _tokenwise_gated_delta(q[0, :, 0, h], s * k[0, :, 0, h], v[0, :, 0, h],
                                              gamma[0, :, h], beta[0, :, h], S0[0, h])
        _close(out[0, :, 0, h], o_ref, 1e-12, "token-wise O")
        _close(st[0, h], s_ref, 1e-12, "token-wise S_T")


def pin_delta_rule_exactness(impl):
    """beta = gamma = 1, unscaled orthonormal key rows: S_t k_i = v_i for every key of frame t."""
    rng = _rng(4)
    B, T, N, H, D = 1, 4, 5, 1, 8
    q = rng.standard_normal((B, T, N, H, D))
    v = rng.standard_normal((B, T, N, H, D))
    k = np.zeros((B, T, N, H, D))
    for t in range(T):
        Qm, _ = np.linalg.qr(rng.standard_normal((D, D)))
        k[0, t, :, 0, :] = Qm[:N]  # N orthonormal rows
    ones = np.ones((B, T, H))
    S0 = rng.standard_normal((B, H, D, D))
    state = S0
    for t in range(T):
        _, state = impl.gdn_frame_forward(q[:, t:t + 1], k[:, t:t + 1], v[:, t:t + 1],
                                          ones[:, t:t + 1], ones[:, t:t + 1], state, 1.0)
        for i in range(N):
            _close(state[0, 0] @ k[0, t, i, 0], v[0, t, i, 0], 1e-12, "S k_i = v_i")


def pin_fixed_point(impl):
    """gamma = 1, v_i = W (s k_i), S_0 = W: the state stays W for any beta; O_t = Q_t W^T."""
    rng = _rng(5)
    B, T, N, H, D = 1, 5, 6, 1, 4
    s = 0.45
    q = rng.standard_normal((B, T, N, H, D))
    k = rng.standard_normal((B, T, N, H, D))
    W = rng.standard_normal((D, D))
    v = np.einsum("ij,btnhj->btnhi", W, s * k)
    gamma = np.ones((B, T, H))
    beta = rng.uniform(0.0, 1.0, size=(B, T, H))
    out, st = impl.gdn_frame_forward(q, k, v, gamma, beta, W[None, None], s)
    _close(st[0, 0], W, 1e-11, "fixed point S_T")
    for t in range(T):
        _close(out[0, t, :, 0], q[0, t, :, 0] @ W.T, 1e-11, "fixed point O_t")


def pin_split_resume(impl):
    """forward(T) = forward(T1) then forward(T - T1) through state_out -> state_in."""
    rng = _rng(6)
    B, T, N, H, D = 2, 7, 5, 2, 4
    q, k, v, gamma, beta = _rand_clip(B, T, N, H, D, rng)
    S0 = rng.standard_normal((B, H, D, D))
    out, st = impl.gdn_frame_forward(q, k, v, gamma, beta, S0, 0.3)
    T1 = 3
    o1, s1 = impl.gdn_frame_forward(q[:, :T1], k[:, :T1], v[:, :T1], gamma[:, :T1],
                                    beta[:, :T1], S0, 0.3)
    o2, s2 = impl.gdn_frame_forward(q[:, T1:], k[:, T1:], v[:, T1:], gamma[:, T1:],
                                    beta[:, T1:], s1, 0.3)
    _close(np.concatenate([o1, o2], axis=1), out, 1e-12, "split O")
    _close(s2, st, 1e-12, "split S_T")


def pin_linearity(impl):
    """(O, S_T) is jointly linear in (V, S_0) for fixed Q, K, gamma, beta."""
    rng = _rng(7)
    B, T, N, H, D = 1, 4, 6, 2, 3
    q, k, v1, gamma, beta = _rand_clip(B, T, N, H, D, rng)
    v2 = rng.standard_normal(v1.shape)
    S1 = rng.standard_normal((B, H, D, D))
    S2 = rng.standard_normal((B, H, D, D))
    a, b = 1.7, -0.6
    o1, s1 = impl.gdn_frame_forward(q, k, v1, gamma, beta, S1, 0.4)
    o2, s2 = impl.gdn_frame_forward(q, k, v2, gamma, beta, S2, 0.4)
    o3, s3 = impl.gdn_frame_forward(q, k, a * v1 + b * v2, gamma, beta, a * S1 + b * S2, 0.4)
    _close(o3, a * o1 + b * o2, 1e-11, "linearity O")
    _close(s3, a * s1 + b * s2, 1e-11, "linearity S_T")


def pin_causal_across_bidirectional_within(impl):
    """Changing frame t+1 leaves O_<=t alone; changing one key of frame t moves every O of frame t."""
    rng = _rng(8)
    B, T, N, H, D = 1, 4, 5, 1, 4
    q, k, v, gamma, beta = _rand_clip(B, T, N, H, D, rng)
    out, _ = impl.gdn_frame_forward(q, k, v, gamma, beta, None, 0.5)
    k2, v2, q2 = k.copy(), v.copy(), q.copy()
    k2[:, 2:] += 1.0
    v2[:, 2:] -= 1.0
    q2[:, 2:] *= 3.0
    out2, _ = impl.gdn_frame_forward(q2, k2, v2, gamma, beta, None, 0.5)
    _close(out2[:, :2], out[:, :2], 1e-14, "causal across frames")
    k3 = k.copy()
    k3[0, 1, N - 1, 0, :] += 2.0  # last token of frame 1
    out3, _ = impl.gdn_frame_forward(q, k3, v, gamma, beta, None, 0.5)
    d = np.abs(out3[0, 1, :, 0] - out[0, 1, :, 0]).max(axis=-1)
    assert np.all(d > 1e-6), f"bidirectional within frame: unchanged rows {np.where(d <= 1e-6)}"
    _close(out3[0, 0], out[0, 0], 1e-14, "earlier frame unchanged")


def pin_unrolled_product_form(impl):
    """S_T = S_0 M_1 ... M_T + sum_t beta_t B_t M_{t+1} ... M_T,  M_t = gamma_t (I - beta_t A_t),
    with A_t and B_t written as token sums (the affine-map composition of the scan)."""
    rng = _rng(9)
    B, T, N, H, D = 1, 5, 6, 1, 4
    q, k, v, gamma, beta = _rand_clip(B, T, N, H, D, rng)
    s = 0.35
    S0 = rng.standard_normal((B, H, D, D))
    _, st = impl.gdn_frame_forward(q, k, v, gamma, beta, S0, s)
    Ms, Cs = [], []
    for t in range(T):
        A = sum(np.outer(s * k[0, t, i, 0], s * k[0, t, i, 0]) for i in range(N))
        Bm = sum(np.outer(v[0, t, i, 0], s * k[0, t, i, 0]) for i in range(N))
        Ms.append(gamma[0, t, 0] * (np.eye(D) - beta[0, t, 0] * A))
        Cs.append(beta[0, t, 0] * Bm)
    P = np.eye(D)
    for M in Ms:
        P = P @ M
    total = S0[0, 0] @ P
    for t in range(T):
        tail = np.eye(D)
        for M in Ms[t + 1:]:
            tail = tail @ M
        total = total + Cs[t] @ tail
    _close(st[0, 0], total, 1e-11, "unrolled product form")


def pin_stats_identity_keys(impl):
    """K = identity rows (N = D), s = 1: A = I and B = V^T."""
    rng = _rng(10)
    D = 6
    K = np.eye(D)
    V = rng.standard_normal((D, D))
    A, Bm = impl.frame_statistics(K, V, 1.0)
    _close(A, np.eye(D), 1e-15, "A = I")
    _close(Bm, V.T, 1e-15, "B = V^T")
    # A is symmetric PSD for any keys, and scales with s^2; B with s
    K = rng.standard_normal((9, D))
    A1, B1 = impl.frame_statistics(K, V[:1].repeat(9, 0), 1.0)
    A2, B2 = impl.frame_statistics(K, V[:1].repeat(9, 0), 0.5)
    _close(A1, A1.T, 1e-14, "A symmetric")
    assert np.linalg.eigvalsh(A1).min() > -1e-12, "A positive semidefinite"
    _close(A2, 0.25 * A1, 1e-14, "A ~ s^2")
    _close(B2, 0.5 * B1, 1e-14, "B ~ s")


def pin_step_is_single_frame(impl):
    """A streaming step equals a one-frame clip with the carried state."""
    rng = _rng(11)
    B, N, H, D = 3, 5, 2, 4
    q, k, v, gamma, beta = _rand_clip(B, 1, N, H, D, rng)
    S0 = rng.standard_normal((B, H, D, D))
    o, s = impl.gdn_frame_step(q[:, 0], k[:, 0], v[:, 0], gamma[:, 0], beta[:, 0], S0, 0.3)
    o_ref, s_ref = impl.gdn_frame_forward(q, k, v, gamma, beta, S0, 0.3)
    _close(o, o_ref[:, 0], 1e-13, "step O")
    _close(s, s_ref, 1e-13, "step S")
    # chained steps = one clip (the carried state is the checkpoint)
    T = 4
    q, k, v, gamma, beta = _rand_clip(B, T, N, H, D, rng)
    o_ref, s_ref = impl.gdn_frame_forward(q, k, v, gamma, beta, S0, 0.3)
    state = S0
    for t in range(T):
        o, state = impl.gdn_frame_step(q[:, t], k[:, t], v[:, t], gamma[:, t], beta[:, t],
                                       state, 0.3)
        _close(o, o_ref[:, t], 1e-12, "chained step O")
    _close(state, s_ref, 1e-12, "chained step S")


# --------------------------------------------------------------------------- LA pins

def pin_la_hand_example(impl):
    with open(os.path.join(GOLDEN, "la_hand_example.json")) as f:
        g = json.load(f)
    q = np.array(g["q"], dtype=np.float64)[None, :, :, None, :]
    k = np.array(g["k"], dtype=np.float64)[None, :, :, None, :]
    v = np.array(g["v"], dtype=np.float64)[None, :, :, None, :]
    out, st, z = impl.la_block_causal(q, k, v, None, None, g["frames_per_block"], g["eps"])
    num = np.array(g["expected_numerator"], dtype=np.float64)
    den = np.array(g["expected_denominator"], dtype=np.float64)
    _close(out[0, :, :, 0, :], num / den[..., None], 1e-12, "LA hand O")
    _close(st[0, 0], g["expected_state"], 1e-14, "LA hand S")
    _close(z[0, 0], g["expected_z"], 1e-14, "LA hand z")


def _la_brute_force(q, k, v, F, eps):
    """Quadratic block-causal attention with a ReLU kernel: token i of block b attends to every
    token j of blocks <= b with weight relu(q_i).relu(k_j), normalised by the weight sum + eps."""
    B, T, N, H, D = q.shape
    out = np.zeros(q.shape)
    for b in range(B):
        for h in range(H):
            for t in range(T):
                last = min((t // F + 1) * F, T)
                Kc = np.maximum(k[b, :last, :, h].reshape(-1, D), 0.0)
                Vc = v[b, :last, :, h].reshape(-1, D)
                for i in range(N):
                    w = Kc @ np.maximum(q[b, t, i, h], 0.0)
                    out[b, t, i, h] = (w @ Vc) / (w.sum() + eps)
    return out


def pin_la_brute_force(impl):
    rng = _rng(12)
    B, T, N, H, D, F = 2, 7, 4, 2, 5, 3  # last block is partial
    q = rng.standard_normal((B, T, N, H, D))
    k = rng.standard_normal((B, T, N, H, D))
    v = rng.standard_normal((B, T, N, H, D))
    out, st, z = impl.la_block_causal(q, k, v, None, None, F)
    _close(out, _la_brute_force(q, k, v, F, 1e-6), 1e-11, "LA brute force")
    # the final state and normaliser are plain sums over every token
    for b in range(B):
        for h in range(H):
            phik = np.maximum(k[b, :, :, h].reshape(-1, D), 0.0)
            _close(st[b, h], phik.T @ v[b, :, :, h].reshape(-1, D), 1e-12, "LA S_T")
            _close(z[b, h], phik.sum(0), 1e-12, "LA z_T")


def pin_la_resume(impl):
    """LA over T frames = LA over the first whole blocks, then the rest from the carried (S, z)."""
    rng = _rng(13)
    B, T, N, H, D, F = 1, 8, 3, 2, 4, 2
    q = rng.standard_normal((B, T, N, H, D))
    k = rng.standard_normal((B, T, N, H, D))
    v = rng.standard_normal((B, T, N, H, D))
    out, st, z = impl.la_block_causal(q, k, v, None, None, F)
    o1, s1, z1 = impl.la_block_causal(q[:, :4], k[:, :4], v[:, :4], None, None, F)
    o2, s2, z2 = impl.la_block_causal(q[:, 4:], k[:, 4:], v[:, 4:], s1, z1, F)
    _close(np.concatenate([o1, o2], axis=1), out, 1e-12, "LA resume O")
    _close(s2, st, 1e-12, "LA resume S")
    _close(z2, z, 1e-12, "LA resume z")


def pin_e4m3_landmarks(impl):
    """E4M3 codes whose values the format's definition fixes (sign, 4-bit exponent with bias 7,
    3-bit mantissa, exponent 0 for subnormals, S.1111.111 for NaN, no infinities)."""
    table = {
        0x00: 0.0, 0x80: -0.0,
        0x01: 2.0 ** -9,             # smallest subnormal: 1/8 * 2^-6
        0x07: 7.0 * 2.0 ** -9,       # largest subnormal
        0x08: 2.0 ** -6,             # smallest normal
        0x30: 0.5, 0x38: 1.0, 0x39: 1.125, 0x3F: 1.875, 0x40: 2.0, 0xB8: -1.0,
        0x77: 240.0,                 # 1.875 * 2^7
        0x7E: 448.0, 0xFE: -448.0,   # largest finite magnitude
    }
    codes = np.array(sorted(table), dtype=np.uint8)
    got = impl.e4m3_decode(codes)
    want = np.array([table[int(c)] for c in codes])
    assert np.array_equal(got, want), (got, want)
    assert np.all(np.isnan(impl.e4m3_decode(np.array([0x7F, 0xFF], dtype=np.uint8))))


def pin_e4m3_ordering(impl):
    """Positive codes 0x00..0x7E decode to strictly increasing values, each negative code is the
    negated positive one, and inside one exponent the spacing is 2^(e-10) (2^-9 subnormal)."""
    pos = impl.e4m3_decode(np.arange(0x7F, dtype=np.uint8))
    assert np.all(np.diff(pos) > 0)
    neg = impl.e4m3_decode(np.arange(0x80, 0xFF, dtype=np.uint8))
    assert np.array_equal(neg, -pos)
    for e in range(1, 16):
        lo = e << 3
        hi = min(lo + 7, 0x7E)
        d = np.diff(impl.e4m3_decode(np.arange(lo, hi + 1, dtype=np.uint8)))
        assert np.all(d == 2.0 ** (e - 10)), (e, d)
    assert np.all(np.diff(pos[:8]) == 2.0 ** -9)


def pin_fp8_scales(impl):
    """Per-frame scales of the fp8 forward: q's scale scales O; k's scale trades against the key
    scale; v's scale together with S_0 scales (O, S_T) (linearity in (V, S_0)); with unit scales
    it is the forward on the decoded values."""
    rng = _rng(21)
    B, T, N, H, D = 1, 3, 5, 2, 4
    codes = [rng.integers(0, 0x7F, size=(B, T, N, H, D)).astype(np.uint8)
             | (rng.integers(0, 2, size=(B, T, N, H, D)).astype(np.uint8) << 7) for _ in range(3)]
    sq, sk, sv = (rng.uniform(0.001, 0.01, size=(B, T, H)) for _ in range(3))
    g = rng.uniform(0.9, 0.999, size=(B, T, H))
    be = rng.uniform(0.1, 0.9, size=(B, T, H))
    S0 = rng.standard_normal((B, H, D, D))
    ks = 0.3
    o, s = impl.gdn_frame_forward_fp8(*codes, sq, sk, sv, g, be, S0, ks)
    o2, s2 = impl.gdn_frame_forward_fp8(*codes, 3.0 * sq, sk, sv, g, be, S0, ks)
    _close(o2, 3.0 * o, 1e-11, "q scale")
    _close(s2, s, 1e-12, "q scale leaves the state")
    o3, s3 = impl.gdn_frame_forward_fp8(*codes, sq, 4.0 * sk, sv, g, be, S0, ks / 4.0)
    _close(o3, o, 1e-11, "k scale vs key scale")
    _close(s3, s, 1e-11, "k scale vs key scale (state)")
    o4, s4 = impl.gdn_frame_forward_fp8(*codes, sq, sk, 2.0 * sv, g, be, 2.0 * S0, ks)
    _close(o4, 2.0 * o, 1e-11, "v scale with S_0")
    _close(s4, 2.0 * s, 1e-11, "v scale with S_0 (state)")
    one = np.ones((B, T, H))
    dec = [impl.e4m3_decode(c) for c in codes]
    o5, s5 = impl.gdn_frame_forward_fp8(*codes, one, one, one, g, be, S0, ks)
    o6, s6 = impl.gdn_frame_forward(*dec, g, be, S0, ks)
    _close(o5, o6, 1e-12, "unit scales")
    _close(s5, s6, 1e-12, "unit scales (state)")


# --------------------------------------------------------------------------- backward pins

def _bwd_case(rng, B=2, T=3, N=3, H=2, D=3):
    q, k, v, gamma, beta = _rand_clip(B, T, N, H, D, rng, g=(0.5, 1.0), b=(0.1, 0.9))
    S0 = rng.standard_normal((B, H, D, D))
    dO = rng.standard_normal((B, T, N, H, D))
    dS = rng.standard_normal((B, H, D, D))
    return q, k, v, gamma, beta, S0, dO, dS


def pin_bwd_hand_example(impl):
    """Exact rationals worked by hand (tests/golden/gdn_backward_hand_example.json): a scalar
    head (D = N = 1) over two frames, every gradient from the derivative of the definition."""
    from fractions import Fraction
    with open(os.path.join(GOLDEN, "gdn_backward_hand_example.json")) as f:
        g = json.load(f)
    tok = lambda x: np.array(x, dtype=np.float64).reshape(1, 2, 1, 1, 1)  # [1,T,N,H,D]
    fr = lambda xs: np.array([float(Fraction(x)) for x in xs])
    dq, dk, dv, dgam, dbet, ds0 = impl.gdn_frame_backward(
        tok(g["q"]), tok(g["k"]), tok(g["v"]), np.array(g["gamma"]).reshape(1, 2, 1),
        np.array(g["beta"]).reshape(1, 2, 1), np.full((1, 1, 1, 1), g["state_in"]),
        tok(g["d_out"]), np.full((1, 1, 1, 1), g["d_state_out"]), g["key_scale"])
    _close(dq.ravel(), fr(g["expected_dq"]), 1e-14, "hand example dq")
    _close(dk.ravel(), fr(g["expected_dk"]), 1e-14, "hand example dk")
    _close(dv.ravel(), fr(g["expected_dv"]), 1e-14, "hand example dv")
    _close(dgam.ravel(), fr(g["expected_dgamma"]), 1e-14, "hand example dgamma")
    _close(dbet.ravel(), fr(g["expected_dbeta"]), 1e-14, "hand example dbeta")
    _close(ds0.ravel(), fr([g["expected_dstate_in"]]), 1e-14, "hand example dS_0")


def pin_bwd_finite_differences(impl):
    """Every gradient against central differences of the (pinned) forward, for the scalar
    L = <dO, O> + <dS_T, S_T>. The forward is a polynomial in every input, so central
    differences with step 1e-5 are exact to about 1e-9 here."""
    rng = _rng(101)
    q, k, v, gamma, beta, S0, dO, dS = _bwd_case(rng)
    D, N = q.shape[-1], q.shape[2]
    ks = 1.0 / np.sqrt(D * N)
    params = {"q": q, "k": k, "v": v, "gamma": gamma, "beta": beta, "S0": S0}

    def loss(p):
        o, st = impl.gdn_frame_forward(p["q"], p["k"], p["v"], p["gamma"], p["beta"], p["S0"], ks)
        return float(np.sum(dO * o) + np.sum(dS * st))

    grads = impl.gdn_frame_backward(q, k, v, gamma, beta, S0, dO, dS, ks)
    names = ["q", "k", "v", "gamma", "beta", "S0"]
    h = 1e-5
    for name, g in zip(names, grads):
        fd = np.zeros(params[name].shape)
        for idx in np.ndindex(*params[name].shape):
            p_plus = {n: a.copy() for n, a in params.items()}
            p_minus = {n: a.copy() for n, a in params.items()}
            p_plus[name][idx] += h
            p_minus[name][idx] -= h
            fd[idx] = (loss(p_plus) - loss(p_minus)) / (2 * h)
        _close(g, fd, 1e-7, f"d{name} vs central differences")


def pin_bwd_adjoint_identity(impl):
    """The forward is linear in (V, S_0) jointly with q, k, gamma, beta fixed (no constant
    term). So for any direction (dV, dS0) the dot-product test must hold:
    <grad_V, dV> + <grad_S0, dS0> = <dO, O(dV, dS0)> + <dS_T, S_T(dV, dS0)>.
    This is exact up to rounding, at a size (T = 6, D = 5) where differences would be slow."""
    rng = _rng(102)
    q, k, v, gamma, beta, S0, dO, dS = _bwd_case(rng, B=1, T=6, N=4, H=2, D=5)
    ks = 1.0 / np.sqrt(5 * 4)
    grads = impl.gdn_frame_backward(q, k, v, gamma, beta, S0, dO, dS, ks)
    dV = rng.standard_normal(v.shape)
    dS0 = rng.standard_normal(S0.shape)
    o, st = impl.gdn_frame_forward(q, k, dV, gamma, beta, dS0, ks)
    lhs = float(np.sum(grads[2] * dV) + np.sum(grads[5] * dS0))
    rhs = float(np.sum(dO * o) + np.sum(dS * st))
    assert abs(lhs - rhs) <= 1e-10 * max(1.0, abs(rhs)), f"adjoint identity: {lhs} vs {rhs}"


def pin_bwd_single_frame_closed_form(impl):
    """One frame from S_0 = 0: S_1 = beta V^T K', so O = beta Q K'^T V (plain unnormalised
    linear attention over the frame, K' = s K). With L = <dO, O> (no state cotangent) the
    textbook gradients are dQ = beta dO V^T K', dV = beta K' Q^T dO, dK = s beta V dO^T Q,
    dbeta = <dO, Q K'^T V>, dgamma = 0 (the gate multiplies the zero state), and
    dS_0 = gamma (dO^T Q)(I - beta A)."""
    rng = _rng(103)
    N, D = 5, 4
    q, k, v, gamma, beta = _rand_clip(1, 1, N, 1, D, rng)
    dO = rng.standard_normal(q.shape)
    s = 0.37
    Q, K, V, g = q[0, 0, :, 0], k[0, 0, :, 0], v[0, 0, :, 0], dO[0, 0, :, 0]
    be, ga = beta[0, 0, 0], gamma[0, 0, 0]
    Ks = s * K
    dq, dk, dv, dgamma, dbeta, dS0 = impl.gdn_frame_backward(q, k, v, gamma, beta, None, dO,
                                                            None, s)
    _close(dq[0, 0, :, 0], be * g @ V.T @ Ks, 1e-12, "dQ")
    _close(dv[0, 0, :, 0], be * Ks @ Q.T @ g, 1e-12, "dV")
    _close(dk[0, 0, :, 0], s * be * V @ g.T @ Q, 1e-12, "dK")
    _close(dbeta[0, 0, 0], np.sum(g * (Q @ Ks.T @ V)), 1e-12, "dbeta")
    _close(dgamma[0, 0, 0], 0.0, 1e-12, "dgamma")
    _close(dS0[0, 0], ga * (g.T @ Q) @ (np.eye(D) - be * Ks.T @ Ks), 1e-12, "dS0")


def pin_bwd_cotangent_linearity(impl):
    """The backward is linear in the cotangents (dO, dS_T): zero cotangents give zero
    gradients, and a combination of cotangents gives the same combination of gradients."""
    rng = _rng(104)
    q, k, v, gamma, beta, S0, dO, dS = _bwd_case(rng, B=1, T=4, N=3, H=1, D=4)
    dO2 = rng.standard_normal(dO.shape)
    dS2 = rng.standard_normal(dS.shape)
    ks = 0.25
    zero = impl.gdn_frame_backward(q, k, v, gamma, beta, S0, np.zeros_like(dO), None, ks)
    for z in zero:
        _close(z, np.zeros_like(z), 0.0, "zero cotangents")
    g1 = impl.gdn_frame_backward(q, k, v, gamma, beta, S0, dO, dS, ks)
    g2 = impl.gdn_frame_backward(q, k, v, gamma, beta, S0, dO2, dS2, ks)
    g3 = impl.gdn_frame_backward(q, k, v, gamma, beta, S0, 2 * dO - 3 * dO2, 2 * dS - 3 * dS2, ks)
    for a, b, c in zip(g1, g2, g3):
        _close(c, 2 * a - 3 * b, 1e-12, "cotangent linearity")


GDN_PINS = [
    pin_hand_example,
    pin_single_frame_closed_form,
    pin_pure_decay,
    pin_tokenwise_reduction,
    pin_delta_rule_exactness,
    pin_fixed_point,
    pin_split_resume,
    pin_linearity,
    pin_causal_across_bidirectional_within,
    pin_unrolled_product_form,
    pin_stats_identity_keys,
    pin_step_is_single_frame,
]
LA_PINS = [pin_la_hand_example, pin_la_brute_force, pin_la_resume]
FP8_PINS = [pin_e4m3_landmarks, pin_e4m3_ordering, pin_fp8_scales]
BWD_PINS = [
    pin_bwd_hand_example,
    pin_bwd_finite_differences,
    pin_bwd_adjoint_identity,
    pin_bwd_single_frame_closed_form,
    pin_bwd_cotangent_linearity,
]
ALL_PINS = GDN_PINS + LA_PINS + FP8_PINS + BWD_PINS
