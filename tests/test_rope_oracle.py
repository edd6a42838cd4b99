"""Pins of the 3D RoPE oracle (``oracle/rope_oracle.py``), CPU only.

The pins are:
* a hand-worked example: one token, D = 12, pairs (1, 0) and (0, 1) per axis slice;
* norm preservation;
* the identity at position zero;
* q.k products invariant to a common shift of positions along each axis, which is the property
  rotary embeddings exist for;
* the slice boundaries: each slice sees only its own axis's position;
* a resumed clip: frames [a, T) embedded with t_offset = a equal the whole clip's.

Planted mistakes in copies of the oracle each fail at least one pin.
"""
import math

import numpy as np
import pytest

import oracle.rope_oracle as ro


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def pin_hand_example(rope, split):
    """D = 12 splits 4 / 4 / 4. The token at frame 1, grid 2 x 3, n = 5 sits at row 1, col 2.
    Pair i of a slice rotates by pos * 10000^(-2i/4): frequencies 1 and 0.01, so the angles are
    (1, 0.01) for time and rows and (2, 0.02) for columns. A pair (1, 0) becomes (cos a, sin a)
    and a pair (0, 1) becomes (-sin a, cos a)."""
    assert tuple(split(12)) == (4, 4, 4)
    x = np.zeros((1, 2, 6, 1, 12))
    x[0, 1, 5, 0] = [1, 0, 0, 1] * 3
    got = rope(x, 2, 3)[0, 1, 5, 0]
    want = []
    for a0, a1 in ((1.0, 0.01), (1.0, 0.01), (2.0, 0.02)):
        want += [math.cos(a0), math.sin(a0), -math.sin(a1), math.cos(a1)]
    assert np.allclose(got, want, atol=1e-15), (got, want)


def pin_split(rope, split):
    """The time slice takes the remainder; rows and columns get 2 * floor(D / 6) dims each."""
    assert tuple(split(128)) == (44, 42, 42)
    assert tuple(split(64)) == (24, 20, 20)
    assert tuple(split(8)) == (4, 2, 2)


def pin_norm_preserved(rope, split):
    x = _rand((2, 3, 6, 2, 16), 1)
    y = rope(x, 2, 3, 500.0, 7)
    assert np.allclose(np.linalg.norm(y, axis=-1), np.linalg.norm(x, axis=-1), rtol=1e-13)
    # every pair separately (rotations act on pairs)
    assert np.allclose(y[..., 0::2] ** 2 + y[..., 1::2] ** 2, x[..., 0::2] ** 2 + x[..., 1::2] ** 2,
                       rtol=1e-12)


def pin_identity_at_origin(rope, split):
    x = _rand((1, 1, 4, 3, 24), 2)
    y = rope(x, 2, 2)
    assert np.array_equal(y[0, 0, 0], x[0, 0, 0])


def pin_shift_invariance(rope, split):
    """<R(p) q, R(p') k> depends on p - p' only: shifting both tokens by a frame (t_offset),
    by a row (n + grid_w) or by a column (n + 1, same row) leaves the product unchanged, while
    moving one token alone changes it."""
    gh, gw, D = 3, 4, 24
    q = _rand((1, 3, gh * gw, 1, D), 3)
    k = _rand((1, 3, gh * gw, 1, D), 4)
    dot = lambda a, b: float(np.dot(a, b))
    rq, rk = rope(q, gh, gw, 100.0, 0), rope(k, gh, gw, 100.0, 0)
    sq, sk = rope(q, gh, gw, 100.0, 5), rope(k, gh, gw, 100.0, 5)
    base = dot(rq[0, 0, 1, 0], rk[0, 2, 6, 0])
    assert abs(base - dot(sq[0, 0, 1, 0], sk[0, 2, 6, 0])) < 1e-12            # time shift
    # the same vectors placed one row lower / one column right
    q2, k2 = q.copy(), k.copy()
    q2[0, 0, 1 + gw, 0], k2[0, 2, 6 + gw, 0] = q[0, 0, 1, 0], k[0, 2, 6, 0]
    r2q, r2k = rope(q2, gh, gw, 100.0, 0), rope(k2, gh, gw, 100.0, 0)
    assert abs(base - dot(r2q[0, 0, 1 + gw, 0], r2k[0, 2, 6 + gw, 0])) < 1e-12
    q3, k3 = q.copy(), k.copy()
    q3[0, 0, 2, 0], k3[0, 2, 7, 0] = q[0, 0, 1, 0], k[0, 2, 6, 0]
    r3q, r3k = rope(q3, gh, gw, 100.0, 0), rope(k3, gh, gw, 100.0, 0)
    assert abs(base - dot(r3q[0, 0, 2, 0], r3k[0, 2, 7, 0])) < 1e-12
    assert abs(base - dot(rq[0, 1, 1, 0], rk[0, 2, 6, 0])) > 1e-6             # one token moved


def pin_slices_see_their_axis(rope, split):
    """A vector living in one slice is rotated by that axis's position only."""
    gh, gw, D = 2, 3, 18
    d_t, d_h, d_w = split(D)
    x = np.zeros((1, 3, gh * gw, 1, D))
    v = _rand((D,), 5)
    x[...] = v
    y = rope(x, gh, gw)
    t_sl = slice(0, d_t)
    h_sl = slice(d_t, d_t + d_h)
    w_sl = slice(d_t + d_h, D)
    # time slice: the same for every token of a frame
    assert np.allclose(y[0, 2, :, 0, t_sl], y[0, 2, 0, 0, t_sl], atol=1e-14)
    # row slice: the same for every frame and every column of a row
    assert np.allclose(y[0, :, 3:6, 0, h_sl], y[0, 0, 3, 0, h_sl], atol=1e-14)
    # column slice: the same for every frame and every row of a column
    assert np.allclose(y[0, :, [1, 4], 0, w_sl], y[0, 0, 1, 0, w_sl], atol=1e-14)
    assert not np.allclose(y[0, 0, 3, 0, h_sl], y[0, 0, 0, 0, h_sl])
    assert not np.allclose(y[0, 0, 1, 0, w_sl], y[0, 0, 0, 0, w_sl])


def pin_resume_offset(rope, split):
    """t_offset is the absolute frame index: the frames [a, T) of a clip, embedded with
    t_offset = a, equal the same frames of the whole clip."""
    x = _rand((1, 6, 4, 2, 16), 6)
    whole = rope(x, 2, 2, 1000.0, 0)
    for a in (1, 4):
        assert np.allclose(rope(x[:, a:], 2, 2, 1000.0, a), whole[:, a:], atol=1e-14)


PINS = [pin_hand_example, pin_split, pin_norm_preserved, pin_identity_at_origin,
        pin_shift_invariance, pin_slices_see_their_axis, pin_resume_offset]


@pytest.mark.parametrize("pin", PINS, ids=lambda p: p.__name__)
def test_rope_oracle_pin(pin):
    pin(ro.rope_3d, ro.rope_3d_split)


def _variant(mistake):
    """The oracle with one planted mistake. Returns (rope, split)."""
    def split(D):
        if mistake == "remainder_to_columns":
            d = 2 * (D // 6)
            return d, d, D - 2 * d
        return ro.rope_3d_split(D)

    def rotate(x, pos, d_a, base):
        i = np.arange(d_a // 2, dtype=np.float64)
        expo = -i / d_a if mistake == "theta_exponent_halved" else -2.0 * i / d_a
        ang = np.asarray(pos, float)[..., None] * base ** expo
        c, s = np.cos(ang), np.sin(ang)
        if mistake == "rotate_half_pairs":
            h = d_a // 2
            xe, xo = x[..., :h], x[..., h:]
            out = np.empty_like(x)
            out[..., :h] = xe * c - xo * s
            out[..., h:] = xe * s + xo * c
            return out
        xe, xo = x[..., 0::2], x[..., 1::2]
        sgn = -1.0 if mistake == "rotation_sign" else 1.0
        out = np.empty_like(x)
        out[..., 0::2] = xe * c - sgn * xo * s
        out[..., 1::2] = sgn * xe * s + xo * c
        return out

    def rope(x, grid_h, grid_w, base=10000.0, t_offset=0):
        x = np.asarray(x, float)
        B, T, N, H, D = x.shape
        d_t, d_h, d_w = split(D)
        t = np.arange(T, dtype=float) + (0 if mistake == "t_offset_ignored" else t_offset)
        n = np.arange(N)
        row, col = (n // grid_w).astype(float), (n % grid_w).astype(float)
        if mistake == "rows_and_columns_swapped":
            row, col = col, row
        shp = (B, T, N, H)
        pt = np.broadcast_to(t[None, :, None, None], shp)
        ph = np.broadcast_to(row[None, None, :, None], shp)
        pw = np.broadcast_to(col[None, None, :, None], shp)
        out = np.empty_like(x)
        out[..., :d_t] = rotate(x[..., :d_t], pt, d_t, base)
        out[..., d_t:d_t + d_h] = rotate(x[..., d_t:d_t + d_h], ph, d_h, base)
        out[..., d_t + d_h:] = rotate(x[..., d_t + d_h:], pw, d_w, base)
        return out

    return rope, split


MISTAKES = ["remainder_to_columns", "theta_exponent_halved", "rotate_half_pairs",
            "rotation_sign", "t_offset_ignored", "rows_and_columns_swapped"]


@pytest.mark.parametrize("mistake", MISTAKES)
def test_rope_mutant_is_caught(mistake):
    rope, split = _variant(mistake)
    failed = []
    for pin in PINS:
        try:
            pin(rope, split)
        except (AssertionError, ValueError):
            failed.append(pin.__name__)
    assert failed, f"mutant {mistake} passes every pin"


def test_unmutated_variant_passes():
    rope, split = _variant("none")
    for pin in PINS:
        pin(rope, split)
