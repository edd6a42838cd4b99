"""A numpy model of exactly the softmax attention kernel's decomposition (CPU): 128-query tiles,
128-key tiles up to the key limit of the tile's last query, the per-row key limit of the chunk
mask, base-2 scores, a running maximum raised only when a row's maximum grows by more than 8,
P rounded to bf16 for the second product and O / l at the end. In float64 without the bf16
rounding it equals the oracle to 1e-12; with it, the error is the size the GPU tests allow for.
"""
import math

import numpy as np
import pytest
import torch

import gdn_inputs
import oracle

TILE = 128


def bf16(x):
    return torch.tensor(x, dtype=torch.float32).to(torch.bfloat16).to(torch.float64).numpy()


def key_limit(r, N, T, F):
    t = r // N
    return min(T, (t // F + 1) * F) * N


def tiled_attention(q, k, v, N, T, F, scale, round_p, stats=None):
    """q, k, v: [L, D] float64 of one (batch, head) over the clip's L = T * N tokens."""
    L, D = q.shape
    c = scale / math.log(2.0)  # scores in base-2 units: S * scale * log2(e)
    out = np.zeros((L, D))
    for q0 in range(0, L, TILE):
        rows = np.arange(q0, min(q0 + TILE, L))
        kmax = np.array([key_limit(r, N, T, F) for r in rows])
        n_kt = -(-kmax.max() // TILE)
        m = np.full(len(rows), -np.inf)
        l = np.zeros(len(rows))
        o = np.zeros((len(rows), D))
        for j in range(n_kt):
            k0 = j * TILE
            keys = np.arange(k0, min(k0 + TILE, L))
            s = (q[rows] @ k[keys].T) * c
            vis = keys[None, :] < kmax[:, None]
            s = np.where(vis, s, -np.inf)
            m_new = np.maximum(m, s.max(axis=1))
            raise_ = m_new > m + 8.0
            alpha = np.where(raise_, np.exp2(m - m_new), 1.0)
            m = np.where(raise_, m_new, m)
            o *= alpha[:, None]
            l *= alpha
            p = np.exp2(s - m[:, None])
            if stats is not None:
                stats["max_weight"] = max(stats.get("max_weight", 0.0), float(p.max()))
                stats["raises"] = stats.get("raises", 0) + int(raise_.sum()) * (j > 0)
            l += p.sum(axis=1)
            o += (bf16(p) if round_p else p) @ v[keys]
        out[rows] = o / l[:, None]
    return out


@pytest.mark.parametrize("case", [(5, 70, 32, 2), (4, 100, 64, 1), (3, 129, 16, 3), (9, 40, 32, 4)],
                         ids=lambda c: "T%dN%dD%dF%d" % c)
def test_tiled_online_softmax_equals_the_oracle(case):
    T, N, D, F = case
    x = gdn_inputs.clip_inputs(1, 1, T, N, D, seed=1600 + T + N)
    f = lambda t: t.float().numpy().astype(np.float64)
    q, k, v = (f(x[n])[0, :, :, 0, :].reshape(T * N, D) for n in ("q", "k", "v"))
    ref = oracle.softmax_attention_chunk_causal(f(x["q"]), f(x["k"]), f(x["v"]), F)
    ref = ref[0, :, :, 0, :].reshape(T * N, D)
    exact = tiled_attention(q, k, v, N, T, F, 1.0 / math.sqrt(D), round_p=False)
    assert np.max(np.abs(exact - ref)) <= 1e-12 * np.max(np.abs(ref))
    # the kernel's bf16 weights: well inside the GPU tests' bars
    rounded = tiled_attention(q, k, v, N, T, F, 1.0 / math.sqrt(D), round_p=True)
    e = np.linalg.norm(rounded - ref) / np.linalg.norm(ref)
    assert e <= 4e-3, e


def test_lazy_rescaling_keeps_weights_bounded_and_result_exact():
    """A sharp softmax (large scale) forces rescaling in later tiles; the stale maximum keeps
    every weight at most 2^8, and the result is still exact."""
    T, N, D, F = 6, 64, 32, 6
    x = gdn_inputs.clip_inputs(1, 1, T, N, D, seed=1700)
    f = lambda t: t.float().numpy().astype(np.float64)
    q, k, v = (f(x[n])[0, :, :, 0, :].reshape(T * N, D) for n in ("q", "k", "v"))
    ref = oracle.softmax_attention_chunk_causal(f(x["q"]), f(x["k"]), f(x["v"]), F, 2.0)
    ref = ref[0, :, :, 0, :].reshape(T * N, D)
    stats = {}
    got = tiled_attention(q, k, v, N, T, F, 2.0, round_p=False, stats=stats)
    assert np.max(np.abs(got - ref)) <= 1e-12 * np.max(np.abs(ref))
    assert stats["raises"] > 0 and stats["max_weight"] <= 2.0 ** 8
