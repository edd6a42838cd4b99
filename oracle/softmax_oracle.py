"""fp64 CPU oracle for the softmax attention of the hybrid DiT's softmax blocks.

TEST INFRASTRUCTURE. Only the tests may import this module; no CUDA code shares anything with
it. It is the plain definition in float64 numpy, one (batch, head) and one chunk of frames at a
time, with matrix products through numpy's ``@``.

What it computes (plain reading of the sources):

* The ai-papers.net article on SANA-WM, section "ハイブリッドアテンション機構", and the gen-hub.ru
  article, section "Архитектура: четыре нетривиальных решения", both place softmax attention in
  5 of the 20 blocks (3, 7, 11, 15, 19), with frame-wise GDN in the other 15.
* The gen-hub.ru article, section "Три режима на любой вкус", lists the inference modes: a
  bidirectional generator and chunk-causal autoregressive ones.

Reading adopted, per head, over the clip's T*N tokens:

    O = softmax(Q K^T * scale + M) V,   scale = 1/sqrt(D) by default

The mask M is 0 where a key is visible and -inf elsewhere. With chunks of F frames, a token of
frame t sees every token of the frames whose chunk t' // F is at most t // F. That is bidirectional
inside a chunk and causal across chunks; F >= T is the fully bidirectional mode. q and k arrive
with any positional encoding already applied. The row-wise softmax subtracts the row maximum
before exponentiating (the same value in exact arithmetic).

Parity status: pinned by ``tests/test_softmax_oracle.py``. The pins are a hand-worked example,
brute force per query on tiny inputs, the mask's invariants and the softmax's invariants, and
planted mistakes each fail a pin.
"""
from __future__ import annotations

import numpy as np

__all__ = ["softmax_attention_chunk_causal"]


def softmax_attention_chunk_causal(q, k, v, frames_per_chunk: int, scale: float | None = None):
    """Chunk-causal (block-causal) softmax attention.

    q, k, v: [B, T, N, H, D]. frames_per_chunk: F >= 1 (F >= T: bidirectional over the clip).
    scale: multiplies Q K^T (default 1/sqrt(D)). Returns out [B, T, N, H, D] float64.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    Bsz, T, N, H, D = q.shape
    F = int(frames_per_chunk)
    if F < 1:
        raise ValueError("frames_per_chunk must be >= 1")
    s = 1.0 / np.sqrt(D) if scale is None else float(scale)
    out = np.zeros((Bsz, T, N, H, D))
    for b in range(Bsz):
        for h in range(H):
            for t0 in range(0, T, F):
                t1 = min(t0 + F, T)
                # queries of this chunk; keys and values of every frame up to the chunk's end
                Q = q[b, t0:t1, :, h, :].reshape(-1, D)
                K = k[b, :t1, :, h, :].reshape(-1, D)
                V = v[b, :t1, :, h, :].reshape(-1, D)
                scores = (Q @ K.T) * s
                scores = scores - scores.max(axis=1, keepdims=True)
                w = np.exp(scores)
                w = w / w.sum(axis=1, keepdims=True)
                out[b, t0:t1, :, h, :] = (w @ V).reshape(t1 - t0, N, D)
    return out
