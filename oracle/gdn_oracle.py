"""fp64 CPU oracle for the frame-wise Gated DeltaNet (GDN) frame scan.

TEST INFRASTRUCTURE. Only the tests, the smoke check in ``__graft_entry__``
and the CPU-baseline leg of ``bench.py`` may import this module. The CUDA
library never calls it and shares no code with it: this is a plain, slow,
obviously correct restatement of what the layer computes, in float64 numpy,
one (batch, head) at a time and one frame at a time. Matrix products go
through numpy's ``@`` (a library primitive); there is no blocking, fusion or
reordering beyond the definition.

What the layer computes (plain reading of the sources):

* "NVIDIA SANA-WM: минутное 720p видео с одной видеокарты" (gen-hub.ru),
  section "Архитектура: четыре нетривиальных решения": Gated DeltaNet adds a
  decay gate gamma that down-weights stale frames and a delta-rule correction
  that updates only the residual between the target value and the current
  prediction; the recurrent state is a constant D x D matrix whatever the video
  length; keys are scaled by 1/sqrt(D*S) (D head dim, S spatial tokens per
  frame), replacing L2 key normalisation.
* "SANA-WM: Efficient Minute-Scale World Modeling with Hybrid Linear Diffusion
  Transformer" (chatpaper.ai abstract), design (1): the GDN is *frame-wise*;
  the ai-papers.net article on SANA-WM, section "ハイブリッドアテンション機構":
  the state is updated recurrently once per frame.

Reading adopted for one head (the token-wise gated delta rule
``S <- gamma*S + beta*(v - gamma*S k) k^T`` applied once per frame, every token
of the frame predicting from the same previous state and the residuals summed):

    k' = s * k,  s = key_scale
    A_t = K'_t^T K'_t                 (D x D)
    B_t = V_t^T K'_t                  (D_v x D_k)
    S_t = gamma_t * S_{t-1} (I - beta_t A_t) + beta_t B_t
    O_t = Q_t S_t^T                   (every token of frame t reads S_t)

so attention is bidirectional inside a frame and causal across frames. The
state is stored D_v x D_k, i.e. ``S @ k`` is a value.

Block-causal linear attention (the predecessor, "SANA-Video: Efficient Video
Generation with Block Linear Diffusion Transformer", ICLR 2026 oral talk
transcript, block KV cache passage): the D x D state of block i is the cached
state of block i-1 plus block i's own K^T V contribution. The ReLU feature map
and the normaliser z follow the workload definition:
``S += relu(K)^T V``, ``z += sum relu(k)``,
``O = relu(Q) S / (relu(Q) z + 1e-6)``; here S is D_k x D_v.
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "e4m3_decode",
    "frame_statistics",
    "frame_update",
    "frame_output",
    "frame_update_backward",
    "gdn_frame_backward",
    "gdn_frame_forward",
    "gdn_frame_forward_fp8",
    "gdn_frame_step",
    "la_block_causal",
]


def _f64(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float64)


def frame_statistics(K: np.ndarray, V: np.ndarray, key_scale: float):
    """A_t and B_t of one frame of one head.

    K, V: (N, D) arrays (any float type; converted exactly to float64).
    Returns A = (sK)^T (sK) (D x D) and B = V^T (sK) (D_v x D_k).
    Sources: gen-hub.ru SANA-WM article, "Архитектура" (key scale 1/sqrt(D*S));
    frame-wise reading of the delta rule (module docstring).
    """
    Ks = key_scale * _f64(K)
    A = Ks.T @ Ks
    B = _f64(V).T @ Ks
    return A, B


def frame_update(S: np.ndarray, A: np.ndarray, B: np.ndarray, gamma: float, beta: float):
    """S_t = gamma * S_{t-1} (I - beta A_t) + beta B_t (gen-hub.ru, "Архитектура":
    decay gate gamma, delta-rule residual correction beta)."""
    D = A.shape[0]
    return gamma * (S @ (np.eye(D) - beta * A)) + beta * B


def frame_output(Q: np.ndarray, S: np.ndarray) -> np.ndarray:
    """O_t = Q_t S_t^T: every token of the frame reads the post-update state."""
    return _f64(Q) @ S.T


def gdn_frame_forward(q, k, v, gamma, beta, state_in, key_scale: float):
    """Frame-wise GDN over a whole clip.

    q, k, v: [B, T, N, H, D]; gamma, beta: [B, T, H]; state_in: [B, H, D, D] or
    None (S_0 = 0). Returns (out [B,T,N,H,D] float64, state_out [B,H,D,D] float64).
    """
    q = np.asarray(q)
    k = np.asarray(k)
    v = np.asarray(v)
    gamma = _f64(gamma)
    beta = _f64(beta)
    Bsz, T, N, H, D = q.shape
    out = np.zeros((Bsz, T, N, H, D), dtype=np.float64)
    state_out = np.zeros((Bsz, H, D, D), dtype=np.float64)
    for b in range(Bsz):
        for h in range(H):
            S = np.zeros((D, D)) if state_in is None else _f64(state_in[b, h]).copy()
            for t in range(T):
                A, Bm = frame_statistics(k[b, t, :, h, :], v[b, t, :, h, :], key_scale)
                S = frame_update(S, A, Bm, gamma[b, t, h], beta[b, t, h])
                out[b, t, :, h, :] = frame_output(q[b, t, :, h, :], S)
            state_out[b, h] = S
    return out, state_out


def gdn_frame_step(q, k, v, gamma, beta, state_in, key_scale: float):
    """One streaming step: a single new frame per stream.

    q, k, v: [B, N, H, D]; gamma, beta: [B, H]; state_in: [B, H, D, D] or None.
    Same arithmetic as ``gdn_frame_forward`` with T = 1 (the chunk-causal /
    distilled autoregressive modes of the gen-hub.ru SANA-WM article, section
    "Три режима на любой вкус", advance the state one frame at a time).
    """
    q = np.asarray(q)[:, None]
    k = np.asarray(k)[:, None]
    v = np.asarray(v)[:, None]
    g = _f64(gamma)[:, None]
    bt = _f64(beta)[:, None]
    out, st = gdn_frame_forward(q, k, v, g, bt, state_in, key_scale)
    return out[:, 0], st


def la_block_causal(q, k, v, state_in, z_in, frames_per_block: int, eps: float = 1e-6):
    """Block-causal linear attention with a ReLU feature map and a normaliser.

    q, k, v: [B, T, N, H, D]; state_in: [B, H, D_k, D_v] or None; z_in: [B, H, D_k]
    or None. Blocks are ``frames_per_block`` consecutive frames (the last block
    may be shorter). For block j:  S += relu(K_j)^T V_j,  z += sum_i relu(k_i),
    then every token of block j reads the updated (S, z):
    O = relu(q) S / (relu(q) . z + eps).
    Source: "SANA-Video ... Block Linear Diffusion Transformer" talk transcript,
    block KV cache passage (additive state, cached between blocks).
    Returns (out float64, state_out [B,H,D,D], z_out [B,H,D]).
    """
    q = np.asarray(q)
    k = np.asarray(k)
    v = np.asarray(v)
    Bsz, T, N, H, D = q.shape
    F = int(frames_per_block)
    out = np.zeros((Bsz, T, N, H, D), dtype=np.float64)
    s_out = np.zeros((Bsz, H, D, D))
    z_out = np.zeros((Bsz, H, D))
    for b in range(Bsz):
        for h in range(H):
            S = np.zeros((D, D)) if state_in is None else _f64(state_in[b, h]).copy()
            z = np.zeros(D) if z_in is None else _f64(z_in[b, h]).copy()
            for t0 in range(0, T, F):
                frames = range(t0, min(t0 + F, T))
                for t in frames:
                    phiK = np.maximum(_f64(k[b, t, :, h, :]), 0.0)
                    S = S + phiK.T @ _f64(v[b, t, :, h, :])
                    z = z + phiK.sum(axis=0)
                for t in frames:
                    phiQ = np.maximum(_f64(q[b, t, :, h, :]), 0.0)
                    out[b, t, :, h, :] = (phiQ @ S) / (phiQ @ z + eps)[:, None]
            s_out[b, h] = S
            z_out[b, h] = z
    return out, s_out, z_out


def e4m3_decode(codes) -> np.ndarray:
    """Value of every 8-bit E4M3 floating-point code, by the format's definition (the OCP 8-bit
    floating-point E4M3 encoding without infinities): bit 7 sign, bits 6..3 exponent e with bias
    7, bits 2..0 mantissa m; e = 0 encodes the subnormals (m / 8) * 2**-6, the code S.1111.111
    is NaN, every other code is (1 + m / 8) * 2**(e - 7). Largest finite magnitude 448."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where((c & 0x80) != 0, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    normal = (1.0 + m / 8.0) * np.exp2((e - 7).astype(np.float64))
    value = np.where(e == 0, (m / 8.0) * 2.0 ** -6, normal)
    value = np.where((e == 15) & (m == 7), np.nan, value)
    return sign * value


def gdn_frame_forward_fp8(q8, k8, v8, q_scale, k_scale, v_scale, gamma, beta, state_in,
                          key_scale: float):
    """The layer on 8-bit E4M3 inputs with one scale per (batch, frame, head).

    The SANA-Streaming entry of the jefxiong.cn AIGC digest (2026-06-01), item 1, contribution
    (3), pairs the fused GDN kernel with mixed-precision quantisation to keep the tensor cores
    busy, and gives no quantiser. Reading adopted: q = decode(q8) * q_scale[b, t, h] for every
    token and dim of frame t of head h (likewise k and v), then exactly the layer of
    ``gdn_frame_forward`` on those values. q8, k8, v8: [B, T, N, H, D] uint8 codes; scales
    [B, T, H]."""
    def dequant(x8, scale):
        return e4m3_decode(x8) * _f64(scale)[:, :, None, :, None]

    return gdn_frame_forward(dequant(q8, q_scale), dequant(k8, k_scale), dequant(v8, v_scale),
                             gamma, beta, state_in, key_scale)


def frame_update_backward(S_prev, A, B, gamma: float, beta: float, G):
    """Adjoint of ``frame_update``: given G = dL/dS_t, return the gradients that flow to the
    update's inputs, (dS_prev, dA, dB, dgamma, dbeta).

    The chatpaper.ai abstract of SANA-WM says the model is trained natively on one-minute
    clips, so the layer needs its backward pass. This function is the chain rule applied to
    S_t = gamma * S_prev @ M + beta * B, where M = I - beta * A:
      dS_prev = gamma * G @ M^T
      dA      = -gamma * beta * S_prev^T @ G
      dB      = beta * G
      dgamma  = <G, S_prev @ M>
      dbeta   = <G, B - gamma * S_prev @ A>
    <X, Y> is the sum of X * Y over all elements."""
    D = A.shape[0]
    M = np.eye(D) - beta * A
    dS_prev = gamma * (G @ M.T)
    dA = -gamma * beta * (S_prev.T @ G)
    dB = beta * G
    dgamma = float(np.sum(G * (S_prev @ M)))
    dbeta = float(np.sum(G * (B - gamma * (S_prev @ A))))
    return dS_prev, dA, dB, dgamma, dbeta


def gdn_frame_backward(q, k, v, gamma, beta, state_in, d_out, d_state_out, key_scale: float):
    """Gradients of the frame-wise GDN layer (``gdn_frame_forward``) for given output and
    final-state cotangents.

    The chatpaper.ai abstract of SANA-WM says the model is trained natively on one-minute
    clips. gen-hub.ru, "Архитектура", says the 1/sqrt(D*S) key scale replaced L2 key
    normalisation and removed NaN divergence in training. So the backward is taken through
    the key scale: k' = s * k, and dk = s * dk'.

    Arguments: q, k, v, d_out: [B, T, N, H, D]; gamma, beta: [B, T, H]; state_in,
    d_state_out: [B, H, D, D] or None (zero).
    Returns (dq, dk, dv [B,T,N,H,D], dgamma, dbeta [B,T,H], dstate_in [B,H,D,D]), all
    float64.

    Per (batch, head): first the forward, keeping every S_t. Then the frames in reverse with
    G = dL/dS_t:
      G_t    = dO_t^T Q_t + (what frame t+1 passed back; d_state_out for the last frame)
      dQ_t   = dO_t S_t                    (from O_t = Q_t S_t^T)
      then ``frame_update_backward`` gives dA_t, dB_t, dgamma_t, dbeta_t and what flows to
      S_{t-1}
      dK'_t  = K'_t (dA_t + dA_t^T) + V_t dB_t    (A_t = K'^T K', B_t = V^T K')
      dV_t   = K'_t dB_t^T
    The gradient that reaches S_0 is dstate_in."""
    q = np.asarray(q)
    k = np.asarray(k)
    v = np.asarray(v)
    d_out = np.asarray(d_out)
    gamma = _f64(gamma)
    beta = _f64(beta)
    s = float(key_scale)
    Bsz, T, N, H, D = q.shape
    dq = np.zeros((Bsz, T, N, H, D))
    dk = np.zeros((Bsz, T, N, H, D))
    dv = np.zeros((Bsz, T, N, H, D))
    dgamma = np.zeros((Bsz, T, H))
    dbeta = np.zeros((Bsz, T, H))
    dstate_in = np.zeros((Bsz, H, D, D))
    for b in range(Bsz):
        for h in range(H):
            # forward, keeping S_{t-1} and the statistics of every frame
            S = np.zeros((D, D)) if state_in is None else _f64(state_in[b, h]).copy()
            states = [S]
            stats = []
            for t in range(T):
                A, Bm = frame_statistics(k[b, t, :, h, :], v[b, t, :, h, :], s)
                stats.append((A, Bm))
                S = frame_update(S, A, Bm, gamma[b, t, h], beta[b, t, h])
                states.append(S)
            # reverse
            G = np.zeros((D, D)) if d_state_out is None else _f64(d_state_out[b, h]).copy()
            for t in range(T - 1, -1, -1):
                Q = _f64(q[b, t, :, h, :])
                Ks = s * _f64(k[b, t, :, h, :])
                V = _f64(v[b, t, :, h, :])
                dO = _f64(d_out[b, t, :, h, :])
                G = G + dO.T @ Q
                dq[b, t, :, h, :] = dO @ states[t + 1]
                A, Bm = stats[t]
                G, dA, dB, dgamma[b, t, h], dbeta[b, t, h] = frame_update_backward(
                    states[t], A, Bm, gamma[b, t, h], beta[b, t, h], G)
                dKs = Ks @ (dA + dA.T) + V @ dB
                dk[b, t, :, h, :] = s * dKs
                dv[b, t, :, h, :] = Ks @ dB.T
            dstate_in[b, h] = G
    return dq, dk, dv, dgamma, dbeta, dstate_in
