"""Plant plausible mistakes in copies of the oracle (on the CPU) and check that every one of
them fails at least one pin. This shows the pins constrain each term, sign, index and
operand order of the oracle, not only its happy path."""
import types

import numpy as np
import pytest

import oracle
import oracle.gdn_oracle as go
from tests import oracle_pins


def _decode_variant(bias=7, subnormals=True):
    """e4m3 decoding with a planted mistake."""
    def decode(codes):
        c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
        sign = np.where((c & 0x80) != 0, -1.0, 1.0)
        e = (c >> 3) & 0xF
        m = (c & 0x7).astype(np.float64)
        normal = (1.0 + m / 8.0) * np.exp2((e - bias).astype(np.float64))
        val = np.where(e == 0, (m / 8.0) * 2.0 ** (1 - bias), normal) if subnormals else normal
        val = np.where((e == 15) & (m == 7), np.nan, val)
        return sign * val
    return decode


def _impl(stats=None, update=None, output=None, forward=None, la=None, decode=None,
          swap_kv_scales=False, backward=None):
    """An oracle copy with some pieces swapped; gdn_frame_step and the fp8 forward follow the
    swapped forward and decoder."""
    decode = decode or go.e4m3_decode
    stats = stats or go.frame_statistics
    update = update or go.frame_update
    output = output or go.frame_output

    def fwd(q, k, v, gamma, beta, state_in, key_scale):
        q, k, v = np.asarray(q), np.asarray(k), np.asarray(v)
        B, T, N, H, D = q.shape
        out = np.zeros(q.shape)
        st = np.zeros((B, H, D, D))
        for b in range(B):
            for h in range(H):
                S = np.zeros((D, D)) if state_in is None else np.array(state_in[b, h], float)
                for t in range(T):
                    A, Bm = stats(k[b, t, :, h], v[b, t, :, h], key_scale)
                    S = update(S, A, Bm, float(gamma[b, t, h]), float(beta[b, t, h]))
                    out[b, t, :, h] = output(q[b, t, :, h], S)
                st[b, h] = S
        return out, st

    forward = forward or fwd

    def step(q, k, v, gamma, beta, state_in, key_scale):
        o, s = forward(np.asarray(q)[:, None], np.asarray(k)[:, None], np.asarray(v)[:, None],
                       np.asarray(gamma)[:, None], np.asarray(beta)[:, None], state_in, key_scale)
        return o[:, 0], s

    def fwd_fp8(q8, k8, v8, q_scale, k_scale, v_scale, gamma, beta, state_in, key_scale):
        if swap_kv_scales:
            k_scale, v_scale = v_scale, k_scale
        deq = lambda x8, sc: decode(x8) * np.asarray(sc, float)[:, :, None, :, None]
        return forward(deq(q8, q_scale), deq(k8, k_scale), deq(v8, v_scale), gamma, beta,
                       state_in, key_scale)

    return types.SimpleNamespace(gdn_frame_forward=forward, gdn_frame_step=step,
                                 la_block_causal=la or oracle.la_block_causal,
                                 frame_statistics=stats, e4m3_decode=decode,
                                 gdn_frame_forward_fp8=fwd_fp8,
                                 gdn_frame_backward=backward or oracle.gdn_frame_backward)


def _old_state_forward(q, k, v, gamma, beta, state_in, key_scale):
    """Mistake: frame t's output reads S_{t-1} instead of S_t."""
    q, k, v = np.asarray(q), np.asarray(k), np.asarray(v)
    B, T, N, H, D = q.shape
    out = np.zeros(q.shape)
    st = np.zeros((B, H, D, D))
    for b in range(B):
        for h in range(H):
            S = np.zeros((D, D)) if state_in is None else np.array(state_in[b, h], float)
            for t in range(T):
                out[b, t, :, h] = q[b, t, :, h] @ S.T
                A, Bm = go.frame_statistics(k[b, t, :, h], v[b, t, :, h], key_scale)
                S = go.frame_update(S, A, Bm, gamma[b, t, h], beta[b, t, h])
            st[b, h] = S
    return out, st


def _la_variant(relu_q=True, relu_k=True, eps=1e-6, transpose_state=False, frame_causal=False):
    def la(q, k, v, state_in, z_in, frames_per_block, eps_=1e-6):
        q, k, v = np.asarray(q, float), np.asarray(k, float), np.asarray(v, float)
        B, T, N, H, D = q.shape
        F = 1 if frame_causal else int(frames_per_block)
        out = np.zeros(q.shape)
        so = np.zeros((B, H, D, D))
        zo = np.zeros((B, H, D))
        fq = (lambda x: np.maximum(x, 0)) if relu_q else (lambda x: x)
        fk = (lambda x: np.maximum(x, 0)) if relu_k else (lambda x: x)
        for b in range(B):
            for h in range(H):
                S = np.zeros((D, D)) if state_in is None else np.array(state_in[b, h], float)
                z = np.zeros(D) if z_in is None else np.array(z_in[b, h], float)
                for t0 in range(0, T, F):
                    fr = range(t0, min(t0 + F, T))
                    for t in fr:
                        pk = fk(k[b, t, :, h])
                        S = S + (v[b, t, :, h].T @ pk if transpose_state else pk.T @ v[b, t, :, h])
                        z = z + pk.sum(0)
                    for t in fr:
                        pq = fq(q[b, t, :, h])
                        with np.errstate(all="ignore"):
                            out[b, t, :, h] = (pq @ S) / (pq @ z + eps)[:, None]
                so[b, h], zo[b, h] = S, z
        return out, so, zo
    return la


def _bwd_variant(mistake):
    """The backward with one planted mistake (named by ``mistake``)."""
    def bwd(q, k, v, gamma, beta, state_in, d_out, d_state_out, s):
        q, k, v, d_out = (np.asarray(x, float) for x in (q, k, v, d_out))
        B, T, N, H, D = q.shape
        dq, dk, dv = np.zeros(q.shape), np.zeros(q.shape), np.zeros(q.shape)
        dg, db = np.zeros((B, T, H)), np.zeros((B, T, H))
        ds0 = np.zeros((B, H, D, D))
        I = np.eye(D)
        for b in range(B):
            for h in range(H):
                S = np.zeros((D, D)) if state_in is None else np.array(state_in[b, h], float)
                states, stats = [S], []
                for t in range(T):
                    A, Bm = go.frame_statistics(k[b, t, :, h], v[b, t, :, h], s)
                    stats.append((A, Bm))
                    S = go.frame_update(S, A, Bm, gamma[b, t, h], beta[b, t, h])
                    states.append(S)
                G = np.zeros((D, D)) if d_state_out is None else np.array(d_state_out[b, h], float)
                for t in range(T - 1, -1, -1):
                    Q, Ks, V, dO = q[b, t, :, h], s * k[b, t, :, h], v[b, t, :, h], d_out[b, t, :, h]
                    g, be = gamma[b, t, h], beta[b, t, h]
                    A, Bm = stats[t]
                    Sp = states[t]
                    if mistake == "state_grad_not_carried":
                        G = dO.T @ Q
                    else:
                        G = G + (Q.T @ dO if mistake == "E_transposed" else dO.T @ Q)
                    dq[b, t, :, h] = dO @ (Sp if mistake == "dq_reads_previous_state" else states[t + 1])
                    M = I - be * A
                    Sg = states[t + 1] if mistake == "dgamma_reads_new_state" else Sp
                    dg[b, t, h] = np.sum(G * (Sg @ M))
                    sign = 1.0 if mistake == "dbeta_gamma_term_sign" else -1.0
                    db[b, t, h] = np.sum(G * (Bm + sign * g * (Sp @ A)))
                    dA = -g * be * (Sp.T @ G)
                    dB = be * G
                    sym = 2 * dA if mistake == "dA_not_symmetrised" else dA + dA.T
                    dKs = Ks @ sym + V @ dB
                    dk[b, t, :, h] = dKs if mistake == "key_scale_dropped_on_dk" else s * dKs
                    dv[b, t, :, h] = Ks @ (dB if mistake == "dv_dB_not_transposed" else dB.T)
                    G = g * ((M @ G) if mistake == "gate_on_wrong_side" else (G @ M.T))
                ds0[b, h] = G
        return dq, dk, dv, dg, db, ds0
    return bwd


BWD_MISTAKES = [
    "E_transposed", "state_grad_not_carried", "dq_reads_previous_state", "dgamma_reads_new_state",
    "dbeta_gamma_term_sign", "dA_not_symmetrised", "key_scale_dropped_on_dk",
    "dv_dB_not_transposed", "gate_on_wrong_side",
]


MUTANTS = {
    "gamma_also_scales_beta_B": dict(update=lambda S, A, B, g, b: g * (S @ (np.eye(len(A)) - b * A) + b * B)),
    "transposed_state_product": dict(update=lambda S, A, B, g, b: g * ((np.eye(len(A)) - b * A) @ S) + b * B),
    "sign_of_delta_term": dict(update=lambda S, A, B, g, b: g * (S @ (np.eye(len(A)) + b * A)) + b * B),
    "beta_dropped_on_A": dict(update=lambda S, A, B, g, b: g * (S @ (np.eye(len(A)) - A)) + b * B),
    "beta_dropped_on_B": dict(update=lambda S, A, B, g, b: g * (S @ (np.eye(len(A)) - b * A)) + B),
    "gamma_dropped": dict(update=lambda S, A, B, g, b: S @ (np.eye(len(A)) - b * A) + b * B),
    "key_scale_once_on_A": dict(stats=lambda K, V, s: (s * (np.asarray(K, float).T @ np.asarray(K, float)),
                                                       np.asarray(V, float).T @ (s * np.asarray(K, float)))),
    "B_transposed": dict(stats=lambda K, V, s: ((s * np.asarray(K, float)).T @ (s * np.asarray(K, float)),
                                                (s * np.asarray(K, float)).T @ np.asarray(V, float))),
    "B_unscaled": dict(stats=lambda K, V, s: ((s * np.asarray(K, float)).T @ (s * np.asarray(K, float)),
                                              np.asarray(V, float).T @ np.asarray(K, float))),
    "output_not_transposed": dict(output=lambda Q, S: np.asarray(Q, float) @ S),
    "output_reads_previous_state": dict(forward=_old_state_forward),
    "la_no_relu_on_q": dict(la=_la_variant(relu_q=False)),
    "la_no_relu_on_k": dict(la=_la_variant(relu_k=False)),
    "la_eps_dropped": dict(la=_la_variant(eps=0.0)),
    "la_state_transposed": dict(la=_la_variant(transpose_state=True)),
    "la_frame_causal_not_block_causal": dict(la=_la_variant(frame_causal=True)),
    "e4m3_exponent_bias_8": dict(decode=_decode_variant(bias=8)),
    "e4m3_subnormals_read_as_normals": dict(decode=_decode_variant(subnormals=False)),
    "fp8_k_and_v_scales_swapped": dict(swap_kv_scales=True),
    **{"bwd_" + m: dict(backward=_bwd_variant(m)) for m in BWD_MISTAKES},
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name):
    impl = _impl(**MUTANTS[name])
    failed = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(impl)
        except (AssertionError, FloatingPointError, ValueError):
            failed.append(pin.__name__)
    assert failed, f"mutant {name} passes every pin"


def test_unmutated_copy_passes():
    impl = _impl(backward=_bwd_variant("none"))
    for pin in oracle_pins.ALL_PINS:
        pin(impl)
