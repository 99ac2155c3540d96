"""The chunk form that the chunked prefill kernels compute, restated in plain
fp64 numpy and checked against the eager oracle.

The kernels process C tokens of a prompt at once.  With Gamma_t the
cumulative log-decay inside the chunk (a scalar per head for GDN, a d_k
vector for KDA and RWKV6) and S the state at the chunk start:

GDN / KDA (delta rule), with the pair weights w[t][s] = e^{Gamma_t - Gamma_s}
(per key for KDA):
    A[t][s] = beta_t sum_j k_tj k_sj w_j[t][s]            (s < t)
    (I + A) W = diag(beta) (e^{Gamma} (.) K),   (I + A) U = diag(beta) V
    B = U - W S
    P[t][s] = sum_j q_tj k_sj w_j[t][s]                   (s <= t)
    O = (e^{Gamma} (.) Q) S + P B
    S <- diag(e^{Gamma_end}) S + (e^{Gamma_end - Gamma} (.) K)^T B
RWKV6 (raw update, output from the state before the token):
    P[t][s] = sum_j r_tj k_sj e^{Gamma_{t-1,j} - Gamma_sj}    (s < t)
    P[t][t] = (u (.) k_t) . r_t
    O = (e^{Gamma_{t-1}} (.) R) S + P V
    S <- diag(e^{Gamma_end}) S + (e^{Gamma_end - Gamma} (.) K)^T V

Expanding the per-token recurrences over C tokens gives these equations;
this test checks that they hold (to fp64 rounding) for chunk sizes from 1 to
past the prompt length, including a ragged last chunk, on the bench's input
recipe and on strongly decaying gates.  It shares nothing with the CUDA code.
"""
import numpy as np
import pytest

from oracle import eager
from synthetic import bonus, initial_state, sequence


def _chunk_form(op, S0, inp, u, C):
    """One unit (a slot-head): S0 [d_k, d_v], inputs [T, d]; returns (o [T, d_v], S_T)."""
    q = inp["r" if op == "rwkv6" else "q"].astype(np.float64)
    k, v = inp["k"].astype(np.float64), inp["v"].astype(np.float64)
    g = inp["log_decay"].astype(np.float64)
    T, dk = k.shape
    if op == "gdn":
        g = np.repeat(g[:, None], dk, axis=1)          # a scalar decay acts on every key alike
    S = S0.astype(np.float64).copy()
    out = []
    for c0 in range(0, T, C):
        Q, K, V, G = q[c0:c0 + C], k[c0:c0 + C], v[c0:c0 + C], np.cumsum(g[c0:c0 + C], axis=0)
        n = len(K)
        if op == "rwkv6":
            Gq = np.vstack([np.zeros((1, dk)), G[:-1]])  # Gamma_{t-1}
            P = np.zeros((n, n))
            for t in range(n):
                for s in range(t):
                    P[t, s] = np.sum(Q[t] * K[s] * np.exp(Gq[t] - G[s]))
                P[t, t] = np.sum(u * K[t] * Q[t])
            B = V
            O = (np.exp(Gq) * Q) @ S + P @ B
        else:
            be = inp["beta"][c0:c0 + C].astype(np.float64)
            A = np.zeros((n, n))
            P = np.zeros((n, n))
            for t in range(n):
                for s in range(t + 1):
                    w = np.exp(G[t] - G[s])
                    P[t, s] = np.sum(Q[t] * K[s] * w)
                    if s < t:
                        A[t, s] = be[t] * np.sum(K[t] * K[s] * w)
            IA = np.eye(n) + A
            W = np.linalg.solve(IA, be[:, None] * np.exp(G) * K)
            U = np.linalg.solve(IA, be[:, None] * V)
            B = U - W @ S
            O = (np.exp(G) * Q) @ S + P @ B
        out.append(O)
        S = np.exp(G[-1])[:, None] * S + (np.exp(G[-1] - G) * K).T @ B
    return np.vstack(out), S


def _unit(seq, b, h):
    return {key: val[:, b, h] for key, val in seq.items()}


@pytest.mark.parametrize("op", ["gdn", "kda", "rwkv6"])
@pytest.mark.parametrize("C", [1, 4, 16, 32, 64])
def test_chunk_form_equals_eager(op, C):
    """T = 45 tokens: full chunks and a ragged tail for every C < 45."""
    B, H, d, T = 2, 2, 16, 45
    seq = sequence(3, op, B, H, d, d, T, bf16=True)
    S0 = initial_state(3, B, H, d, d)
    u = bonus(3, H, d) if op == "rwkv6" else None
    for b in range(B):
        for h in range(H):
            one = _unit(seq, b, h)
            o_ref, S_ref, _ = eager(op, S0[b, h], one, None if u is None else u[h])
            o, S = _chunk_form(op, S0[b, h], one, None if u is None else u[h], C)
            scale_o, scale_s = np.abs(o_ref).max(), np.abs(S_ref).max()
            assert np.abs(o - o_ref).max() <= 1e-12 * scale_o, (b, h)
            assert np.abs(S - S_ref).max() <= 1e-12 * scale_s, (b, h)


@pytest.mark.parametrize("op", ["kda", "rwkv6"])
def test_chunk_form_strong_decay(op):
    """Per-step log-decays of -40 on some keys: a 16-token chunk's cumulative
    log-decay reaches -640, far past what fp32 could divide by (e^87), yet no
    weight divides by it, so the chunk form stays finite and equal to the
    recurrence."""
    B, H, d, T, C = 1, 1, 8, 40, 16
    seq = sequence(5, op, B, H, d, d, T, bf16=True)
    one = _unit(seq, 0, 0)
    one["log_decay"] = one["log_decay"].copy()
    one["log_decay"][:, :3] = -40.0
    S0 = initial_state(5, B, H, d, d)[0, 0]
    u = bonus(5, H, d)[0] if op == "rwkv6" else None
    o_ref, S_ref, _ = eager(op, S0, one, u)
    o, S = _chunk_form(op, S0, one, u, C)
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(S))
    assert np.abs(o - o_ref).max() <= 1e-12 * np.abs(o_ref).max()
    assert np.abs(S - S_ref).max() <= 1e-12 * np.abs(S_ref).max()
