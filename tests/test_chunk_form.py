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

Two rearrangements that the tensor-memory kernels make are checked as well:
blocks of pairs of a 32-token chunk as products of rows scaled once each
through a token between them (tokens 15, 7 and 23), and (I + A)^{-1} by
16 x 16 blocks.
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


def _pair_weights(K, Q, G, Gq, be):
    """A and P of one chunk pair by pair (per-key weights e^{Gq_t - G_s})."""
    n = len(K)
    A, P = np.zeros((n, n)), np.zeros((n, n))
    for t in range(n):
        for s in range(t):
            P[t, s] = np.sum(Q[t] * K[s] * np.exp(Gq[t] - G[s]))
            if be is not None:
                A[t, s] = be[t] * np.sum(K[t] * K[s] * np.exp(G[t] - G[s]))
    return A, P


@pytest.mark.parametrize("op", ["kda", "rwkv6"])
@pytest.mark.parametrize("strong", [False, True])
def test_pair_blocks_through_a_reference_token(op, strong):
    """The tensor-memory kernels form blocks of pairs of a 32-token chunk as
    products of rows scaled once each, through a token r between s and t:
    e^{G_t - G_s} = e^{G_t - G_r} e^{G_r - G_s}.  The 16 x 16 block t >= 16 > s
    goes through token 15; inside each half, the 8 x 8 block of its second
    quarter against its first goes through token 7 or 23.  Every exponent is
    <= 0 (no cumulative decay is divided by) and each block equals the
    pair-by-pair one."""
    d, C = 16, 32
    seq = sequence(11, op, 1, 1, d, d, C, bf16=True)
    one = _unit(seq, 0, 0)
    g = one["log_decay"].astype(np.float64).copy()
    if strong:
        g[:, :5] = -40.0
    G = np.cumsum(g, axis=0)
    Gq = G if op == "kda" else np.vstack([np.zeros((1, d)), G[:-1]])   # Gamma_{t-1} for RWKV6's P
    K = one["k"].astype(np.float64)
    Q = one["r" if op == "rwkv6" else "q"].astype(np.float64)
    be = one["beta"].astype(np.float64) if op == "kda" else None
    A, P = _pair_weights(K, Q, G, Gq, be)

    # level 1: t >= 16 > s through token 15; level 2: second quarter against
    # first quarter of each half, through token 7 or 23
    blocks = [(slice(16, 32), slice(0, 16), 15), (slice(8, 16), slice(0, 8), 7), (slice(24, 32), slice(16, 24), 23)]
    for hi, lo, r in blocks:
        ds, dt, dq = G[r] - G[lo], G[hi] - G[r], Gq[hi] - G[r]
        assert ds.max() <= 0 and dt.max() <= 0 and dq.max() <= 0
        Ks, Kt, Qt = K[lo] * np.exp(ds), K[hi] * np.exp(dt), Q[hi] * np.exp(dq)
        assert np.abs(Qt @ Ks.T - P[hi, lo]).max() <= 1e-12 * max(np.abs(P).max(), 1e-300), r
        if be is not None:
            assert np.abs(be[hi, None] * (Kt @ Ks.T) - A[hi, lo]).max() <= 1e-12 * np.abs(A).max(), r
    # what is left pair by pair: the strict pairs inside the four quarters
    left = sum(1 for t in range(C) for s_ in range(t) if t // 8 == s_ // 8)
    assert left == 4 * 28


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_blocked_inverse_of_unit_lower(seed):
    """(I + A)^{-1} for a strictly lower 32 x 32 A as the kernels form it: the
    diagonal blocks T11, T22 column by column by forward substitution, then
    T21 = -T22 (A21 T11); T12 = 0.  Checked against a dense inverse, and
    W = T R against a triangular solve."""
    rng = np.random.default_rng(seed)
    n = 32
    A = np.tril(rng.standard_normal((n, n)) * 0.3, -1)
    T = np.zeros((n, n))
    for c in range(n):
        r0 = c & ~15
        x = np.zeros(16)
        for i in range(16):
            t = r0 + i
            x[i] = 1.0 if t == c else 0.0 if t < c else -A[t, r0:r0 + i] @ x[:i]
        T[r0:r0 + 16, c] = x
    T[16:, :16] = -T[16:, 16:] @ (A[16:, :16] @ T[:16, :16])
    I = np.eye(n)
    ref = np.linalg.inv(I + A)
    assert np.abs(T - ref).max() <= 1e-10 * np.abs(ref).max()
    R = rng.standard_normal((n, 8))
    assert np.allclose(T @ R, np.linalg.solve(I + A, R), rtol=0, atol=1e-10 * np.abs(R).max() * np.abs(ref).max())
