"""Pins for the fp64 oracle, against facts that do not come from the oracle.

Each pin is independent of the oracle's own code: hand-worked numbers, the
Householder product form of the delta rule written as explicit matrix
products, exact storage under orthonormal keys, the beta=0/alpha=1 no-op, the
RWKV6 closed-form sum evaluated by scalar loops, and its reduction to causal
linear attention.  The last test plants plausible mistakes in copies of the
oracle and checks that some pin catches each one.
"""
import json
import math
import os

import numpy as np
import pytest

from oracle import deferred, eager, gdn_eager, kda_eager, rwkv6_eager

RTOL_GOLDEN = 2e-6      # decays enter as fp32 logs of 0.5 / 1.0


def relerr(x, ref):
    x, ref = np.asarray(x, np.float64), np.asarray(ref, np.float64)
    return float(np.max(np.abs(x - ref)) / max(np.max(np.abs(ref)), 1e-300))


def _golden(golden_dir):
    with open(os.path.join(golden_dir, "hand_worked_d2.json")) as f:
        return json.load(f)


def _golden_inputs(g, op):
    st = g[op]["steps"]
    S0 = np.array(g[op]["S0"], np.float64)
    if op == "rwkv6":
        inp = {"r": np.array([s["r"] for s in st], float),
               "k": np.array([s["k"] for s in st], float),
               "v": np.array([s["v"] for s in st], float),
               "log_decay": np.log(np.array([s["w"] for s in st], np.float32)).astype(np.float32)}
        return S0, inp, np.array(g[op]["u"], float)
    inp = {"q": np.array([s["q"] for s in st], float),
           "k": np.array([s["k"] for s in st], float),
           "v": np.array([s["v"] for s in st], float),
           "log_decay": np.log(np.array([s["alpha"] for s in st], np.float32)).astype(np.float32),
           "beta": np.array([s["beta"] for s in st], float)}
    return S0, inp, None


@pytest.mark.parametrize("op", ["gdn", "kda", "rwkv6"])
def test_hand_worked_examples(golden_dir, op):
    g = _golden(golden_dir)
    S0, inp, u = _golden_inputs(g, op)
    o, S, _ = eager(op, S0, inp, u=u)
    assert relerr(o, g[op]["o"]) < RTOL_GOLDEN
    assert relerr(S, g[op]["S_final"]) < RTOL_GOLDEN
    for M in (1, 2, 3):
        od, Sd, _ = deferred(op, M, S0, inp, u=u)
        assert relerr(od, g[op]["o"]) < RTOL_GOLDEN
        assert relerr(Sd, g[op]["S_final"]) < RTOL_GOLDEN


def _tiny_delta_inputs(rng, op, T, d_k, d_v, units=()):
    k = rng.standard_normal((T,) + units + (d_k,))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    q = rng.standard_normal((T,) + units + (d_k,))
    v = rng.standard_normal((T,) + units + (d_v,))
    gshape = (T,) + units + ((d_k,) if op == "kda" else ())
    la = (-np.log1p(np.exp(rng.standard_normal(gshape)))).astype(np.float32)
    be = 1.0 / (1.0 + np.exp(-rng.standard_normal((T,) + units)))
    return {"q": q, "k": k, "v": v, "log_decay": la, "beta": be}


def _householder_states(op, S0, inp):
    """S_t from A_t = (I - beta k k^T) diag(alpha) unrolled as matrix products."""
    T = inp["k"].shape[0]
    d_k = S0.shape[0]
    A, W = [], []
    for t in range(T):
        alpha = np.exp(np.asarray(inp["log_decay"][t], np.float64))
        D = alpha * np.eye(d_k) if op == "gdn" else np.diag(alpha)
        kk = inp["k"][t].reshape(d_k, 1)
        A.append((np.eye(d_k) - inp["beta"][t] * (kk @ kk.T)) @ D)
        W.append(inp["beta"][t] * (kk @ inp["v"][t].reshape(1, -1)))
    states = []
    for t in range(T):
        P = np.eye(d_k)
        for j in range(t, -1, -1):          # A_t A_{t-1} ... A_0
            P = P @ A[j]
        S = P @ S0
        for i in range(t + 1):
            Q = np.eye(d_k)
            for j in range(t, i, -1):       # A_t ... A_{i+1}
                Q = Q @ A[j]
            S = S + Q @ W[i]
        states.append(S)
    return states


@pytest.mark.parametrize("op", ["gdn", "kda"])
@pytest.mark.parametrize("shape", [(4, 3), (5, 5), (3, 6)])
def test_householder_product_form(op, shape):
    d_k, d_v = shape
    rng = np.random.default_rng(11 + d_k * 7 + d_v)
    T = 6
    S0 = rng.standard_normal((d_k, d_v))
    inp = _tiny_delta_inputs(rng, op, T, d_k, d_v)
    fn = gdn_eager if op == "gdn" else kda_eager
    o, S_T, kept = fn(S0, inp["q"], inp["k"], inp["v"], inp["log_decay"], inp["beta"],
                      record=set(range(T)))
    ref = _householder_states(op, S0, inp)
    for t in range(T):
        assert relerr(kept[t], ref[t]) < 1e-12
        assert relerr(o[t], ref[t].T @ inp["q"][t]) < 1e-12
    assert relerr(S_T, ref[-1]) < 1e-12


@pytest.mark.parametrize("op", ["gdn", "kda"])
def test_delta_rule_stores_orthonormal_keys(op):
    rng = np.random.default_rng(5)
    d_k, d_v = 6, 5
    Q, _ = np.linalg.qr(rng.standard_normal((d_k, d_k)))
    keys = Q.T                               # rows are orthonormal
    T = d_k
    vals = rng.standard_normal((T, d_v))
    S0 = rng.standard_normal((d_k, d_v))
    qsel = [(3 * t) % (t + 1) for t in range(T)]   # some earlier-or-current key
    inp = {"q": keys[qsel], "k": keys, "v": vals,
           "log_decay": np.zeros((T,) if op == "gdn" else (T, d_k), np.float32),
           "beta": np.ones(T)}
    o, S, kept = eager(op, S0, inp, record=set(range(T)))
    for t in range(T):
        for i in range(t + 1):
            np.testing.assert_allclose(kept[t].T @ keys[i], vals[i], atol=1e-12, rtol=0)
        np.testing.assert_allclose(o[t], vals[qsel[t]], atol=1e-12, rtol=0)


@pytest.mark.parametrize("op", ["gdn", "kda"])
def test_noop_beta0_alpha1(op):
    rng = np.random.default_rng(9)
    d_k, d_v, T = 5, 4, 7
    S0 = rng.standard_normal((d_k, d_v))
    inp = _tiny_delta_inputs(rng, op, T, d_k, d_v)
    inp["beta"] = np.zeros(T)
    inp["log_decay"] = np.zeros_like(inp["log_decay"])
    o, S, _ = eager(op, S0, inp)
    assert np.array_equal(S, S0)
    for t in range(T):
        assert relerr(o[t], S0.T @ inp["q"][t]) < 1e-14
    for M in (1, 4, 8):
        od, Sd, _ = deferred(op, M, S0, inp)
        assert relerr(od, o) < 1e-14 and relerr(Sd, S0) < 1e-14


def _rwkv6_tiny(rng, T, d_k, d_v):
    return {"r": rng.standard_normal((T, d_k)), "k": rng.standard_normal((T, d_k)),
            "v": rng.standard_normal((T, d_v)),
            "log_decay": (-np.exp(rng.standard_normal((T, d_k)) * 0.5 - 0.5)).astype(np.float32)}


def test_rwkv6_closed_form_sum():
    rng = np.random.default_rng(3)
    d_k, d_v, T = 4, 3, 6
    S0 = rng.standard_normal((d_k, d_v))
    u = rng.standard_normal(d_k) * 0.1
    inp = _rwkv6_tiny(rng, T, d_k, d_v)
    w = np.exp(np.asarray(inp["log_decay"], np.float64))
    r, k, v = inp["r"], inp["k"], inp["v"]
    o, _, _ = rwkv6_eager(S0, u, r, k, v, inp["log_decay"])
    for t in range(T):
        want = [0.0] * d_v
        for c in range(d_v):
            acc = 0.0
            for i in range(t):                      # past tokens, decayed
                dot = 0.0
                for j in range(d_k):
                    prod = 1.0
                    for m in range(i + 1, t):
                        prod *= w[m, j]
                    dot += r[t, j] * prod * k[i, j]
                acc += dot * v[i, c]
            bon = sum(u[j] * k[t, j] * r[t, j] for j in range(d_k))
            acc += bon * v[t, c]                    # current token through the bonus
            for j in range(d_k):                    # initial state, decayed
                prod = 1.0
                for m in range(t):
                    prod *= w[m, j]
                acc += S0[j, c] * prod * r[t, j]
            want[c] = acc
        assert relerr(o[t], want) < 1e-13


def test_rwkv6_reduces_to_causal_linear_attention():
    rng = np.random.default_rng(4)
    d_k, d_v, T = 4, 5, 7
    inp = _rwkv6_tiny(rng, T, d_k, d_v)
    inp["log_decay"] = np.zeros_like(inp["log_decay"])
    o, _, _ = rwkv6_eager(np.zeros((d_k, d_v)), np.zeros(d_k), inp["r"], inp["k"], inp["v"],
                          inp["log_decay"])
    for t in range(T):
        want = sum((float(np.dot(inp["k"][i], inp["r"][t])) * inp["v"][i] for i in range(t)),
                   np.zeros(d_v))
        np.testing.assert_allclose(o[t], want, atol=1e-13, rtol=0)


def _units_inputs(op, rng, T, units, d_k, d_v):
    if op == "rwkv6":
        inp = {"r": rng.standard_normal((T,) + units + (d_k,)),
               "k": rng.standard_normal((T,) + units + (d_k,)),
               "v": rng.standard_normal((T,) + units + (d_v,)),
               "log_decay": (-np.exp(rng.standard_normal((T,) + units + (d_k,)) * 0.5 - 0.5)
                             ).astype(np.float32)}
        return inp, rng.standard_normal(units[-1:] + (d_k,)) * 0.1
    return _tiny_delta_inputs(rng, op, T, d_k, d_v, units), None


@pytest.mark.parametrize("op", ["gdn", "kda", "rwkv6"])
def test_deferred_equals_eager_every_M(op):
    rng = np.random.default_rng(21)
    units, d_k, d_v, T = (2, 3), 4, 3, 40
    S0 = rng.standard_normal(units + (d_k, d_v)) * 0.5
    inp, u = _units_inputs(op, rng, T, units, d_k, d_v)
    o_ref, S_ref, kept = eager(op, S0, inp, u=u, record=set(range(T)))
    for M in range(1, 34):
        o, S, merges = deferred(op, M, S0, inp, u=u)
        assert relerr(o, o_ref) < 1e-12, M
        assert relerr(S, S_ref) < 1e-12, M
        assert sorted(merges) == [t for t in range(T) if (t + 1) % M == 0], M
        for t, Sbar in merges.items():       # each merged base is the eager state
            assert relerr(Sbar, kept[t]) < 1e-12, (M, t)


def test_deferred_M1_is_eager_on_workload_draws():
    from synthetic import initial_state, sequence
    for op in ("gdn", "kda", "rwkv6"):
        S0 = initial_state(0, 2, 2, 8, 8)
        inp = sequence(0, op, 2, 2, 8, 8, 12, bf16=True)
        u = np.full((2, 8), 0.05) if op == "rwkv6" else None
        o_ref, S_ref, _ = eager(op, S0, inp, u=u)
        o, S, _ = deferred(op, 1, S0, inp, u=u)
        assert relerr(o, o_ref) < 1e-13 and relerr(S, S_ref) < 1e-13


# ---- planted mistakes: each must be caught by some pin --------------------------

def _mutant_gdn(kind):
    def run(S0, q, k, v, la, be, record=()):
        S = np.array(S0, np.float64)
        T = q.shape[0]
        o = np.empty(q.shape[:-1] + (S.shape[-1],))
        kept = {}
        for t in range(T):
            a = math.exp(float(la[t]))
            prev = S
            if kind == "no_decay_in_correction":
                b = be[t] * (v[t] - S.T @ k[t])
            elif kind == "transposed_read":
                b = be[t] * (v[t] - (a * S) @ k[t])
            elif kind == "sign":
                b = be[t] * (v[t] + (a * S).T @ k[t])
            else:
                b = be[t] * (v[t] - (a * S).T @ k[t])
            S = a * S + np.outer(k[t], b)
            o[t] = (prev.T if kind == "output_from_previous_state" else S.T) @ q[t]
            if t in record:
                kept[t] = S.copy()
        return o, S, kept
    return run


@pytest.mark.parametrize("kind", ["no_decay_in_correction", "transposed_read", "sign",
                                  "output_from_previous_state"])
def test_planted_mistakes_are_caught(golden_dir, kind):
    run = _mutant_gdn(kind)
    caught = []
    g = _golden(golden_dir)
    S0, inp, _ = _golden_inputs(g, "gdn")
    o, S, _ = run(S0, inp["q"], inp["k"], inp["v"], inp["log_decay"], inp["beta"])
    caught.append(relerr(o, g["gdn"]["o"]) > 1e-3 or relerr(S, g["gdn"]["S_final"]) > 1e-3)
    rng = np.random.default_rng(2)
    d = 5
    S0 = rng.standard_normal((d, d))
    tin = _tiny_delta_inputs(rng, "gdn", 5, d, d)
    o, _, kept = run(S0, tin["q"], tin["k"], tin["v"], tin["log_decay"], tin["beta"],
                     record=set(range(5)))
    ref = _householder_states("gdn", S0, tin)
    caught.append(any(relerr(kept[t], ref[t]) > 1e-6 or relerr(o[t], ref[t].T @ tin["q"][t]) > 1e-6
                      for t in range(5)))
    assert all(caught), caught
