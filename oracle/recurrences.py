"""Plain fp64 recurrences of the three DeltaLog operators -- test infrastructure.

Shapes: the state ``S0[..., d_k, d_v]`` carries any number of leading unit
axes (slots, heads); per-step inputs carry a leading time axis ``[T, ..., d]``
and the same unit axes.  Every input is upcast to fp64 on entry; gates arrive
as fp32 natural-log decays and are exponentiated here in fp64.

Sources.  The operator list and their decay / update semantics are from the
DeltaLog technical summary (gist.science, section "Kernel implementation",
operator list): GDN = head-wise scalar decay with delta-rule correction, KDA =
per-key decay with delta-rule correction, RWKV6 = per-key decay with a raw
value update.  The formulas are the standard decode recurrences of those
models, restated:

GDN    S_t = a_t S_{t-1} + k_t b_t^T,  b_t = beta_t (v_t - a_t S_{t-1}^T k_t),
       o_t = S_t^T q_t                          (a_t scalar per head)
KDA    S_t = diag(a_t) S_{t-1} + k_t b_t^T,
       b_t = beta_t (v_t - (diag(a_t) S_{t-1})^T k_t),  o_t = S_t^T q_t
RWKV6  o_t = (S_{t-1} + diag(u) k_t v_t^T)^T r_t,
       S_t = diag(w_t) S_{t-1} + k_t v_t^T

The deferred schedule follows the DeltaLog summary's "Method -- core
mechanism (base + log)": a dense base, a bounded log of compact factors with
a log-decay snapshot per entry, M-1 append steps that leave the base alone,
and a merge every M steps that folds base + replayed log into the base and
empties the log.
"""
from __future__ import annotations

import numpy as np

_EINSUM_TK = "...kv,...k->...v"   # S^T x : contract the key axis of S with x


def _f64(x):
    return np.asarray(x, dtype=np.float64)


def _stateT_dot(S, x):
    """S^T x for every unit: sum over the key index k of S[k, v] x[k]."""
    return np.einsum(_EINSUM_TK, S, x)


def _outer(a, b):
    """a b^T for every unit."""
    return a[..., :, None] * b[..., None, :]


def gdn_eager(S0, q, k, v, log_alpha, beta, record=()):
    """Eager GDN decode; returns ``(o[T,...,d_v], S_T, {t: S_t for t in record})``.

    ``log_alpha`` is ``[T, ...]`` (one scalar per unit), ``beta`` ``[T, ...]``.
    """
    S = _f64(S0).copy()
    q, k, v, la, be = map(_f64, (q, k, v, log_alpha, beta))
    T = q.shape[0]
    o = np.empty(q.shape[:-1] + (S.shape[-1],))
    kept = {}
    for t in range(T):
        alpha = np.exp(la[t])[..., None, None]
        decayed = alpha * S                                   # a_t S_{t-1}
        b = be[t][..., None] * (v[t] - _stateT_dot(decayed, k[t]))
        S = decayed + _outer(k[t], b)
        o[t] = _stateT_dot(S, q[t])
        if t in record:
            kept[t] = S.copy()
    return o, S, kept


def kda_eager(S0, q, k, v, log_alpha, beta, record=()):
    """Eager KDA decode; ``log_alpha`` is ``[T, ..., d_k]`` (one per key)."""
    S = _f64(S0).copy()
    q, k, v, la, be = map(_f64, (q, k, v, log_alpha, beta))
    T = q.shape[0]
    o = np.empty(q.shape[:-1] + (S.shape[-1],))
    kept = {}
    for t in range(T):
        alpha = np.exp(la[t])[..., :, None]                   # diag(a_t) scales rows
        decayed = alpha * S
        b = be[t][..., None] * (v[t] - _stateT_dot(decayed, k[t]))
        S = decayed + _outer(k[t], b)
        o[t] = _stateT_dot(S, q[t])
        if t in record:
            kept[t] = S.copy()
    return o, S, kept


def rwkv6_eager(S0, u, r, k, v, log_w, record=()):
    """Eager RWKV6 decode; ``u`` broadcasts against ``[..., d_k]``."""
    S = _f64(S0).copy()
    u, r, k, v, lw = map(_f64, (u, r, k, v, log_w))
    T = r.shape[0]
    o = np.empty(r.shape[:-1] + (S.shape[-1],))
    kept = {}
    for t in range(T):
        bonus = _outer(u * k[t], v[t])                       # diag(u) k_t v_t^T
        o[t] = _stateT_dot(S + bonus, r[t])                   # reads S_{t-1}
        S = np.exp(lw[t])[..., :, None] * S + _outer(k[t], v[t])
        if t in record:
            kept[t] = S.copy()
    return o, S, kept


def eager(op, S0, inp, u=None, record=()):
    """Dispatch on ``op`` with the dict layout of ``synthetic.step_inputs``."""
    if op == "gdn":
        return gdn_eager(S0, inp["q"], inp["k"], inp["v"], inp["log_decay"], inp["beta"], record)
    if op == "kda":
        return kda_eager(S0, inp["q"], inp["k"], inp["v"], inp["log_decay"], inp["beta"], record)
    if op == "rwkv6":
        return rwkv6_eager(S0, u, inp["r"], inp["k"], inp["v"], inp["log_decay"], record)
    raise ValueError(op)


def deferred(op, M, S0, inp, u=None, record_merges=True):
    """The DeltaLog schedule in fp64: dense base + bounded log.

    Per unit, ``Lam`` is the cumulative natural-log decay since the last merge
    (a per-key vector; GDN's scalar is broadcast over the keys, which is the
    same operator).  The log holds at most M-1 entries ``(a_i, b_i, Lam_i)``
    with ``a_i = k_i``; ``b_i`` is the delta-corrected value (GDN/KDA) or the
    raw value ``v_i`` (RWKV6); ``Lam_i`` is the snapshot after step i's decay.
    The logical state after step t is
        S_t = diag(e^{Lam_t}) Sbar + sum_i diag(e^{Lam_t - Lam_i}) a_i b_i^T.
    Steps with n+1 < M append; the step with n+1 == M folds the log (and its
    own entry) into the base and empties the log.

    Returns ``(o[T,...,d_v], logical S_T, {t: Sbar after the merge at t})``.
    """
    if M < 1:
        raise ValueError("M must be >= 1")
    Sbar = _f64(S0).copy()
    d_k = Sbar.shape[-2]
    qr = _f64(inp["r"] if op == "rwkv6" else inp["q"])
    k, v, ld = _f64(inp["k"]), _f64(inp["v"]), _f64(inp["log_decay"])
    be = _f64(inp["beta"]) if op != "rwkv6" else None
    uu = _f64(u) if op == "rwkv6" else None
    T = qr.shape[0]
    units = Sbar.shape[:-2]
    o = np.empty(qr.shape[:-1] + (Sbar.shape[-1],))
    log = []                      # list of (a_i, b_i, Lam_i), oldest first
    merges = {}
    for t in range(T):
        # a1: decay bookkeeping (per-key vector form)
        step_ld = ld[t][..., None] * np.ones(d_k) if op == "gdn" else ld[t]
        lam_prev = log[-1][2] if log else np.zeros(units + (d_k,))
        lam_t = lam_prev + step_ld
        if op == "rwkv6":
            # output from S_{t-1} (+ bonus): base scaled by e^{Lam_{t-1}}
            s = _stateT_dot(Sbar, np.exp(lam_prev) * qr[t])
            for a_i, b_i, lam_i in log:
                c = np.sum(np.exp(lam_prev - lam_i) * a_i * qr[t], axis=-1)
                s = s + c[..., None] * b_i
            kappa = np.sum(uu * k[t] * qr[t], axis=-1)
            b_t = v[t]
            o[t] = s + kappa[..., None] * b_t
        else:
            # a3/a4: (decayed S_{t-1})^T k_t from base + replayed log
            p = _stateT_dot(Sbar, np.exp(lam_t) * k[t])
            s = _stateT_dot(Sbar, np.exp(lam_t) * qr[t])
            for a_i, b_i, lam_i in log:
                ratio = np.exp(lam_t - lam_i)
                p = p + np.sum(ratio * a_i * k[t], axis=-1)[..., None] * b_i
                s = s + np.sum(ratio * a_i * qr[t], axis=-1)[..., None] * b_i
            b_t = be[t][..., None] * (v[t] - p)
            # a5: o_t = S_t^T q_t, with S_t's newest term k_t b_t^T
            kappa = np.sum(k[t] * qr[t], axis=-1)
            o[t] = s + kappa[..., None] * b_t
        entry = (k[t], b_t, lam_t)
        if len(log) + 1 < M:
            log.append(entry)                                   # a6: append
        else:
            # a7: merge -- materialise base + every entry (this one included)
            new = np.exp(lam_t)[..., :, None] * Sbar
            for a_i, b_i, lam_i in log + [entry]:
                new = new + _outer(np.exp(lam_t - lam_i) * a_i, b_i)
            Sbar = new
            log = []
            if record_merges:
                merges[t] = Sbar.copy()
    # logical state at the end (base + whatever is still in the log)
    if log:
        lam_last = log[-1][2]
        S_end = np.exp(lam_last)[..., :, None] * Sbar
        for a_i, b_i, lam_i in log:
            S_end = S_end + _outer(np.exp(lam_last - lam_i) * a_i, b_i)
    else:
        S_end = Sbar.copy()
    return o, S_end, merges
