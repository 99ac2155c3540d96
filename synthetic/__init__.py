"""Seeded synthetic decode workloads for GDN, KDA and RWKV6.

This module only draws random inputs. It holds none of the DeltaLog method's
arithmetic (no recurrence, no log, no decay products): both the CUDA library's
tests/benchmark and the CPU oracle consume exactly the arrays made here.

Distributions follow the workload recipe of the DeltaLog paper's evaluation
as restated for this library (DeltaLog: Deferred Materialization of Recurrent
States for Linear Attention Decoding, "Operators" of the kernel section: GDN
head-wise scalar decay with delta rule, KDA per-key decay with delta rule,
RWKV6 per-key decay with raw value update):

* initial state ``S0 ~ N(0, 0.02)`` (0.02 is the standard deviation), fp32;
* GDN / KDA: ``q, k ~ N(0, 1)`` L2-normalised over ``d_k`` in fp32, then cast
  to the input dtype; ``v ~ N(0, 1)``; decay gate ``g ~ N(0, 1)`` (one per
  head for GDN, one per key for KDA) turned into ``log alpha = -softplus(g)``
  in fp64 and rounded to fp32; ``beta = sigmoid(N(0, 1))`` per head, fp32;
* RWKV6: ``r, k, v ~ N(0, 1)`` (not normalised); ``x ~ N(-0.5, 0.5)`` per key
  and ``log w = -exp(x)`` in fp64 rounded to fp32; bonus ``u ~ N(0, 0.1)`` of
  shape ``[H, d_k]``, fp32.

Gates are handed over as fp32 log-decays (never rounded to bf16); q/k/v/r are
rounded to bf16 (round to nearest even) when the input dtype is bf16, and the
bf16-rounded values are what both sides consume (returned here as float32
arrays that hold bf16-exact values).

Reproducibility scheme: every tensor is cut into fixed chunks and each chunk
draws from its own ``numpy.random.SeedSequence([seed, tag, index])`` stream,
so a chunk is the same whichever thread makes it or whichever subset of slots
or steps a caller asks for.  Chunks: the initial state per slot ``b``; all
per-step inputs per step ``t`` (drawn in the order q|r, k, v, gate, beta).
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

GDN, KDA, RWKV6 = "gdn", "kda", "rwkv6"
OPS = (GDN, KDA, RWKV6)

_TAG_STATE = 1
_TAG_STEP = 2
_TAG_BONUS = 3


def _rng(seed: int, tag: int, index: int = 0) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, tag, index])))


def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bfloat16 (ties to even); float32 out."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = ((u >> 16) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + bias) & np.uint32(0xFFFF0000)).view(np.float32)


def _l2_normalise(x: np.ndarray) -> np.ndarray:
    n = np.sqrt(np.sum(x * x, axis=-1, keepdims=True, dtype=np.float32))
    return (x / np.maximum(n, np.float32(1e-12))).astype(np.float32)


def _softplus64(g: np.ndarray) -> np.ndarray:
    g = g.astype(np.float64)
    return np.maximum(g, 0.0) + np.log1p(np.exp(-np.abs(g)))


def _threads() -> int:
    return max(1, min(16, os.cpu_count() or 1))


def initial_state(seed: int, B: int, H: int, d_k: int, d_v: int, slots=None) -> np.ndarray:
    """``S0[len(slots), H, d_k, d_v]`` float32 ~ N(0, 0.02); default all B slots."""
    slots = list(range(B)) if slots is None else list(slots)
    out = np.empty((len(slots), H, d_k, d_v), dtype=np.float32)

    def fill(j):
        r = _rng(seed, _TAG_STATE, slots[j])
        out[j] = r.standard_normal((H, d_k, d_v), dtype=np.float32) * np.float32(0.02)

    with ThreadPoolExecutor(_threads()) as ex:
        list(ex.map(fill, range(len(slots))))
    return out


def bonus(seed: int, H: int, d_k: int) -> np.ndarray:
    """RWKV6 bonus ``u[H, d_k]`` float32 ~ N(0, 0.1)."""
    return (_rng(seed, _TAG_BONUS).standard_normal((H, d_k), dtype=np.float32)
            * np.float32(0.1))


def step_inputs(seed: int, op: str, B: int, H: int, d_k: int, d_v: int, t: int,
                bf16: bool) -> dict:
    """Inputs of decode step ``t`` for all B slots and H heads.

    Returns float32 arrays: ``q`` (``r`` for RWKV6) and ``k`` of shape
    ``[B, H, d_k]``, ``v`` ``[B, H, d_v]``, ``log_decay`` (``[B, H]`` for GDN,
    ``[B, H, d_k]`` for KDA/RWKV6) and ``beta`` ``[B, H]`` (GDN/KDA only).
    """
    if op not in OPS:
        raise ValueError(f"unknown op {op!r}")
    r = _rng(seed, _TAG_STEP, t)
    f32 = np.float32
    a = r.standard_normal((B, H, d_k), dtype=f32)
    k = r.standard_normal((B, H, d_k), dtype=f32)
    v = r.standard_normal((B, H, d_v), dtype=f32)
    cast = round_to_bf16 if bf16 else (lambda x: x.astype(f32))
    out = {}
    if op == RWKV6:
        x = r.standard_normal((B, H, d_k), dtype=f32) * f32(0.5) - f32(0.5)
        out["r"] = cast(a)
        out["k"] = cast(k)
        out["v"] = cast(v)
        out["log_decay"] = (-np.exp(x.astype(np.float64))).astype(f32)
        return out
    gshape = (B, H) if op == GDN else (B, H, d_k)
    g = r.standard_normal(gshape, dtype=f32)
    braw = r.standard_normal((B, H), dtype=f32)
    out["q"] = cast(_l2_normalise(a))
    out["k"] = cast(_l2_normalise(k))
    out["v"] = cast(v)
    out["log_decay"] = (-_softplus64(g)).astype(f32)
    out["beta"] = (1.0 / (1.0 + np.exp(-braw.astype(np.float64)))).astype(f32)
    return out


def sequence(seed: int, op: str, B: int, H: int, d_k: int, d_v: int, T: int,
             bf16: bool, t0: int = 0) -> dict:
    """Steps ``t0 .. t0+T-1`` stacked on a leading time axis ``[T, ...]``."""
    steps = [None] * T

    def fill(j):
        steps[j] = step_inputs(seed, op, B, H, d_k, d_v, t0 + j, bf16)

    with ThreadPoolExecutor(_threads()) as ex:
        list(ex.map(fill, range(T)))
    return {key: np.stack([s[key] for s in steps]) for key in steps[0]}
