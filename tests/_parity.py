"""Shared driver for GPU-vs-oracle parity tests (test infrastructure).

Both sides read the same seeded arrays from ``synthetic``; the GPU side runs
through the C ABI (via the ctypes-backed ``DeltaLog`` handle), the oracle
runs the fp64 eager recurrence on CPU.  Error metric (the paper's "maximum
relative error", read per tensor): max|x - ref| / max|ref|.
"""
from __future__ import annotations

import numpy as np
import torch

from oracle import eager as oracle_eager
from synthetic import bonus, initial_state, sequence

TOL = {torch.bfloat16: 5e-3, torch.float32: 1e-4}


def relerr(x, ref) -> float:
    x = np.asarray(x, np.float64)
    ref = np.asarray(ref, np.float64)
    return float(np.max(np.abs(x - ref)) / max(float(np.max(np.abs(ref))), 1e-30))


def make_inputs(op, B, H, dk, dv, T, dtype, seed=0):
    bf16 = dtype == torch.bfloat16
    S0 = initial_state(seed, B, H, dk, dv)
    seq = sequence(seed, op, B, H, dk, dv, T, bf16=bf16)
    u = bonus(seed, H, dk) if op == "rwkv6" else None
    return S0, seq, u


def to_device(seq, dtype, dev="cuda"):
    """Per-step device tensors: q/r/k/v in the input dtype, gates fp32."""
    out = {}
    for key, arr in seq.items():
        t = torch.from_numpy(np.ascontiguousarray(arr))
        out[key] = t.to(device=dev, dtype=dtype if key in ("q", "r", "k", "v") else torch.float32)
    return out


def step_args(op, dseq, t):
    first = dseq["r"] if op == "rwkv6" else dseq["q"]
    beta = None if op == "rwkv6" else dseq["beta"][t]
    return first[t], dseq["k"][t], dseq["v"][t], dseq["log_decay"][t], beta


def run_gpu(op, S0, seq, u, M, dtype, eager=False, record_merges=True, kernel="auto", tiles=0,
            log_b_bf16=False, log_lam_f16=False):
    """Run T steps through the library; returns (o[T,B,H,dv], {t: Sbar}, final logical S).

    ``kernel`` selects the dl_step kernel ("auto" or "register")."""
    from recurrent_state_update_deltalog_b200 import DeltaLog
    B, H, dk, dv = S0.shape
    T = seq["k"].shape[0]
    dseq = to_device(seq, dtype)
    h = DeltaLog(B, H, dk, dv, M, op=op, dtype=dtype)
    h.set_step_kernel(kernel)
    h.set_value_tiles(tiles)
    if log_b_bf16:
        h.set_log_b_bf16(True)
    if log_lam_f16:
        h.set_log_lam_f16(True)
    try:
        h.load_state(torch.from_numpy(S0).cuda())
        if u is not None:
            h.set_bonus(torch.from_numpy(u).cuda())
        outs = torch.empty((T, B, H, dv), dtype=dtype, device="cuda")
        merges = {}
        for t in range(T):
            args = step_args(op, dseq, t)
            if eager:
                h.eager_step(*args, out=outs[t])
            else:
                h.step(*args, out=outs[t])
                if record_merges and (t + 1) % M == 0:
                    assert h.log_len == 0
                    merges[t] = h.read_state().cpu().numpy()
        final = h.read_state().cpu().numpy()
        h.check_device()
        torch.cuda.synchronize()
        return outs.float().cpu().numpy(), merges, final
    finally:
        h.close()


def run_oracle(op, S0, seq, u, record=()):
    return oracle_eager(op, S0, seq, u=u, record=record)
