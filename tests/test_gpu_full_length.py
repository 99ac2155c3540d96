"""GPU parity over the whole sequence of every decode workload, at full size.

Each case launches the workload's full batch (every slot and head) for its
whole token count, through the C ABI, and checks sampled (slot, head) units
element by element against the fp64 oracle: every output o_t, the state at
every merge step (every 32 tokens for the eager kernel and M = 1), and the
final logical state.  Several merge intervals and the eager kernel run side
by side on the same token stream.

Inputs.  The checked units (24 sampled units plus the first and the last)
receive the seeded draws of ``synthetic`` (a batch of one head per checked
unit), which the oracle consumes as well.  Every other unit receives draws
from the same distributions made on the device by a seeded torch generator:
units are independent (each owns its state, log and inputs), so those values
cannot reach a checked unit, and drawing the full batch on the host would take
hours (3.6 s per token for KDA at B = 1024).  Tolerances: max relative error
5e-3 per tensor for bf16 inputs.
"""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

from _parity import TOL, relerr, run_oracle
from synthetic import bonus, initial_state, sequence

pytestmark = pytest.mark.gpu

BF16 = torch.bfloat16


def _device_draws(gen, op, B, H, d):
    """One token's inputs for all B x H units, drawn on the device with the
    workload's distributions (q, k L2-normalised for GDN/KDA; log-decays
    -softplus(N(0,1)) or -exp(N(-0.5, 0.5)); beta = sigmoid(N(0,1)))."""
    def n(*shape):
        return torch.randn(shape, generator=gen, device="cuda", dtype=torch.float32)
    if op == "rwkv6":
        return {"r": n(B, H, d).to(BF16), "k": n(B, H, d).to(BF16), "v": n(B, H, d).to(BF16),
                "log_decay": -torch.exp(n(B, H, d) * 0.5 - 0.5)}
    q = F.normalize(n(B, H, d), dim=-1, eps=1e-12)
    k = F.normalize(n(B, H, d), dim=-1, eps=1e-12)
    g = n(B, H) if op == "gdn" else n(B, H, d)
    return {"q": q.to(BF16), "k": k.to(BF16), "v": n(B, H, d).to(BF16),
            "log_decay": -F.softplus(g), "beta": torch.sigmoid(n(B, H))}


def _full_length(op, B, H, d, T, variants, n_units=24, seed=0):
    """Run every variant ("eager", a merge interval M, or (M, "lam_f16") for
    fp16 per-key log-gates) over T tokens of the full batch; compare the
    sampled units' outputs and states with the oracle's."""
    from recurrent_state_update_deltalog_b200 import DeltaLog
    rng = np.random.default_rng(1234)
    flat = np.unique(np.concatenate([rng.choice(B * H, size=n_units, replace=False), [0, B * H - 1]]))
    bs, hs = flat // H, flat % H
    n = flat.size
    bi = torch.from_numpy(bs).cuda()
    hi = torch.from_numpy(hs).cuda()
    slots = sorted(set(bs.tolist()))
    pos = {b: j for j, b in enumerate(slots)}
    pick_slot = torch.tensor([pos[b] for b in bs.tolist()], device="cuda")

    # checked units: seeded host draws, one head per unit
    S0_s = initial_state(seed, n, 1, d, d)[:, 0]
    seq_s = {k: np.ascontiguousarray(v[:, :, 0]) for k, v in sequence(seed, op, n, 1, d, d, T, bf16=True).items()}
    u = bonus(seed, H, d) if op == "rwkv6" else None
    dev_s = {k: torch.from_numpy(v).to("cuda", BF16 if k in ("q", "r", "k", "v") else torch.float32)
             for k, v in seq_s.items()}

    gen = torch.Generator(device="cuda")
    gen.manual_seed(seed + 7)
    S0 = torch.randn((B, H, d, d), generator=gen, device="cuda") * 0.02
    S0[bi, hi] = torch.from_numpy(S0_s).cuda()

    def interval(v):
        return 1 if v == "eager" else v[0] if isinstance(v, tuple) else v

    def record_steps(v):
        every = 32 if interval(v) == 1 else interval(v)
        return [t for t in range(T) if (t + 1) % every == 0]

    handles, outs, states = {}, {}, {}
    for v in variants:
        h = DeltaLog(B, H, d, d, interval(v), op=op, dtype=BF16)
        if isinstance(v, tuple) and "lam_f16" in v:
            h.set_log_lam_f16(True)
        h.load_state(S0)
        if u is not None:
            h.set_bonus(torch.from_numpy(u).cuda())
        handles[v] = h
        outs[v] = torch.empty((T, n, d), dtype=BF16, device="cuda")
        states[v] = {}
    rec = {v: set(record_steps(v)) for v in variants}
    o_buf = torch.empty((B, H, d), dtype=BF16, device="cuda")
    s_buf = torch.empty((len(slots), H, d, d), dtype=torch.float32, device="cuda")

    def sampled_states(h):
        for j, b in enumerate(slots):
            h.slot_read(b, out=s_buf[j])
        return s_buf[pick_slot, hi].clone()

    first = "r" if op == "rwkv6" else "q"
    try:
        for t in range(T):
            x = _device_draws(gen, op, B, H, d)
            for key in x:
                x[key][bi, hi] = dev_s[key][t]
            args = (x[first], x["k"], x["v"], x["log_decay"], x.get("beta"))
            for v, h in handles.items():
                (h.eager_step if v == "eager" else h.step)(*args, out=o_buf)
                outs[v][t] = o_buf[bi, hi]
                if t in rec[v]:
                    states[v][t] = sampled_states(h)
        final = {v: sampled_states(h) for v, h in handles.items()}
        for h in handles.values():
            h.check_device()
    finally:
        for h in handles.values():
            h.close()

    all_rec = set().union(*rec.values())
    o_ref, S_ref, kept = run_oracle(op, S0_s, seq_s, u[hs] if u is not None else None, record=all_rec)
    tol = TOL[BF16]
    for v in variants:
        e_o = relerr(outs[v].float().cpu().numpy(), o_ref)
        assert e_o < tol, f"{op} {v}: outputs {e_o:.3e}"
        for t, s in states[v].items():
            e = relerr(s.cpu().numpy(), kept[t])
            assert e < tol, f"{op} {v}: state after token {t}: {e:.3e}"
        e_s = relerr(final[v].cpu().numpy(), S_ref)
        assert e_s < tol, f"{op} {v}: final state {e_s:.3e}"


def test_gdn_b256_h32_d128_256_tokens():
    """GDN decode at large batch: every merge interval of the workload, and the eager kernel."""
    _full_length("gdn", 256, 32, 128, 256, ["eager", 1, 4, 8, 16])


def test_kda_b128_h32_d128_256_tokens():
    _full_length("kda", 128, 32, 128, 256, ["eager", 8, (8, "lam_f16")])


def test_rwkv6_b128_h64_d64_256_tokens():
    _full_length("rwkv6", 128, 64, 64, 256, ["eager", 8, (8, "lam_f16")])


@pytest.mark.parametrize("op", ["gdn", "kda"])
def test_b1024_h32_d128_512_tokens(op):
    """The largest point of the B x M sweep: 2.15 GB of state per handle, 65,536 CTAs a launch."""
    _full_length(op, 1024, 32, 128, 512, ["eager", 8, 32] + ([(32, "lam_f16")] if op == "kda" else []))
