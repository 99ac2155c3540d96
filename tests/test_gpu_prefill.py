"""Prefill -> decode hand-off (dl_prefill) against the fp64 oracle.

Packed prompts of ragged lengths (0, 1, and several tiles of tokens) run on
pool slots given by an index map; every token's output and each slot's
final state must match the eager recurrence from the prompt's initial state,
and decoding must continue from the handed-off state across merges.
"""
import numpy as np
import pytest
import torch

from _parity import TOL, make_inputs, relerr, run_oracle, step_args, to_device
from synthetic import initial_state, sequence

pytestmark = pytest.mark.gpu

OPS = ["gdn", "kda", "rwkv6"]


def _pack(seq, lens):
    """Rows of a [T, R, H, ...] sequence packed token-major: row r's first
    lens[r] tokens, rows one after another."""
    out = {}
    for key, arr in seq.items():
        out[key] = np.concatenate([arr[:n, r] for r, n in enumerate(lens)], axis=0)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    return out, cu


def _device_packed(packed, dtype):
    return {key: torch.from_numpy(np.ascontiguousarray(a)).to(
        device="cuda", dtype=dtype if key in ("q", "r", "k", "v") else torch.float32)
        for key, a in packed.items()}


def _prefill_args(op, d):
    first = d["r"] if op == "rwkv6" else d["q"]
    return first, d["k"], d["v"], d["log_decay"], (None if op == "rwkv6" else d["beta"])


def _oracle_row(op, S_init, seq, r, n, u):
    """Eager oracle of row r over its first n tokens from state S_init [H, dk, dv]."""
    one = {key: val[:n, r:r + 1] for key, val in seq.items()}
    if n == 0:
        return np.zeros((0, 1) + seq["v"].shape[2:]), S_init[None].astype(np.float64)
    o, S, _ = run_oracle(op, S_init[None], one, u)
    return o, S


# the chunked kernels serve bf16-input handles only (their refusal for fp32
# inputs is tested below)
_KERNELS = [(op, dt, k) for op in OPS for dt in (torch.bfloat16, torch.float32)
            for k in ("auto", "recurrent", "chunked") if k != "chunked" or dt == torch.bfloat16]


@pytest.mark.parametrize("op,dtype,kernel", _KERNELS)
@pytest.mark.parametrize("dims", [(64, 64), (128, 128), (64, 128), (128, 64)])
def test_prefill_then_decode(op, dims, dtype, kernel):
    """Prompts of 37, 0, 1, 130 (several chunks and a ragged tail) and 5 tokens."""
    _prefill_then_decode(op, dims, dtype, kernel, H=3)


@pytest.mark.parametrize("op", OPS)
def test_prefill_then_decode_many_heads(op):
    """The same with 5 rows x 16 heads at d_k = d_v = 128 (80 whole-head CTAs
    of the tensor-memory kernels)."""
    _prefill_then_decode(op, (128, 128), torch.bfloat16, "chunked", H=16)


def _prefill_then_decode(op, dims, dtype, kernel, H, log_lam_f16=False):
    from recurrent_state_update_deltalog_b200 import DeltaLog
    dk, dv = dims
    B, M, T_dec = 8, 4, 7
    lens = [37, 0, 1, 130, 5]
    slots = [6, 0, 3, 1, 4]
    rows = len(lens)
    bf16 = dtype == torch.bfloat16
    seq = sequence(21, op, rows, H, dk, dv, max(lens), bf16=bf16)
    u = make_inputs(op, 1, H, dk, dv, 1, dtype, seed=21)[2]
    packed, cu = _pack(seq, lens)
    tol = TOL[dtype]

    S_pool = initial_state(5, B, H, dk, dv)             # other slots keep this
    h = DeltaLog(B, H, dk, dv, M, op=op, dtype=dtype)
    h.set_prefill_kernel(kernel)
    h.set_log_lam_f16(log_lam_f16)
    h.load_state(torch.from_numpy(S_pool).cuda())
    if u is not None:
        h.set_bonus(torch.from_numpy(u).cuda())
    # two decode tokens first, so that the log holds entries at the hand-off
    warm = make_inputs(op, B, H, dk, dv, 2, dtype, seed=22)[1]
    dwarm = to_device(warm, dtype)
    for t in range(2):
        h.step(*step_args(op, dwarm, t))
    _, S_ref, _ = run_oracle(op, S_pool, warm, u)

    d = _device_packed(packed, dtype)
    o = h.prefill(*_prefill_args(op, d), cu_seqlens=torch.from_numpy(cu).cuda(),
                  slot_idx=torch.tensor(slots, dtype=torch.int32, device="cuda"), zero_state=True)
    assert h.log_len == 2                                # the handle's cycle is unchanged
    big = (dk, dv) == (128, 128)   # the automatic rule
    min_avg = 16 if big else 32
    auto_chunked = dtype == torch.bfloat16 and sum(lens) >= min_avg * rows
    want = "chunked" if kernel == "chunked" or (kernel == "auto" and auto_chunked) else "recurrent"
    assert h.last_prefill_kernel == want
    got = o.float().cpu().numpy()
    zero = np.zeros((H, dk, dv))
    for r, (n, b) in enumerate(zip(lens, slots)):
        o_r, S_r = _oracle_row(op, zero, seq, r, n, u)
        if n:
            assert relerr(got[cu[r]:cu[r + 1]], o_r[:, 0]) < tol, r
        S_ref[b] = S_r[0]
        assert relerr(h.slot_read(b).cpu().numpy(), S_ref[b]) < tol, (r, b)
    for b in (2, 5, 7):                                  # slots not named are untouched
        assert relerr(h.slot_read(b).cpu().numpy(), S_ref[b]) < tol, b

    # decode continues from the handed-off states, across a merge
    dec = make_inputs(op, B, H, dk, dv, T_dec, dtype, seed=23)[1]
    ddec = to_device(dec, dtype)
    outs = [h.step(*step_args(op, ddec, t)).float().cpu().numpy() for t in range(T_dec)]
    o_ref, S_fin, _ = run_oracle(op, S_ref, dec, u)
    assert relerr(np.stack(outs), o_ref) < tol
    assert relerr(h.read_state().cpu().numpy(), S_fin) < tol
    h.check_device()
    h.close()


@pytest.mark.parametrize("op,kernel", [(op, k) for op in OPS for k in ("auto", "recurrent", "chunked")])
def test_prefill_continues_logical_state(op, kernel):
    """Without DL_PREFILL_ZERO_STATE a prompt continues from the slot's
    logical state (base + log), e.g. the second chunk of a long prompt."""
    _prefill_continues(op, kernel)


@pytest.mark.parametrize("op", ["kda", "rwkv6"])
@pytest.mark.parametrize("kernel", ["recurrent", "chunked"])
def test_prefill_with_f16_log_gates(op, kernel):
    """The hand-off folds (continued prompts) and clears (new prompts) a log
    whose per-key snapshots are fp16 log-gates."""
    _prefill_continues(op, kernel, log_lam_f16=True)
    _prefill_then_decode(op, (128, 128), torch.bfloat16, kernel, H=3, log_lam_f16=True)


def _prefill_continues(op, kernel, log_lam_f16=False):
    from recurrent_state_update_deltalog_b200 import DeltaLog
    dtype, dk, dv, B, H, M = torch.bfloat16, 128, 128, 4, 2, 8
    S0, warm, u = make_inputs(op, B, H, dk, dv, 5, dtype, seed=31)
    h = DeltaLog(B, H, dk, dv, M, op=op, dtype=dtype)
    h.set_prefill_kernel(kernel)
    h.set_log_lam_f16(log_lam_f16)
    h.load_state(torch.from_numpy(S0).cuda())
    if u is not None:
        h.set_bonus(torch.from_numpy(u).cuda())
    dwarm = to_device(warm, dtype)
    for t in range(5):
        h.step(*step_args(op, dwarm, t))
    _, S_ref, _ = run_oracle(op, S0, warm, u)
    lens = [20, 97, 0, 9]
    seq = sequence(32, op, B, H, dk, dv, max(lens), bf16=True)
    packed, cu = _pack(seq, lens)
    d = _device_packed(packed, dtype)
    o = h.prefill(*_prefill_args(op, d), cu_seqlens=torch.from_numpy(cu).cuda())   # row r = slot r
    got = o.float().cpu().numpy()
    for r, n in enumerate(lens):
        o_r, S_r = _oracle_row(op, S_ref[r], seq, r, n, u)
        if n:
            assert relerr(got[cu[r]:cu[r + 1]], o_r[:, 0]) < TOL[dtype], r
        assert relerr(h.slot_read(r).cpu().numpy(), S_r[0]) < TOL[dtype], r
    h.check_device()
    h.close()


def test_prefill_bad_seqlen_raises_device_flag():
    from recurrent_state_update_deltalog_b200 import DeltaLog, DeltaLogError
    op, dtype, d, B, H = "gdn", torch.float32, 64, 3, 2
    lens = [4, 6, 3]
    seq = sequence(41, op, B, H, d, d, 6, bf16=False)
    packed, cu = _pack(seq, lens)
    bad = cu.copy()
    bad[2] = 99                                          # row 1 ends past the batch, row 2 starts there
    h = DeltaLog(B, H, d, d, 4, op=op, dtype=dtype)
    dd = _device_packed(packed, dtype)
    o = torch.zeros((int(cu[-1]), H, d), device="cuda")
    h.prefill(*_prefill_args(op, dd), cu_seqlens=torch.from_numpy(bad).cuda(), zero_state=True, out=o)
    with pytest.raises(DeltaLogError, match="0x4"):
        h.check_device()
    o_r, S_r = _oracle_row(op, np.zeros((H, d, d)), seq, 0, 4, None)
    assert relerr(o[:4].cpu().numpy(), o_r[:, 0]) < TOL[dtype]          # row 0 ran
    assert np.all(o[4:].cpu().numpy() == 0)                              # rows 1 and 2 skipped
    h.close()


def test_prefill_arguments():
    from recurrent_state_update_deltalog_b200 import DeltaLog, DeltaLogError
    h = DeltaLog(2, 2, 64, 64, 4, op="gdn", dtype=torch.float32)
    e3 = torch.empty((0, 2, 64), device="cuda")
    e2 = torch.empty((0, 2), device="cuda")
    cu = torch.zeros(3, dtype=torch.int32, device="cuda")
    h.prefill(e3, e3, e3, e2, e2, cu_seqlens=cu, zero_state=True)      # two empty prompts
    assert np.all(h.read_state().cpu().numpy() == 0)
    with pytest.raises(ValueError):
        h.prefill(e3, e3, e3, e2, e2, cu_seqlens=torch.zeros(4, dtype=torch.int32, device="cuda"))
    h.close()


@pytest.mark.parametrize("op,H,d,kernel", [(op, H, d, k) for op, H, d in (("gdn", 32, 128), ("kda", 32, 128),
                                                                         ("rwkv6", 64, 64))
                                           for k in ("chunked", "recurrent")])
def test_prefill_full_size_sampled(op, H, d, kernel):
    """The launch bench.py --prefill times (B = 64 prompts of L = 512 tokens,
    every row from zero): two sampled rows checked token by token, with their
    final states, against the oracle."""
    from recurrent_state_update_deltalog_b200 import DeltaLog
    from synthetic import bonus
    B, L, dtype = 64, 512, torch.bfloat16
    seq = sequence(0, op, B, H, d, d, L, bf16=True)
    u = bonus(0, H, d) if op == "rwkv6" else None
    packed, cu = _pack(seq, [L] * B)
    dev = _device_packed(packed, dtype)
    del packed
    h = DeltaLog(B, H, d, d, 8, op=op, dtype=dtype)
    h.set_prefill_kernel(kernel)
    if u is not None:
        h.set_bonus(torch.from_numpy(u).cuda())
    o = h.prefill(*_prefill_args(op, dev), cu_seqlens=torch.from_numpy(cu).cuda(), zero_state=True)
    zero = np.zeros((H, d, d))
    for r in (0, 37):
        o_r, S_r = _oracle_row(op, zero, seq, r, L, u)
        assert relerr(o[r * L:(r + 1) * L].float().cpu().numpy(), o_r[:, 0]) < TOL[dtype], r
        assert relerr(h.slot_read(r).cpu().numpy(), S_r[0]) < TOL[dtype], r
    h.check_device()
    h.close()


def test_chunked_prefill_refused_where_it_does_not_apply():
    """The chunked kernels serve bf16-input handles only."""
    from recurrent_state_update_deltalog_b200 import DeltaLog, DeltaLogError
    for op, dtype in (("gdn", torch.float32), ("kda", torch.float32), ("rwkv6", torch.float32)):
        h = DeltaLog(2, 2, 64, 64, 4, op=op, dtype=dtype)
        h.set_prefill_kernel("chunked")
        x = torch.zeros((3, 2, 64), device="cuda", dtype=dtype)
        g = torch.zeros((3, 2) if op == "gdn" else (3, 2, 64), device="cuda")
        b = None if op == "rwkv6" else torch.zeros((3, 2), device="cuda")
        cu = torch.tensor([0, 3, 3], dtype=torch.int32, device="cuda")
        with pytest.raises(DeltaLogError):
            h.prefill(x, x, x, g, b, cu_seqlens=cu, zero_state=True)
        h.close()


@pytest.mark.parametrize("op,kernel", [(op, k) for op in OPS for k in ("recurrent", "chunked")])
@pytest.mark.parametrize("d,H", [(64, 2), (128, 2), (128, 48), (128, 96), (64, 80)])
def test_prefill_strong_decay(op, kernel, d, H):
    """Log-decays of -40 per token (on three keys for KDA/RWKV6, on every
    tenth token for GDN): cumulative decays far past fp32 range inside a
    chunk, which no kernel may divide by.  Two rows of H = 96 or 80 heads
    launch more CTAs than the GPU has SMs, so the chunked kernels run their
    256-thread variant (for KDA and RWKV6, with both levels of pair blocks);
    the smaller cases run the 512-thread one."""
    from recurrent_state_update_deltalog_b200 import DeltaLog
    dtype, lens = torch.bfloat16, [100, 37]
    rows = len(lens)
    seq = sequence(51, op, rows, H, d, d, max(lens), bf16=True)
    seq["log_decay"] = seq["log_decay"].copy()
    if op == "gdn":
        seq["log_decay"][::10] = -40.0
    else:
        seq["log_decay"][..., :3] = -40.0
    u = make_inputs(op, 1, H, d, d, 1, dtype, seed=51)[2]
    packed, cu = _pack(seq, lens)
    h = DeltaLog(rows, H, d, d, 4, op=op, dtype=dtype)
    h.set_prefill_kernel(kernel)
    if u is not None:
        h.set_bonus(torch.from_numpy(u).cuda())
    o = h.prefill(*_prefill_args(op, _device_packed(packed, dtype)), cu_seqlens=torch.from_numpy(cu).cuda(),
                  zero_state=True)
    got = o.float().cpu().numpy()
    assert np.all(np.isfinite(got))
    zero = np.zeros((H, d, d))
    for r, n in enumerate(lens):
        o_r, S_r = _oracle_row(op, zero, seq, r, n, u)
        assert relerr(got[cu[r]:cu[r + 1]], o_r[:, 0]) < TOL[dtype], r
        assert relerr(h.slot_read(r).cpu().numpy(), S_r[0]) < TOL[dtype], r
    h.check_device()
    h.close()
