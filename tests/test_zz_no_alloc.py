"""dl_decode_static, the allocation-free decode call, against the handle API.

Some callers cannot allocate device memory: a plugin inside an inference
engine that hands out all device memory from its own pool, a process with a
fixed device memory budget, or a loop that cannot take an allocation's
implicit synchronisation.  They cannot create a handle, so dl_decode_static
decodes on a dense state they own and keeps the log in one fixed device array
of the library.  Here it runs twice in a row through the C ABI: the second
call starts from the first call's state and finds the first call's log still
in the array.  Outputs and states must match a handle loaded with the same
state that runs the same dl_step calls and then dl_merge, within the parity
tolerances (5e-3 for bf16 inputs, 1e-4 for fp32).  This file is named so that
pytest collects it last.
"""
import ctypes

import pytest
import torch

from _parity import TOL, make_inputs, relerr, step_args, to_device

pytestmark = pytest.mark.gpu

OPS = {"gdn": 0, "kda": 1, "rwkv6": 2}


def _p(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p()


def _decode_static(op, S, u, dseq, t0, t1, M, dtype, err):
    """One dl_decode_static call over tokens [t0, t1); returns o [T, B, H, d_v]."""
    from recurrent_state_update_deltalog_b200 import _native as N
    B, H, dk, dv = S.shape
    first = "r" if op == "rwkv6" else "q"
    x = {k: v[t0:t1].contiguous() for k, v in dseq.items()}
    o = torch.empty((t1 - t0, B, H, dv), dtype=dtype, device="cuda")
    N.call("dl_decode_static", OPS[op], B, H, dk, dv, M, 1 if dtype == torch.bfloat16 else 0, _p(S), _p(u),
           t1 - t0, _p(x[first]), _p(x["k"]), _p(x["v"]), _p(x["log_decay"]), _p(x.get("beta")), _p(o),
           _p(err), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return o


def _handle_run(op, S0, u, dseq, bounds, M, dtype):
    """The same tokens through dl_create / dl_step / dl_merge / dl_read_state."""
    from recurrent_state_update_deltalog_b200 import DeltaLog
    B, H, dk, dv = S0.shape
    h = DeltaLog(B, H, dk, dv, M, op=op, dtype=dtype)
    try:
        h.load_state(S0)
        if u is not None:
            h.set_bonus(u)
        res = []
        for t0, t1 in bounds:
            o = torch.stack([h.step(*step_args(op, dseq, t)) for t in range(t0, t1)])
            h.merge()
            res.append((o, h.read_state()))
        h.check_device()
        return res
    finally:
        h.close()


@pytest.mark.parametrize("op,dims,M,dtype", [
    ("gdn", (128, 128), 4, torch.bfloat16),
    ("kda", (128, 128), 8, torch.bfloat16),
    ("rwkv6", (64, 64), 4, torch.bfloat16),
    ("gdn", (64, 128), 3, torch.float32),
    ("kda", (128, 64), 1, torch.float32),
])
def test_decode_static_matches_handle_on_two_calls(op, dims, M, dtype):
    B, H = 37, 8          # 296 units: the value-tile split of two CTAs a head applies
    dk, dv = dims
    T1, T2 = 11, 6        # the first call ends mid-cycle (its log is folded at the end)
    S0_np, seq, u_np = make_inputs(op, B, H, dk, dv, T1 + T2, dtype, seed=5)
    dseq = to_device(seq, dtype)
    S0 = torch.from_numpy(S0_np).cuda()
    u = torch.from_numpy(u_np).cuda() if u_np is not None else None

    ref = _handle_run(op, S0, u, dseq, [(0, T1), (T1, T1 + T2)], M, dtype)

    S = S0.clone()
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    o1 = _decode_static(op, S, u, dseq, 0, T1, M, dtype, err)
    S1 = S.clone()
    o2 = _decode_static(op, S, u, dseq, T1, T1 + T2, M, dtype, err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    tol = TOL[dtype]
    for (o_ref, s_ref), o, s in zip(ref, (o1, o2), (S1, S)):
        e_o = relerr(o.float().cpu().numpy(), o_ref.float().cpu().numpy())
        e_s = relerr(s.cpu().numpy(), s_ref.cpu().numpy())
        assert e_o < tol and e_s < tol, (e_o, e_s)


def test_decode_static_rejects_requests_beyond_the_array():
    """A log larger than the fixed array is refused before any launch, with the
    size it would need; the caller's state is left as it was."""
    from recurrent_state_update_deltalog_b200 import _native as N
    B, H, d, M = 128, 32, 128, 8          # 4096 units x 5,408 bytes > 16 MiB
    S = torch.zeros((B, H, d, d), device="cuda")
    S[0, 0, 0, 0] = 1.0
    x = torch.zeros((1, B, H, d), dtype=torch.bfloat16, device="cuda")
    g = torch.zeros((1, B, H), device="cuda")
    o = torch.empty((1, B, H, d), dtype=torch.bfloat16, device="cuda")
    lib = N.load()
    st = lib.dl_decode_static(0, B, H, d, d, M, 1, _p(S), None, 1, _p(x), _p(x), _p(x), _p(g), _p(g), _p(o),
                              None, None)
    assert st == -1
    msg = lib.dl_last_error().decode()
    assert "needs" in msg and str(N.DL_STATIC_SCRATCH_BYTES) in msg
    torch.cuda.synchronize()
    assert float(S[0, 0, 0, 0]) == 1.0 and int(torch.count_nonzero(S)) == 1
