"""GPU parity: libdeltalog (through the C ABI) against the fp64 oracle.

Tolerances: max relative error 5e-3 for bf16 inputs/outputs and 1e-4 for fp32,
per tensor (all outputs stacked; each merged base; the final logical state).
"""
import numpy as np
import pytest
import torch

from _parity import TOL, make_inputs, relerr, run_gpu, run_oracle, step_args, to_device

pytestmark = pytest.mark.gpu

OPS = ["gdn", "kda", "rwkv6"]


KERNELS = ["auto", "register"]


def _check_run(op, B, H, dk, dv, M, T, dtype, eager=False, seed=0, kernel="auto", tiles=0):
    S0, seq, u = make_inputs(op, B, H, dk, dv, T, dtype, seed)
    merge_steps = [t for t in range(T) if (t + 1) % M == 0] if not eager else []
    o_ref, S_ref, kept = run_oracle(op, S0, seq, u, record=set(merge_steps))
    o, merges, final = run_gpu(op, S0, seq, u, M, dtype, eager=eager, kernel=kernel, tiles=tiles)
    tol = TOL[dtype]
    e_o = relerr(o, o_ref)
    assert e_o < tol, f"outputs: {e_o:.3e}"
    for t in merge_steps:
        e = relerr(merges[t], kept[t])
        assert e < tol, f"merged base at t={t}: {e:.3e}"
    e_s = relerr(final, S_ref)
    assert e_s < tol, f"final state: {e_s:.3e}"
    return e_o, e_s


@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("M", [8, 1])
def test_gdn_single_head_fp32(M, kernel):
    """B=H=1, d=64, fp32 inputs, 64 steps, seed 0."""
    _check_run("gdn", 1, 1, 64, 64, M, 64, torch.float32, kernel=kernel)


@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("op", OPS)
@pytest.mark.parametrize("dims", [(64, 64), (128, 128), (64, 128), (128, 64)])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_deferred_shapes(op, dims, dtype, kernel):
    """Ragged B*H, every shape, M=4 with a tail that ends mid-cycle."""
    _check_run(op, 3, 5, dims[0], dims[1], 4, 11, dtype, kernel=kernel)


@pytest.mark.parametrize("op", OPS)
@pytest.mark.parametrize("M", [1, 2, 3, 8, 16, 32, 33, 64])
def test_deferred_every_M(op, M):
    _check_run(op, 2, 3, 128, 128, M, min(2 * M + 3, 70), torch.bfloat16)


def test_step_kernel_selection_is_reported():
    from recurrent_state_update_deltalog_b200 import DeltaLog, DeltaLogError
    from recurrent_state_update_deltalog_b200 import _native as N
    S0, seq, _ = make_inputs("gdn", 4, 8, 128, 128, 2, torch.bfloat16)
    dseq = to_device(seq, torch.bfloat16)
    h = DeltaLog(4, 8, 128, 128, 8, op="gdn")
    assert h.last_step_kernel is None
    h.step(*step_args("gdn", dseq, 0))
    assert h.last_step_kernel == "register"
    h.set_step_kernel("register")
    h.step(*step_args("gdn", dseq, 1))
    assert h.last_step_kernel == "register"
    with pytest.raises(DeltaLogError) as ei:   # no other step kernel exists
        N.call("dl_set_option", h._h, N.DL_OPT_STEP_KERNEL, 2)
    assert ei.value.status == -1
    h.close()


@pytest.mark.parametrize("tiles", [1, 2, 4])
@pytest.mark.parametrize("op", OPS)
@pytest.mark.parametrize("dims", [(64, 64), (128, 128), (64, 128), (128, 64)])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_value_tiles(op, dims, dtype, tiles):
    """Register-tile kernel with each head's d_v columns split over 1, 2 or 4
    CTAs (a split that would leave fewer than 32 columns falls back to fewer)."""
    _check_run(op, 3, 5, dims[0], dims[1], 4, 11, dtype, kernel="register", tiles=tiles)


@pytest.mark.parametrize("tiles", [2, 4])
@pytest.mark.parametrize("op", OPS)
@pytest.mark.parametrize("M", [2, 8, 33, 64])
def test_value_tiles_every_M(op, M, tiles):
    _check_run(op, 2, 3, 128, 128, M, min(2 * M + 3, 70), torch.bfloat16, kernel="register", tiles=tiles)


@pytest.mark.parametrize("op", OPS)
def test_many_units_per_sm(op):
    """More units than resident CTAs: several waves per launch (B*H = 2000)."""
    _check_run(op, 125, 16, 64, 64, 4, 9, torch.bfloat16)
    _check_run(op, 40, 16, 128, 128, 3, 7, torch.bfloat16)


@pytest.mark.parametrize("op", OPS)
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_eager_kernel(op, dtype):
    _check_run(op, 3, 4, 128, 128, 1, 9, dtype, eager=True)
    _check_run(op, 2, 3, 64, 64, 1, 9, dtype, eager=True)


@pytest.mark.parametrize("op", OPS)
def test_M1_deferred_matches_eager_kernel(op):
    S0, seq, u = make_inputs(op, 4, 4, 128, 128, 10, torch.float32)
    o_d, _, s_d = run_gpu(op, S0, seq, u, 1, torch.float32, record_merges=False)
    o_e, _, s_e = run_gpu(op, S0, seq, u, 1, torch.float32, eager=True)
    assert relerr(o_d, o_e) < 1e-5 and relerr(s_d, s_e) < 1e-5


def _full_size_case(op, B, H, d, M, T, n_units=24, kernel="auto"):
    """Full-size launch; sampled (slot, head) units checked against the oracle."""
    dtype = torch.bfloat16
    S0, seq, u = make_inputs(op, B, H, d, d, T, dtype)
    rng = np.random.default_rng(1234)
    flat = rng.choice(B * H, size=n_units, replace=False)
    flat = np.unique(np.concatenate([flat, [0, B * H - 1]]))
    bs, hs = flat // H, flat % H
    S0_s = S0[bs, hs]
    seq_s = {k: v[:, bs, hs] for k, v in seq.items()}
    u_s = u[hs] if u is not None else None
    merge_steps = [t for t in range(T) if (t + 1) % M == 0]
    o_ref, S_ref, kept = run_oracle(op, S0_s, seq_s, u_s, record=set(merge_steps))
    o, merges, final = run_gpu(op, S0, seq, u, M, dtype, kernel=kernel)
    assert relerr(o[:, bs, hs], o_ref) < TOL[dtype]
    for t in merge_steps:
        assert relerr(merges[t][bs, hs], kept[t]) < TOL[dtype]
    assert relerr(final[bs, hs], S_ref) < TOL[dtype]
    # properties over every unit: finite outputs, untouched dtype range
    assert np.isfinite(o).all() and np.isfinite(final).all()


@pytest.mark.parametrize("M", [8, 4, 16, 1])
def test_full_size_gdn_b256_h32_d128(M):
    _full_size_case("gdn", 256, 32, 128, M, 2 * M + 3 if M > 1 else 6)


def test_full_size_gdn_b256_h32_d128_register_kernel():
    _full_size_case("gdn", 256, 32, 128, 8, 19, kernel="register")


def test_full_size_kda_b128_h32_d128():
    _full_size_case("kda", 128, 32, 128, 8, 19)


def test_full_size_rwkv6_b128_h64_d64():
    _full_size_case("rwkv6", 128, 64, 64, 8, 19)


# ---- handle semantics through the C ABI ---------------------------------------

@pytest.mark.parametrize("op", OPS)
def test_explicit_merge_and_read_state(op):
    """dl_merge mid-cycle, dl_read_state leaves the handle untouched."""
    from recurrent_state_update_deltalog_b200 import DeltaLog
    B, H, d, M, T = 2, 3, 64, 8, 13
    S0, seq, u = make_inputs(op, B, H, d, d, T, torch.float32)
    o_ref, S_ref, kept = run_oracle(op, S0, seq, u, record=set(range(T)))
    dseq = to_device(seq, torch.float32)
    h = DeltaLog(B, H, d, d, M, op=op, dtype=torch.float32)
    h.load_state(torch.from_numpy(S0).cuda())
    if u is not None:
        h.set_bonus(torch.from_numpy(u).cuda())
    outs = []
    for t in range(T):
        outs.append(h.step(*step_args(op, dseq, t)).cpu().numpy())
        s1 = h.read_state().cpu().numpy()
        s2 = h.read_state().cpu().numpy()
        assert np.array_equal(s1, s2)
        assert relerr(s1, kept[t]) < 1e-4, t
        if t == 4:
            assert h.log_len == 5
            h.merge()
            assert h.log_len == 0
            assert relerr(h.read_state().cpu().numpy(), kept[t]) < 1e-4
    assert relerr(np.stack(outs), o_ref) < 1e-4
    h.merge()
    h.merge()                      # no-op on an empty log
    assert relerr(h.read_state().cpu().numpy(), S_ref) < 1e-4
    h.close()


def test_eager_needs_empty_log_and_load_state_resets():
    from recurrent_state_update_deltalog_b200 import DeltaLog, DeltaLogError
    S0, seq, _ = make_inputs("gdn", 1, 2, 64, 64, 3, torch.float32)
    dseq = to_device(seq, torch.float32)
    h = DeltaLog(1, 2, 64, 64, 4, op="gdn", dtype=torch.float32)
    h.load_state(torch.from_numpy(S0).cuda())
    h.step(*step_args("gdn", dseq, 0))
    with pytest.raises(DeltaLogError) as ei:
        h.eager_step(*step_args("gdn", dseq, 1))
    assert ei.value.status == -6
    h.load_state(torch.from_numpy(S0).cuda())
    assert h.log_len == 0
    h.eager_step(*step_args("gdn", dseq, 0))
    with pytest.raises(DeltaLogError):
        DeltaLog(1, 2, 64, 64, 4, op="gdn").set_bonus(torch.zeros(2, 64, device="cuda"))
    h.close()


@pytest.mark.parametrize("prefetch", [False, True])
@pytest.mark.parametrize("op", OPS)
def test_step_host_matches_device_step(op, prefetch):
    from recurrent_state_update_deltalog_b200 import DeltaLog
    B, H, d, M, T = 4, 8, 128, 4, 9
    S0, seq, u = make_inputs(op, B, H, d, d, T, torch.bfloat16)
    dseq = to_device(seq, torch.bfloat16)
    hseq = {k: v.cpu().pin_memory() for k, v in dseq.items()}
    hd = DeltaLog(B, H, d, d, M, op=op)
    hh = DeltaLog(B, H, d, d, M, op=op)
    hh.set_host_prefetch(prefetch)
    for h in (hd, hh):
        h.load_state(torch.from_numpy(S0).cuda())
        if u is not None:
            h.set_bonus(torch.from_numpy(u).cuda())
    ods, ohs = [], []
    for t in range(T):   # all calls queued back to back; one sync at the end
        ods.append(hd.step(*step_args(op, dseq, t)))
        ohs.append(hh.step_host(*step_args(op, hseq, t)))
    torch.cuda.synchronize()
    for od, oh in zip(ods, ohs):
        assert torch.equal(od.cpu(), oh)
    assert torch.equal(hd.read_state(), hh.read_state())
    hd.close()
    hh.close()


def test_zero_log_decay_and_beta_zero_keep_state():
    """beta = 0 and alpha = 1: the state never changes and o = S0^T q (GDN/KDA)."""
    from recurrent_state_update_deltalog_b200 import DeltaLog
    for op in ("gdn", "kda"):
        S0, seq, _ = make_inputs(op, 2, 2, 64, 64, 9, torch.float32)
        seq["beta"][:] = 0
        seq["log_decay"][:] = 0
        o, merges, final = run_gpu(op, S0, seq, None, 4, torch.float32)
        assert np.array_equal(final, S0)
        want = np.einsum("bhkv,tbhk->tbhv", S0.astype(np.float64), seq["q"].astype(np.float64))
        assert relerr(o, want) < 1e-5


def _extreme_gates(op, seq, levels, seed):
    """Overwrite the gates with a seeded mix of extreme log-decays (per head
    for GDN, per key otherwise) and betas of 0, 1/2 and 1."""
    rng = np.random.default_rng(seed)
    ld = seq["log_decay"]
    seq["log_decay"] = rng.choice(np.asarray(levels, np.float32), size=ld.shape).astype(np.float32)
    if "beta" in seq:
        seq["beta"] = rng.choice(np.asarray([0.0, 0.5, 1.0], np.float32), size=seq["beta"].shape)
    return seq


@pytest.mark.parametrize("op", OPS)
@pytest.mark.parametrize("dims", [(64, 64), (128, 128)])
@pytest.mark.parametrize("M", [8, 64])
def test_extreme_gates(op, dims, M):
    """Decays of 0 (no decay), -1e-7, -2 and -40 per step, mixed across keys
    and steps, and betas of 0, 1/2 and 1: over cycles of up to 64 steps the
    cumulative log-decay reaches about -2500, where exp(Lam_t) underflows
    while ratios of recent entries stay near 1."""
    dk, dv = dims
    T = 2 * M + 3
    S0, seq, u = make_inputs(op, 3, 2, dk, dv, T, torch.bfloat16, seed=13)
    seq = _extreme_gates(op, seq, [0.0, -1e-7, -2.0, -40.0], seed=14)
    o, merges, final = run_gpu(op, S0, seq, u, M, torch.bfloat16)
    o_ref, S_ref, rec = run_oracle(op, S0, seq, u, record=tuple(merges))
    assert np.isfinite(o).all() and np.isfinite(final).all()
    assert relerr(o, o_ref) < TOL[torch.bfloat16]
    for t, S in merges.items():
        assert relerr(S, rec[t]) < TOL[torch.bfloat16], t
    assert relerr(final, S_ref) < TOL[torch.bfloat16]


@pytest.mark.parametrize("op", OPS)
def test_extreme_gates_fp32(op):
    """fp32 inputs with decays of 0, -1e-7, -2 and -20 at M = 8: the fp32
    snapshots (|Lam| <= 140) keep the replay ratios inside the fp32 tolerance."""
    M, T = 8, 19
    S0, seq, u = make_inputs(op, 3, 2, 128, 128, T, torch.float32, seed=15)
    seq = _extreme_gates(op, seq, [0.0, -1e-7, -2.0, -20.0], seed=16)
    o, merges, final = run_gpu(op, S0, seq, u, M, torch.float32)
    o_ref, S_ref, _ = run_oracle(op, S0, seq, u)
    assert relerr(o, o_ref) < TOL[torch.float32]
    assert relerr(final, S_ref) < TOL[torch.float32]


def test_inputs_aligned_to_their_element_only():
    """q/k/v views offset by one element (2-byte aligned) give the same result."""
    from recurrent_state_update_deltalog_b200 import DeltaLog
    B, H, d, M, T = 2, 4, 64, 4, 6
    S0, seq, _ = make_inputs("gdn", B, H, d, d, T, torch.bfloat16)
    o_ref, S_ref, _ = run_oracle("gdn", S0, seq, None)
    dseq = to_device(seq, torch.bfloat16)
    shifted = {}
    for key in ("q", "k", "v"):
        flat = torch.zeros(dseq[key].numel() + 1, dtype=torch.bfloat16, device="cuda")
        flat[1:] = dseq[key].reshape(-1)
        shifted[key] = flat[1:].view(dseq[key].shape)
    h = DeltaLog(B, H, d, d, M, op="gdn")
    h.load_state(torch.from_numpy(S0).cuda())
    outs = []
    for t in range(T):
        outs.append(h.step(shifted["q"][t], shifted["k"][t], shifted["v"][t],
                           dseq["log_decay"][t], dseq["beta"][t]).float().cpu().numpy())
    assert relerr(np.stack(outs), o_ref) < 5e-3
    h.close()


@pytest.mark.parametrize("op", OPS)
def test_programmatic_launch_gives_identical_results(op):
    """Steps launched as programmatic dependents (default) and plainly (PDL off)
    produce bit-identical outputs and states."""
    from recurrent_state_update_deltalog_b200 import DeltaLog
    B, H, d, M, T = 64, 8, 128, 4, 10
    S0, seq, u = make_inputs(op, B, H, d, d, T, torch.bfloat16)
    dseq = to_device(seq, torch.bfloat16)
    res = []
    for pdl in (True, False):
        h = DeltaLog(B, H, d, d, M, op=op)
        h.set_pdl(pdl)
        h.load_state(torch.from_numpy(S0).cuda())
        if u is not None:
            h.set_bonus(torch.from_numpy(u).cuda())
        out = torch.empty((B, H, d), dtype=torch.bfloat16, device="cuda")   # one reused buffer
        outs = []
        for t in range(T):
            h.step(*step_args(op, dseq, t), out=out)
            outs.append(out.clone())
        res.append((torch.stack(outs).cpu(), h.read_state().cpu()))
        h.close()
    assert torch.equal(res[0][0], res[1][0]) and torch.equal(res[0][1], res[1][1])


@pytest.mark.parametrize("mapped", [False, True])
@pytest.mark.parametrize("op", OPS)
def test_inputs_rewritten_in_place_before_each_step(op, mapped):
    """A serving loop reuses one set of input buffers: a kernel of the caller
    (here a torch copy, and for mapped steps a fresh slot permutation) writes
    token t's q/k/v, gates and slot map in place right before dl_step.  With
    programmatic launch on, the step may start while that copy drains, so it
    must read none of them before the copy has completed.  The outputs and
    states must equal those of plain launches and of untouched per-token
    buffers bit for bit, and the oracle's."""
    from recurrent_state_update_deltalog_b200 import DeltaLog
    B, H, d, M, T = 96, 8, 128, 4, 11
    S0, seq, u = make_inputs(op, B, H, d, d, T, torch.bfloat16)
    dseq = to_device(seq, torch.bfloat16)
    perms = [torch.from_numpy(np.random.default_rng(100 + t).permutation(B).astype(np.int32)).cuda()
             for t in range(T)]

    def token(t):   # inputs of token t in batch-row order (row r on slot perm[r])
        args = step_args(op, dseq, t)
        if not mapped:
            return args
        p = perms[t].long()
        return tuple(x[p] if x is not None else None for x in args)

    toks = [token(t) for t in range(T)]
    res = []
    for pdl, reuse in ((True, True), (False, True), (False, False)):
        h = DeltaLog(B, H, d, d, M, op=op)
        h.set_pdl(pdl)
        h.load_state(torch.from_numpy(S0).cuda())
        if u is not None:
            h.set_bonus(torch.from_numpy(u).cuda())
        bufs = [torch.empty_like(x) if x is not None else None for x in toks[0]]
        ibuf = torch.empty(B, dtype=torch.int32, device="cuda")
        outs = torch.empty((T, B, H, d), dtype=torch.bfloat16, device="cuda")
        for t in range(T):
            if reuse:
                for b, x in zip(bufs, toks[t]):
                    if b is not None:
                        b.copy_(x)
                ibuf.copy_(perms[t])
                args, idx = bufs, ibuf
            else:
                args, idx = toks[t], perms[t]
            h.step(*args, out=outs[t], **({"slot_idx": idx} if mapped else {}))
        if mapped:   # back to slot order
            outs = torch.stack([torch.empty_like(outs[t]).index_copy_(0, perms[t].long(), outs[t])
                                for t in range(T)])
        h.check_device()
        res.append((outs.cpu(), h.read_state().cpu()))
        h.close()
    for o, s in res[1:]:
        assert torch.equal(res[0][0], o) and torch.equal(res[0][1], s)
    o_ref, S_ref, _ = run_oracle(op, S0, seq, u)
    assert relerr(res[0][0].float().numpy(), o_ref) < TOL[torch.bfloat16]
    assert relerr(res[0][1].numpy(), S_ref) < TOL[torch.bfloat16]


# ---- per-slot admission (serving: admit / evict / flush one slot) ---------------

def _oracle_step(op, S, seq, t, u):
    """One eager step of every unit (fp64): returns (o_t, S_t)."""
    one = {key: val[t:t + 1] for key, val in seq.items()}
    o, S_next, _ = run_oracle(op, S, one, u)
    return o[0], S_next


@pytest.mark.parametrize("op", OPS)
@pytest.mark.parametrize("dims,M", [((64, 64), 3), ((128, 128), 4), ((128, 128), 8), ((64, 128), 5)])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_slot_admission(op, dims, M, dtype):
    """Slots loaded, merged and zeroed mid-cycle keep the handle's log length
    (their entries are cleared), and every output and state follows the eager
    recurrence restarted from the loaded state."""
    from recurrent_state_update_deltalog_b200 import DeltaLog
    from synthetic import initial_state
    B, H, T = 6, 3, 20
    dk, dv = dims
    S0, seq, u = make_inputs(op, B, H, dk, dv, T, dtype)
    fresh = initial_state(7, B, H, dk, dv)                       # states of admitted sequences
    dseq = to_device(seq, dtype)
    tol = TOL[dtype]
    h = DeltaLog(B, H, dk, dv, M, op=op, dtype=dtype)
    h.load_state(torch.from_numpy(S0).cuda())
    if u is not None:
        h.set_bonus(torch.from_numpy(u).cuda())
    S_ref = S0.astype(np.float64)
    n = 0
    events = {2: ("load", 2), 5: ("merge", 4), 7: ("zero", 0), 11: ("load", 1), 13: ("flush", None),
              15: ("load", 5)}
    outs, refs = [], []
    for t in range(T):
        ev = events.get(t)
        if ev:
            kind, b = ev
            if kind == "load":
                h.slot_load(b, torch.from_numpy(fresh[b]).cuda())
                S_ref[b] = fresh[b]
            elif kind == "zero":
                h.slot_load(b)
                S_ref[b] = 0
            elif kind == "merge":
                h.slot_merge(b)
            else:
                got = h.read_state().cpu().numpy()
                assert relerr(got, S_ref) < tol
                h.merge()
                n = 0
            if b is not None:                                  # the slot reads back as set
                assert relerr(h.slot_read(b).cpu().numpy(), S_ref[b]) < tol, (t, b)
        assert h.log_len == n
        o = h.step(*step_args(op, dseq, t))
        outs.append(o.float().cpu().numpy())
        o_ref, S_ref = _oracle_step(op, S_ref, seq, t, u)
        refs.append(o_ref)
        n = 0 if n + 1 == M else n + 1
        if t in (8, 16):
            for b in (0, 3):
                assert relerr(h.slot_read(b).cpu().numpy(), S_ref[b]) < tol, (t, b)
    assert relerr(np.stack(outs), np.stack(refs)) < tol
    assert relerr(h.read_state().cpu().numpy(), S_ref) < tol
    h.check_device()
    h.close()


def test_slot_arguments_rejected():
    from recurrent_state_update_deltalog_b200 import DeltaLog, DeltaLogError
    h = DeltaLog(2, 2, 64, 64, 4, op="gdn")
    for bad in (-1, 2):
        with pytest.raises(DeltaLogError):
            h.slot_merge(bad)
        with pytest.raises(DeltaLogError):
            h.slot_load(bad)
    h.close()


# ---- slot index map (serving batch over a state pool) ---------------------------

def _batch(seq, t, idx):
    """Inputs of step t gathered into batch rows (padding and out-of-range rows
    take the nearest slot's)."""
    return {key: val[t:t + 1, np.clip(np.asarray(idx), 0, val.shape[1] - 1)] for key, val in seq.items()}


def _run_indexed(op, dims, M, dtype, eager=False, log_b_bf16=False, log_lam_f16=False):
    from recurrent_state_update_deltalog_b200 import DeltaLog
    from synthetic import initial_state
    B, H, T = 8, 3, 18
    dk, dv = dims
    S0, seq, u = make_inputs(op, B, H, dk, dv, T, dtype, seed=3)
    fresh = initial_state(11, B, H, dk, dv)
    tol = TOL[dtype]
    rng = np.random.default_rng(5)
    h = DeltaLog(B, H, dk, dv, M, op=op, dtype=dtype)
    h.set_log_b_bf16(log_b_bf16)
    h.set_log_lam_f16(log_lam_f16)
    h.load_state(torch.from_numpy(S0).cuda())
    if u is not None:
        h.set_bonus(torch.from_numpy(u).cuda())
    S_ref = S0.astype(np.float64)
    live = [0, 1, 2, 3, 4, 5]
    events = {4: ("evict", 2), 6: ("admit", 6), 9: ("admit", 2), 11: ("admit", 7), 14: ("evict", 0)}
    for t in range(T):
        ev = events.get(t)
        if ev and ev[0] == "evict":
            live.remove(ev[1])
        elif ev:
            b = ev[1]
            if eager:   # the dense kernel keeps absent slots as they are; load like a new sequence
                h.load_state(h.read_state().index_copy_(0, torch.tensor([b], device="cuda"),
                                                       torch.from_numpy(fresh[b:b + 1]).cuda()))
            else:
                h.slot_load(b, torch.from_numpy(fresh[b]).cuda())
            S_ref[b] = fresh[b]
            live.append(b)
        pad = int(rng.integers(0, 3))
        idx = list(rng.permutation(live)) + [-1] * pad
        idx = idx[:B]
        one = _batch(seq, t, idx)
        dseq = to_device(one, dtype)
        sentinel = 7.0
        out = torch.full((len(idx), H, dv), sentinel, dtype=dtype, device="cuda")
        args = step_args(op, dseq, 0)
        d_idx = torch.tensor(idx, dtype=torch.int32, device="cuda")
        (h.eager_step if eager else h.step)(*args, out=out, slot_idx=d_idx)
        o_all, S_all = _oracle_step(op, S_ref, seq, t, u)
        got = out.float().cpu().numpy()
        rows = [r for r, b in enumerate(idx) if b >= 0]
        pads = [r for r, b in enumerate(idx) if b < 0]
        assert np.all(got[pads] == sentinel), t
        # o_t of the step's live rows as one tensor (max relative error per tensor)
        assert relerr(got[rows], o_all[[idx[r] for r in rows]]) < tol, t
        S_ref[live] = S_all[live]
    for b in live:
        assert relerr(h.slot_read(b).cpu().numpy(), S_ref[b]) < tol, b
    h.check_device()
    h.close()


@pytest.mark.parametrize("op", OPS)
@pytest.mark.parametrize("dims,M", [((64, 64), 3), ((128, 128), 8), ((64, 128), 5)])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_slot_index_map(op, dims, M, dtype):
    """Batch rows on pool slots given by an index map: permuted every token,
    padding rows untouched, slots evicted (left out) and admitted mid-cycle."""
    _run_indexed(op, dims, M, dtype)


@pytest.mark.parametrize("op", OPS)
def test_slot_index_map_eager(op):
    _run_indexed(op, (128, 128), 1, torch.bfloat16, eager=True)


def _run_hold(op, dims, M, dtype, eager=False, tiles=0, log_b_bf16=False, log_lam_f16=False):
    """Slots that sit tokens out: named as slot | HOLD, across merge steps and
    from the first or up to the last token.  The oracle does not advance a held
    slot; its output row stays untouched and its state must equal the one it
    paused with at every token, and every active output must match."""
    from recurrent_state_update_deltalog_b200 import DeltaLog
    B, H, T = 7, 3, 21
    dk, dv = dims
    S0, seq, u = make_inputs(op, B, H, dk, dv, T, dtype, seed=9)
    tol = TOL[dtype]
    rng = np.random.default_rng(21)
    paused = {1: range(2, 9), 3: range(5, 7), 4: range(0, 3), 5: range(16, T), 0: (M - 1, 10)}
    h = DeltaLog(B, H, dk, dv, M, op=op, dtype=dtype)
    h.set_value_tiles(tiles)
    h.set_log_b_bf16(log_b_bf16)
    h.set_log_lam_f16(log_lam_f16)
    h.load_state(torch.from_numpy(S0).cuda())
    if u is not None:
        h.set_bonus(torch.from_numpy(u).cuda())
    S_ref = S0.astype(np.float64)
    try:
        for t in range(T):
            held = [b for b, r in paused.items() if t in r]
            active = [b for b in range(B) if b not in held]
            rows = list(rng.permutation(active)) + [b | DeltaLog.HOLD for b in held]
            order = rng.permutation(len(rows))
            idx = [int(rows[i]) for i in order]
            plain = [b & ~DeltaLog.HOLD if b >= 0 else b for b in idx]
            dseq = to_device(_batch(seq, t, plain), dtype)
            sentinel = 7.0
            out = torch.full((len(idx), H, dv), sentinel, dtype=dtype, device="cuda")
            d_idx = torch.tensor(idx, dtype=torch.int32, device="cuda")
            (h.eager_step if eager else h.step)(*step_args(op, dseq, 0), out=out, slot_idx=d_idx)
            o_all, S_all = _oracle_step(op, S_ref, seq, t, u)
            got = out.float().cpu().numpy()
            act_rows = [r for r, b in enumerate(idx) if 0 <= b < B]
            idle_rows = [r for r, b in enumerate(idx) if not 0 <= b < B]
            assert np.all(got[idle_rows] == sentinel), t
            assert relerr(got[act_rows], o_all[[idx[r] for r in act_rows]]) < tol, t
            S_ref[active] = S_all[active]
            for b in held:    # a held slot reads back exactly as it paused
                assert relerr(h.slot_read(b).cpu().numpy(), S_ref[b]) < tol, (t, b)
        assert (h.log_len == T % M) or eager
        for b in range(B):
            assert relerr(h.slot_read(b).cpu().numpy(), S_ref[b]) < tol, b
        h.merge()
        assert relerr(h.read_state().cpu().numpy(), S_ref) < tol
        h.check_device()
    finally:
        h.close()


@pytest.mark.parametrize("op", OPS)
@pytest.mark.parametrize("dims,M", [((64, 64), 3), ((128, 128), 4), ((128, 128), 8), ((64, 128), 5)])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_held_slots(op, dims, M, dtype):
    _run_hold(op, dims, M, dtype)


@pytest.mark.parametrize("op", OPS)
@pytest.mark.parametrize("tiles", [2, 4])
def test_held_slots_value_tiles(op, tiles):
    """Held slots with each head split over several CTAs (each writes its
    columns of the null entry; the first writes a_n and the snapshot)."""
    _run_hold(op, (128, 128), 4, torch.bfloat16, tiles=tiles)


@pytest.mark.parametrize("op", ["gdn", "kda"])
def test_held_slots_bf16_log(op):
    _run_hold(op, (128, 128), 8, torch.bfloat16, log_b_bf16=True)


@pytest.mark.parametrize("op", OPS)
def test_held_slots_eager(op):
    """The dense kernel leaves a held slot's state as it is."""
    _run_hold(op, (64, 64), 1, torch.bfloat16, eager=True)


def test_slot_index_out_of_range_raises_device_flag():
    """An index past the pool skips its row and raises the device error word;
    the other rows are computed as usual."""
    from recurrent_state_update_deltalog_b200 import DeltaLog, DeltaLogError
    op, B, H, dk, dv = "gdn", 4, 2, 64, 64
    S0, seq, u = make_inputs(op, B, H, dk, dv, 1, torch.float32)
    h = DeltaLog(B, H, dk, dv, 4, op=op, dtype=torch.float32)
    h.load_state(torch.from_numpy(S0).cuda())
    idx = [1, 9, 3]
    dseq = to_device(_batch(seq, 0, idx), torch.float32)
    out = torch.zeros((3, H, dv), device="cuda")
    h.step(*step_args(op, dseq, 0), out=out, slot_idx=torch.tensor(idx, dtype=torch.int32, device="cuda"))
    with pytest.raises(DeltaLogError, match="0x2"):
        h.check_device()
    h.check_device()                                   # the word was cleared
    o_all, _ = _oracle_step(op, S0.astype(np.float64), seq, 0, u)
    got = out.cpu().numpy()
    assert relerr(got[0], o_all[1]) < 1e-4 and relerr(got[2], o_all[3]) < 1e-4
    assert np.all(got[1] == 0)
    h.close()


def test_slot_index_map_arguments():
    import ctypes

    from recurrent_state_update_deltalog_b200 import DeltaLog, DeltaLogError
    from recurrent_state_update_deltalog_b200 import _native as N
    h = DeltaLog(2, 2, 64, 64, 4, op="gdn", dtype=torch.float32)
    z = torch.zeros((3, 2, 64), device="cuda")
    g = torch.zeros((3, 2), device="cuda")
    with pytest.raises(ValueError):                    # more rows than slots
        h.step(z, z, z, g, g, slot_idx=torch.zeros(3, dtype=torch.int32, device="cuda"))
    e = torch.empty((0, 2, 64), device="cuda")
    ge = torch.empty((0, 2), device="cuda")
    h.step(e, e, e, ge, ge, slot_idx=torch.empty(0, dtype=torch.int32, device="cuda"))  # no-op
    assert h.log_len == 0
    with pytest.raises(DeltaLogError):                 # a map pointer that is not 4-byte aligned
        N.call("dl_step_indexed", h._h, ctypes.c_void_p(torch.zeros(2, dtype=torch.int32, device="cuda")
                                                         .data_ptr() + 2), 1, None, None, None, None, None,
               None, None)
    h.close()


@pytest.mark.parametrize("op", OPS)
@pytest.mark.parametrize("d", [64, 128])
def test_auto_merge_interval(op, d):
    """A handle created with M = "auto" takes dl_suggest_m's interval and its
    outputs and state follow the oracle across two merges."""
    from recurrent_state_update_deltalog_b200 import DeltaLog, suggest_m
    B, H = 3, 2
    h = DeltaLog(B, H, d, d, "auto", op=op, dtype=torch.bfloat16)
    assert h.M == suggest_m(op, d, d) and 2 <= h.M <= 64
    T = 2 * h.M + 3
    S0, seq, u = make_inputs(op, B, H, d, d, T, torch.bfloat16, seed=4)
    dseq = to_device(seq, torch.bfloat16)
    h.load_state(torch.from_numpy(S0).cuda())
    if u is not None:
        h.set_bonus(torch.from_numpy(u).cuda())
    outs = [h.step(*step_args(op, dseq, t)).float().cpu().numpy() for t in range(T)]
    assert h.log_len == T % h.M
    o_ref, S_ref, _ = run_oracle(op, S0, seq, u)
    assert relerr(np.stack(outs), o_ref) < TOL[torch.bfloat16]
    assert relerr(h.read_state().cpu().numpy(), S_ref) < TOL[torch.bfloat16]
    h.close()


# ---- bf16 value-factor log ------------------------------------------------------

@pytest.mark.parametrize("op", ["gdn", "kda"])
@pytest.mark.parametrize("dims", [(64, 64), (128, 128), (64, 128), (128, 64)])
@pytest.mark.parametrize("M", [4, 8, 16, 32])
def test_log_b_bf16(op, dims, M):
    """b_i rounded to bf16 in the log: outputs, merged bases and the final
    state stay within the bf16-input tolerance of the fp64 eager recurrence
    over 80 tokens (several merges; a tail that ends mid-cycle)."""
    B, H, T = 3, 4, 80
    dk, dv = dims
    S0, seq, u = make_inputs(op, B, H, dk, dv, T, torch.bfloat16, seed=6)
    o, merges, final = run_gpu(op, S0, seq, u, M, torch.bfloat16, log_b_bf16=True)
    o_ref, S_ref, rec = run_oracle(op, S0, seq, u, record=tuple(merges))
    tol = TOL[torch.bfloat16]
    assert relerr(o, o_ref) < tol
    for t, S in merges.items():
        assert relerr(S, rec[t]) < tol, t
    assert relerr(final, S_ref) < tol


def test_log_b_bf16_differs_from_fp32_log_and_option_rules():
    """The option really rounds b_i (the outputs move, within tolerance), and
    it is refused for fp32 handles and while the log holds entries."""
    from recurrent_state_update_deltalog_b200 import DeltaLog, DeltaLogError
    op, B, H, d, M, T = "gdn", 2, 2, 64, 8, 20
    S0, seq, u = make_inputs(op, B, H, d, d, T, torch.bfloat16, seed=8)
    o32, _, _ = run_gpu(op, S0, seq, u, M, torch.bfloat16)
    o16, _, _ = run_gpu(op, S0, seq, u, M, torch.bfloat16, log_b_bf16=True)
    assert not np.array_equal(o32, o16)
    o_ref, _, _ = run_oracle(op, S0, seq, u)
    assert relerr(o16, o_ref) < TOL[torch.bfloat16]
    h = DeltaLog(B, H, d, d, M, op=op, dtype=torch.float32)
    with pytest.raises(DeltaLogError):
        h.set_log_b_bf16(True)
    h.close()
    h = DeltaLog(B, H, d, d, M, op=op, dtype=torch.bfloat16)
    dseq = to_device(seq, torch.bfloat16)
    h.step(*step_args(op, dseq, 0))
    with pytest.raises(DeltaLogError):
        h.set_log_b_bf16(True)
    h.merge()
    h.set_log_b_bf16(True)
    h.close()


@pytest.mark.parametrize("op", ["gdn", "kda"])
def test_log_b_bf16_with_slot_map_and_admission(op):
    """The bf16 b-log under a slot index map with eviction and admission."""
    _run_indexed(op, (128, 128), 8, torch.bfloat16, log_b_bf16=True)


# ---- compact per-key snapshots: fp16 log-gates (DL_OPT_LOG_LAM_F16) ----------------

@pytest.mark.parametrize("op", ["kda", "rwkv6"])
@pytest.mark.parametrize("dims", [(64, 64), (128, 128), (64, 128), (128, 64)])
@pytest.mark.parametrize("M", [4, 8, 16, 32])
@pytest.mark.parametrize("log_b_bf16", [False, True])
def test_log_lam_f16(op, dims, M, log_b_bf16):
    """Per-key snapshots kept as fp16 log-gates (with and without the bf16
    b-log): outputs, merged bases and the final state stay within the
    bf16-input tolerance of the fp64 eager recurrence over 256 tokens."""
    if log_b_bf16 and op == "rwkv6":
        pytest.skip("RWKV6's log already holds raw bf16 values")
    B, H, T = 3, 4, 256
    dk, dv = dims
    S0, seq, u = make_inputs(op, B, H, dk, dv, T, torch.bfloat16, seed=8)
    o, merges, final = run_gpu(op, S0, seq, u, M, torch.bfloat16, log_b_bf16=log_b_bf16, log_lam_f16=True)
    o_ref, S_ref, rec = run_oracle(op, S0, seq, u, record=tuple(merges))
    tol = TOL[torch.bfloat16]
    assert relerr(o, o_ref) < tol
    for t, S in merges.items():
        assert relerr(S, rec[t]) < tol, t
    assert relerr(final, S_ref) < tol


@pytest.mark.parametrize("op", ["kda", "rwkv6"])
@pytest.mark.parametrize("M", [8, 64])
def test_log_lam_f16_extreme_gates(op, M):
    """fp16 log-gates under decays of 0, -1e-7, -2 and -40 mixed across keys
    and steps: a gate rounds to fp16 relative to itself, so a strongly decayed
    key next to one that barely decays keeps its ratios."""
    B, H, d, T = 2, 3, 128, 2 * M + 5
    S0, seq, u = make_inputs(op, B, H, d, d, T, torch.bfloat16, seed=12)
    seq = _extreme_gates(op, seq, [0.0, -1e-7, -2.0, -40.0], seed=13)
    o, merges, final = run_gpu(op, S0, seq, u, M, torch.bfloat16, log_lam_f16=True)
    o_ref, S_ref, rec = run_oracle(op, S0, seq, u, record=tuple(merges))
    tol = TOL[torch.bfloat16]
    assert relerr(o, o_ref) < tol
    for t, S in merges.items():
        assert relerr(S, rec[t]) < tol, t
    assert relerr(final, S_ref) < tol


@pytest.mark.parametrize("op", ["kda", "rwkv6"])
def test_log_lam_f16_with_slot_map_admission_and_holds(op):
    """fp16 log-gates through the slot index map (eviction, admission: cleared
    entries are zero gates) and held slots (null entries are zero gates)."""
    _run_indexed(op, (128, 128), 8, torch.bfloat16, log_lam_f16=True)
    _run_hold(op, (128, 128), 4, torch.bfloat16, log_lam_f16=True)


def test_log_lam_f16_option_rules():
    from recurrent_state_update_deltalog_b200 import DeltaLog, DeltaLogError
    h = DeltaLog(2, 2, 64, 64, 4, op="kda", dtype=torch.float32)
    with pytest.raises(DeltaLogError) as ei:
        h.set_log_lam_f16(True)
    assert ei.value.status == -2
    h.close()
    S0, seq, u = make_inputs("kda", 2, 2, 64, 64, 2, torch.bfloat16)
    dseq = to_device(seq, torch.bfloat16)
    h = DeltaLog(2, 2, 64, 64, 4, op="kda")
    h.step(*step_args("kda", dseq, 0))
    with pytest.raises(DeltaLogError) as ei:   # only with an empty log
        h.set_log_lam_f16(True)
    assert ei.value.status == -6
    h.merge()
    h.set_log_lam_f16(True)
    h.close()
    h = DeltaLog(2, 2, 64, 64, 4, op="gdn")     # GDN: accepted, nothing changes
    h.set_log_lam_f16(True)
    h.close()


# ---- failure paths made on purpose (no fault: a wait that nothing completes) ------

@pytest.mark.parametrize("M", [4, 2])
def test_stalled_log_wait_times_out_and_reports(M):
    """With DL_OPT_TEST_STALL_LOG the log barrier expects bytes that no copy
    delivers: every unit of the step gives up after its bounded wait, writes
    nothing (output rows keep their sentinel; at M = 2 the step is a merge and
    the base keeps its value) and dl_check_device reports the timeout bit.  The
    context stays usable: a fresh handle then matches the oracle."""
    from recurrent_state_update_deltalog_b200 import DeltaLog, DeltaLogError
    op, B, H, d, T = "gdn", 3, 4, 64, 6
    S0, seq, u = make_inputs(op, B, H, d, d, T, torch.bfloat16, seed=4)
    dseq = to_device(seq, torch.bfloat16)
    h = DeltaLog(B, H, d, d, M, op=op)
    h.load_state(torch.from_numpy(S0).cuda())
    h.step(*step_args(op, dseq, 0))                  # n = 0: no log to wait for
    h.check_device()
    h.set_test_stall_log(True)
    out = torch.full((B, H, d), 7.0, dtype=torch.bfloat16, device="cuda")
    h.step(*step_args(op, dseq, 1), out=out)         # n = 1: every unit stalls
    with pytest.raises(DeltaLogError) as ei:
        h.check_device()
    assert ei.value.status == -5 and "0x1" in str(ei.value)
    assert torch.all(out == 7.0)
    if M == 2:   # the stalled merge left the base alone (step 0 only appended)
        assert torch.equal(h.read_state().cpu(), torch.from_numpy(S0))
    h.check_device()                                 # the word was cleared
    h.close()
    o, _, final = run_gpu(op, S0, seq, u, M, torch.bfloat16)
    o_ref, S_ref, _ = run_oracle(op, S0, seq, u)
    assert relerr(o, o_ref) < 5e-3 and relerr(final, S_ref) < 5e-3


def test_create_too_large_returns_oom_and_leaks_nothing():
    """A handle whose state cannot be allocated (4.4 TB) fails with DL_ERR_OOM,
    frees what it took, and a small handle works afterwards."""
    from recurrent_state_update_deltalog_b200 import DeltaLog, DeltaLogError
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    with pytest.raises(DeltaLogError) as ei:
        DeltaLog(1 << 20, 64, 128, 128, 8, op="gdn")
    assert ei.value.status == -4
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 >= free0          # nothing kept (the driver may release unrelated memory meanwhile)
    _check_run("gdn", 2, 3, 64, 64, 4, 9, torch.bfloat16)
