"""The seeded workload generator: determinism, chunking, dtype rounding, recipe."""
import numpy as np
import pytest
import torch

from synthetic import bonus, initial_state, round_to_bf16, sequence, step_inputs


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(100000).astype(np.float32) * 3,
                        np.array([0.0, -0.0, 1.0, 1.00390625, 1.01171875, 65504.0], np.float32)])
    want = torch.from_numpy(x).to(torch.bfloat16).float().numpy()
    assert np.array_equal(round_to_bf16(x), want)


def test_state_chunks_are_slot_local():
    full = initial_state(0, 6, 2, 8, 4)
    part = initial_state(0, 6, 2, 8, 4, slots=[4, 1])
    assert np.array_equal(part[0], full[4]) and np.array_equal(part[1], full[1])
    assert not np.array_equal(full[0], initial_state(1, 6, 2, 8, 4)[0])


def test_sequence_is_deterministic_and_step_local():
    a = sequence(0, "gdn", 3, 2, 16, 16, 5, bf16=True)
    b = sequence(0, "gdn", 3, 2, 16, 16, 3, bf16=True, t0=2)
    for key in a:
        assert np.array_equal(a[key][2:], b[key])


@pytest.mark.parametrize("op", ["gdn", "kda", "rwkv6"])
def test_recipe_shapes_and_ranges(op):
    s = step_inputs(0, op, 64, 4, 32, 16, 0, bf16=True)
    first = "r" if op == "rwkv6" else "q"
    assert s[first].shape == (64, 4, 32) and s["k"].shape == (64, 4, 32)
    assert s["v"].shape == (64, 4, 16)
    for key in (first, "k", "v"):
        assert np.array_equal(s[key], round_to_bf16(s[key]))    # bf16-exact values
    ld = s["log_decay"]
    assert ld.dtype == np.float32 and np.all(ld < 0)
    if op == "gdn":
        assert ld.shape == (64, 4)
    else:
        assert ld.shape == (64, 4, 32)
    if op != "rwkv6":
        n = np.linalg.norm(s["q"].astype(np.float64), axis=-1)
        assert np.all(np.abs(n - 1) < 1e-2)                    # unit norm up to bf16 rounding
        assert np.all((s["beta"] > 0) & (s["beta"] < 1))
        assert "beta" in s and s["beta"].shape == (64, 4)
    else:
        assert "beta" not in s


def test_fp32_inputs_are_not_rounded():
    s = step_inputs(0, "gdn", 4, 1, 64, 64, 0, bf16=False)
    assert not np.array_equal(s["v"], round_to_bf16(s["v"]))


def test_moments():
    S0 = initial_state(0, 8, 4, 32, 32)
    assert abs(S0.std() - 0.02) < 1e-3 and abs(S0.mean()) < 1e-3
    u = bonus(0, 64, 64)
    assert abs(u.std() - 0.1) < 0.01
    s = step_inputs(0, "rwkv6", 32, 8, 64, 64, 0, bf16=False)
    x = np.log(-s["log_decay"].astype(np.float64))          # log w = -exp(x)
    assert abs(x.mean() + 0.5) < 0.02 and abs(x.std() - 0.5) < 0.02
