"""C-ABI checks that need no GPU: the library loads, exports every declared
symbol, and rejects bad arguments before touching the device."""
import ctypes
import os
import re

import pytest

from recurrent_state_update_deltalog_b200 import _native as N
from recurrent_state_update_deltalog_b200.build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    for f in os.listdir(os.path.join(ROOT, "include")):
        if f.endswith(".h"):
            text = open(os.path.join(ROOT, "include", f)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names |= set(re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(dl_\w+)\s*\(", text, flags=re.M))
    return names


@pytest.fixture(scope="module")
def lib():
    build()
    return N.load()


def test_every_declared_symbol_is_exported(lib):
    declared = _declared()
    assert {"dl_create", "dl_step", "dl_merge", "dl_eager_step", "dl_destroy"} <= declared
    for name in declared:
        assert hasattr(lib, name), name
    assert declared == set(N.SIGNATURES), declared ^ set(N.SIGNATURES)


def test_build_targets_sm100a_only():
    from recurrent_state_update_deltalog_b200 import build as B
    assert B.ARCH == ["-gencode", "arch=compute_100a,code=sm_100a"]
    assert all("sm_" not in f or "sm_100a" in f for f in B.NVCC_FLAGS)


def test_strerror(lib):
    for code, name in N.STATUS.items():
        assert lib.dl_strerror(code)
    assert lib.dl_strerror(-99) == b"unknown status"


@pytest.mark.parametrize("args,status", [
    ((1, 1, 64, 64, -1, 0, 0), -2),     # M < 0 (0 is DL_M_AUTO)
    ((1, 1, 64, 64, 65, 0, 0), -2),     # M > DL_MAX_M
    ((1, 1, 96, 64, 8, 0, 0), -2),      # unsupported d_k
    ((1, 1, 64, 32, 8, 0, 0), -2),      # unsupported d_v
    ((0, 1, 64, 64, 8, 0, 0), -1),      # B = 0
    ((1, -2, 64, 64, 8, 0, 0), -1),     # H < 0
    ((1, 1, 64, 64, 8, 3, 0), -1),      # unknown op
    ((1, 1, 64, 64, 8, 0, 7), -1),      # unknown dtype
])
def test_create_rejects_bad_arguments(lib, args, status):
    h = ctypes.c_void_p()
    assert lib.dl_create(ctypes.byref(h), *args) == status
    assert not h.value
    assert lib.dl_last_error()


def test_null_handle_paths(lib):
    assert lib.dl_create(None, 1, 1, 64, 64, 8, 0, 0) == -1
    p = ctypes.c_void_p(16)
    for fn in ("dl_step", "dl_eager_step", "dl_step_host"):
        assert getattr(lib, fn)(None, p, p, p, p, p, p, None) == -1
    for fn in ("dl_step_indexed", "dl_eager_step_indexed"):
        assert getattr(lib, fn)(None, p, 1, p, p, p, p, p, p, None) == -1
        assert getattr(lib, fn)(None, None, 0, None, None, None, None, None, None, None) == -1
    assert lib.dl_prefill(None, None, 1, p, 1, 0, p, p, p, p, p, p, None) == -1
    assert lib.dl_merge(None, None) == -1
    assert lib.dl_read_state(None, p, None) == -1
    assert lib.dl_load_state(None, p, None) == -1
    assert lib.dl_set_bonus(None, p, None) == -1
    assert lib.dl_check_device(None, None) == -1
    assert lib.dl_slot_load(None, 0, p, None) == -1
    assert lib.dl_slot_merge(None, 0, None) == -1
    assert lib.dl_slot_read(None, 0, p, None) == -1
    n = ctypes.c_int()
    assert lib.dl_log_len(None, ctypes.byref(n)) == -1
    assert lib.dl_destroy(None) == 0


def test_python_binding_fails_loudly_without_library(tmp_path):
    import importlib
    mod = importlib.reload(N)
    try:
        mod._lib = None
        with pytest.raises(ImportError):
            mod.load(str(tmp_path / "missing.so"))
    finally:
        importlib.reload(N)


# ---- merge-interval choice (host only) ----------------------------------------

def _suggest(lib, op, dk, dv, dtype=1):
    m = ctypes.c_int(-1)
    assert lib.dl_suggest_m(op, dk, dv, dtype, ctypes.byref(m)) == 0
    return m.value


def test_suggest_m_rejects_bad_arguments(lib):
    m = ctypes.c_int()
    assert lib.dl_suggest_m(3, 64, 64, 1, ctypes.byref(m)) == -1
    assert lib.dl_suggest_m(0, 96, 64, 1, ctypes.byref(m)) == -1
    assert lib.dl_suggest_m(0, 64, 64, 5, ctypes.byref(m)) == -1
    assert lib.dl_suggest_m(0, 64, 64, 1, None) == -1
    assert lib.dl_merge_interval(None, ctypes.byref(m)) == -1


@pytest.mark.parametrize("op", [0, 1, 2])
@pytest.mark.parametrize("dk,dv", [(64, 64), (64, 128), (128, 64), (128, 128)])
@pytest.mark.parametrize("dtype", [0, 1])
def test_suggest_m_near_stationary_point(lib, op, dk, dv, dtype):
    """The chosen M sits next to the stationary point of the per-token cost
    S/M + e(M-1)/M + rho(M-1)/2, i.e. M* = sqrt(2(S - e)/rho), for rho between
    the entry's bytes (pure traffic) and three times that."""
    import math
    M = _suggest(lib, op, dk, dv, dtype)
    es = 2 if dtype == 1 else 4
    e = dk * es + dv * (es if op == 2 else 4) + (4 if op == 0 else 4 * dk)
    S = 4 * dk * dv
    lo, hi = math.sqrt(2 * (S - e) / (3 * e)), math.sqrt(2 * (S - e) / e)
    assert 2 <= M <= 64
    assert math.floor(lo) <= M <= math.ceil(hi), (M, lo, hi)
    if dk != dv:                                    # uncalibrated shapes: pure traffic
        assert M in (math.floor(hi), math.ceil(hi))


@pytest.mark.parametrize("op,d,band", [
    (0, 128, (9, 12)), (1, 128, (7, 11)), (2, 64, (8, 9)),
    (0, 64, (9, 12)), (1, 64, (5, 8)), (2, 128, (8, 12)),
])
def test_suggest_m_inside_measured_band(lib, op, d, band):
    """Within the band of M whose measured B200 throughput is within 1% of
    the best point of a fine sweep (M = 4..16, bf16 inputs, large batch)."""
    M = _suggest(lib, op, d, d)
    assert band[0] <= M <= band[1], M


def test_suggest_m_orders(lib):
    """More state per entry favours longer cycles; fatter entries shorter ones."""
    for op in (0, 1, 2):
        assert _suggest(lib, op, 128, 128) >= _suggest(lib, op, 64, 64) - 1
        assert _suggest(lib, op, 128, 128, 0) <= _suggest(lib, op, 128, 128, 1)
