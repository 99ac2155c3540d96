"""ctypes binding of libdeltalog's C ABI (argument marshalling only).

Every function here forwards to the ``extern "C"`` entry point of the same
name declared in ``include/deltalog.h``; all arithmetic runs in the CUDA
library.  Loading fails loudly if the library has not been built.
"""
from __future__ import annotations

import ctypes
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libdeltalog.so")

DL_GDN, DL_KDA, DL_RWKV6 = 0, 1, 2
DL_F32, DL_BF16 = 0, 1
DL_OK = 0
DL_MAX_M = 64
DL_M_AUTO = 0
DL_PREFILL_ZERO_STATE = 1
DL_STATIC_SCRATCH_BYTES = 16 << 20
DL_SLOT_HOLD = 0x40000000
DL_OPT_STEP_KERNEL = 0
DL_OPT_HOST_PREFETCH = 1
DL_OPT_PDL = 2
DL_OPT_VALUE_TILES = 3
DL_OPT_LOG_B_BF16 = 4
DL_OPT_PREFILL_KERNEL = 5
DL_OPT_TEST_STALL_LOG = 6
DL_OPT_LOG_LAM_F16 = 7
DL_PREFILL_AUTO, DL_PREFILL_RECURRENT, DL_PREFILL_CHUNKED = 0, 1, 2
DL_STEP_AUTO, DL_STEP_REGISTER = 0, 1
STATUS = {0: "DL_OK", -1: "DL_ERR_ARG", -2: "DL_ERR_UNSUPPORTED", -3: "DL_ERR_CUDA",
          -4: "DL_ERR_OOM", -5: "DL_ERR_DEVICE", -6: "DL_ERR_STATE"}

# name -> (restype, argtypes)
_P = ctypes.c_void_p
_I = ctypes.c_int
SIGNATURES = {
    "dl_create": (_I, [ctypes.POINTER(_P), _I, _I, _I, _I, _I, _I, _I]),
    "dl_destroy": (_I, [_P]),
    "dl_load_state": (_I, [_P, _P, _P]),
    "dl_set_bonus": (_I, [_P, _P, _P]),
    "dl_suggest_m": (_I, [_I, _I, _I, _I, ctypes.POINTER(_I)]),
    "dl_merge_interval": (_I, [_P, ctypes.POINTER(_I)]),
    "dl_prefill": (_I, [_P, _P, _I, _P, ctypes.c_longlong, _I, _P, _P, _P, _P, _P, _P, _P]),
    "dl_last_prefill_kernel": (_I, [_P, ctypes.POINTER(_I)]),
    "dl_step": (_I, [_P, _P, _P, _P, _P, _P, _P, _P]),
    "dl_step_indexed": (_I, [_P, _P, _I, _P, _P, _P, _P, _P, _P, _P]),
    "dl_step_host": (_I, [_P, _P, _P, _P, _P, _P, _P, _P]),
    "dl_eager_step": (_I, [_P, _P, _P, _P, _P, _P, _P, _P]),
    "dl_eager_step_indexed": (_I, [_P, _P, _I, _P, _P, _P, _P, _P, _P, _P]),
    "dl_merge": (_I, [_P, _P]),
    "dl_read_state": (_I, [_P, _P, _P]),
    "dl_set_option": (_I, [_P, _I, _I]),
    "dl_last_step_kernel": (_I, [_P, ctypes.POINTER(_I)]),
    "dl_log_len": (_I, [_P, ctypes.POINTER(_I)]),
    "dl_slot_load": (_I, [_P, _I, _P, _P]),
    "dl_slot_merge": (_I, [_P, _I, _P]),
    "dl_slot_read": (_I, [_P, _I, _P, _P]),
    "dl_check_device": (_I, [_P, _P]),
    "dl_decode_static": (_I, [_I, _I, _I, _I, _I, _I, _I, _P, _P, _I, _P, _P, _P, _P, _P, _P, _P, _P]),
    "dl_strerror": (ctypes.c_char_p, [_I]),
    "dl_last_error": (ctypes.c_char_p, []),
}

_lib = None


class DeltaLogError(RuntimeError):
    def __init__(self, fn: str, status: int, message: str):
        super().__init__(f"{fn} -> {STATUS.get(status, status)}: {message}")
        self.status = status


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libdeltalog (once) and declare every exported signature."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(
            f"libdeltalog.so not found at {path}; build it with "
            "`python -m recurrent_state_update_deltalog_b200.build` (there is no CPU fallback)")
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def check(fn: str, status: int) -> None:
    if status != DL_OK:
        msg = load().dl_last_error().decode(errors="replace")
        raise DeltaLogError(fn, status, msg)


def call(fn: str, *args) -> int:
    """Call an entry point and raise DeltaLogError on a non-zero status."""
    st = getattr(load(), fn)(*args)
    check(fn, st)
    return st
