"""PyTorch-facing handle over libdeltalog (marshalling only).

PyTorch supplies device memory and streams; every step of the decode path
runs inside the CUDA library.  Shapes and dtypes are checked here only to
turn a caller mistake into a Python exception before the pointer crosses the
C ABI.
"""
from __future__ import annotations

import ctypes

import torch

from . import _native as N

OPS = {"gdn": N.DL_GDN, "kda": N.DL_KDA, "rwkv6": N.DL_RWKV6}
DTYPES = {torch.float32: N.DL_F32, torch.bfloat16: N.DL_BF16}


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def suggest_m(op, d_k, d_v, dtype=torch.bfloat16):
    """Merge interval the library's cost model picks for this operator and
    head shape (``dl_suggest_m``; no device needed)."""
    m = ctypes.c_int()
    N.call("dl_suggest_m", OPS[op], int(d_k), int(d_v), DTYPES[dtype], ctypes.byref(m))
    return m.value


class DeltaLog:
    """One library handle: B slots x H heads of d_k x d_v fp32 state, merge interval M
    (``"auto"`` or 0: the library's choice, see :func:`suggest_m`; read back as ``.M``).

    ``op`` is ``"gdn"``, ``"kda"`` or ``"rwkv6"``; ``dtype`` is the dtype of
    q/k/v/o (``torch.bfloat16`` or ``torch.float32``).  The handle lives on the
    CUDA device that is current (or given) at construction.
    """

    HOLD = N.DL_SLOT_HOLD   # slot-map bit of a slot that sits a token out

    def __init__(self, B, H, d_k, d_v, M, op="gdn", dtype=torch.bfloat16, device=None):
        if op not in OPS:
            raise ValueError(f"op must be one of {sorted(OPS)}")
        if dtype not in DTYPES:
            raise ValueError("dtype must be torch.bfloat16 or torch.float32")
        M = N.DL_M_AUTO if M == "auto" else int(M)
        self.B, self.H, self.d_k, self.d_v = B, H, d_k, d_v
        self.op, self.dtype = op, dtype
        self.device = torch.device("cuda", torch.cuda.current_device() if device is None
                                   else torch.device(device).index or 0)
        self._h = ctypes.c_void_p()
        with torch.cuda.device(self.device):
            N.call("dl_create", ctypes.byref(self._h), B, H, d_k, d_v, M, OPS[op], DTYPES[dtype])
        m = ctypes.c_int()
        N.call("dl_merge_interval", self._h, ctypes.byref(m))
        self.M = m.value

    # -- helpers -------------------------------------------------------------
    def _stream(self, stream):
        s = stream if stream is not None else torch.cuda.current_stream(self.device)
        return ctypes.c_void_p(s.cuda_stream)

    def _check(self, name, t, shape, dtype, cuda=True):
        if t is None:
            raise ValueError(f"{name} is required")
        if tuple(t.shape) != tuple(shape):
            raise ValueError(f"{name}: expected shape {tuple(shape)}, got {tuple(t.shape)}")
        if t.dtype != dtype:
            raise ValueError(f"{name}: expected {dtype}, got {t.dtype}")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
        if cuda and t.device != self.device:
            raise ValueError(f"{name} must live on {self.device}")
        if not cuda and t.device.type != "cpu":
            raise ValueError(f"{name} must be a host tensor")

    def _decay_shape(self):
        return (self.B, self.H) if self.op == "gdn" else (self.B, self.H, self.d_k)

    def _check_step(self, q, k, v, log_decay, beta, out, cuda, rows=None):
        B, H = self.B if rows is None else rows, self.H
        self._check("q", q, (B, H, self.d_k), self.dtype, cuda)
        self._check("k", k, (B, H, self.d_k), self.dtype, cuda)
        self._check("v", v, (B, H, self.d_v), self.dtype, cuda)
        self._check("log_decay", log_decay, (B,) + self._decay_shape()[1:], torch.float32, cuda)
        if self.op == "rwkv6":
            if beta is not None:
                raise ValueError("beta must be None for rwkv6")
        else:
            self._check("beta", beta, (B, H), torch.float32, cuda)
        self._check("out", out, (B, H, self.d_v), self.dtype, cuda)

    def _alloc_out(self, cuda, rows=None):
        shape = (self.B if rows is None else rows, self.H, self.d_v)
        if cuda:
            return torch.empty(shape, dtype=self.dtype, device=self.device)
        return torch.empty(shape, dtype=self.dtype, pin_memory=True)

    def _slot_map(self, slot_idx):
        if slot_idx is None:
            return None
        if not isinstance(slot_idx, torch.Tensor) or slot_idx.dim() != 1 or slot_idx.numel() > self.B:
            raise ValueError(f"slot_idx must be 1-D with at most B={self.B} entries")
        self._check("slot_idx", slot_idx, (slot_idx.numel(),), torch.int32)
        return slot_idx.numel()

    # -- API -----------------------------------------------------------------
    def load_state(self, S, stream=None):
        self._check("S", S, (self.B, self.H, self.d_k, self.d_v), torch.float32)
        N.call("dl_load_state", self._h, _ptr(S), self._stream(stream))

    def set_bonus(self, u, stream=None):
        self._check("u", u, (self.H, self.d_k), torch.float32)
        N.call("dl_set_bonus", self._h, _ptr(u), self._stream(stream))

    def step(self, q, k, v, log_decay, beta=None, out=None, stream=None, slot_idx=None):
        """One DeltaLog decode token (append, or merge on the M-th step); returns o.

        With ``slot_idx`` (int32 [rows] on the device), inputs and output have
        ``rows`` batch rows and row r runs on slot ``slot_idx[r]`` (negative:
        padding row, left untouched); every live slot must be named, either
        active or held (``slot | DeltaLog.HOLD``: no input read, no output
        written, state kept exactly)."""
        rows = self._slot_map(slot_idx)
        out = self._alloc_out(True, rows) if out is None else out
        self._check_step(q, k, v, log_decay, beta, out, True, rows)
        if rows is None:
            N.call("dl_step", self._h, _ptr(q), _ptr(k), _ptr(v), _ptr(log_decay), _ptr(beta),
                   _ptr(out), self._stream(stream))
        else:
            N.call("dl_step_indexed", self._h, _ptr(slot_idx), rows, _ptr(q), _ptr(k), _ptr(v),
                   _ptr(log_decay), _ptr(beta), _ptr(out), self._stream(stream))
        return out

    def prefill(self, q, k, v, log_decay, beta=None, cu_seqlens=None, slot_idx=None,
                zero_state=False, out=None, stream=None):
        """Prefill -> decode hand-off over packed prompts (``dl_prefill``).

        q, k, v, log_decay, beta hold ``total`` tokens in dl_step's per-slot
        layouts ([total, H, ...]); ``cu_seqlens`` (int32 [rows + 1], device)
        splits them into rows; row r runs on slot ``slot_idx[r]`` (int32
        [rows], device; default: slot r).  Each named slot's base then holds
        the state after its last token.  Returns o [total, H, d_v]."""
        if cu_seqlens is None:
            raise ValueError("cu_seqlens is required")
        total = q.shape[0]
        rows = cu_seqlens.numel() - 1
        if rows < 0 or rows > self.B:
            raise ValueError(f"cu_seqlens must hold rows + 1 offsets with rows <= B={self.B}")
        self._check("cu_seqlens", cu_seqlens, (rows + 1,), torch.int32)
        if slot_idx is not None:
            self._check("slot_idx", slot_idx, (rows,), torch.int32)
        out = self._alloc_out(True, total) if out is None else out
        self._check_step(q, k, v, log_decay, beta, out, True, total)
        flags = N.DL_PREFILL_ZERO_STATE if zero_state else 0
        N.call("dl_prefill", self._h, _ptr(slot_idx), rows, _ptr(cu_seqlens), total, flags,
               _ptr(q), _ptr(k), _ptr(v), _ptr(log_decay), _ptr(beta), _ptr(out), self._stream(stream))
        return out

    def step_host(self, q, k, v, log_decay, beta=None, out=None, stream=None):
        """dl_step on host tensors (pinned for async copies); o is ready after a stream sync."""
        out = self._alloc_out(False) if out is None else out
        self._check_step(q, k, v, log_decay, beta, out, False)
        N.call("dl_step_host", self._h, _ptr(q), _ptr(k), _ptr(v), _ptr(log_decay), _ptr(beta),
               _ptr(out), self._stream(stream))
        return out

    def eager_step(self, q, k, v, log_decay, beta=None, out=None, stream=None, slot_idx=None):
        """Dense baseline: S_{t-1} read and S_t written every token (needs an empty log).
        ``slot_idx`` as in :meth:`step`; slots not named keep their state."""
        rows = self._slot_map(slot_idx)
        out = self._alloc_out(True, rows) if out is None else out
        self._check_step(q, k, v, log_decay, beta, out, True, rows)
        if rows is None:
            N.call("dl_eager_step", self._h, _ptr(q), _ptr(k), _ptr(v), _ptr(log_decay), _ptr(beta),
                   _ptr(out), self._stream(stream))
        else:
            N.call("dl_eager_step_indexed", self._h, _ptr(slot_idx), rows, _ptr(q), _ptr(k), _ptr(v),
                   _ptr(log_decay), _ptr(beta), _ptr(out), self._stream(stream))
        return out

    def merge(self, stream=None):
        N.call("dl_merge", self._h, self._stream(stream))

    def read_state(self, out=None, stream=None):
        if out is None:
            out = torch.empty((self.B, self.H, self.d_k, self.d_v), dtype=torch.float32,
                              device=self.device)
        self._check("out", out, (self.B, self.H, self.d_k, self.d_v), torch.float32)
        N.call("dl_read_state", self._h, _ptr(out), self._stream(stream))
        return out

    def set_step_kernel(self, kind):
        """``"auto"`` (default) or ``"register"``: which kernel runs dl_step."""
        vals = {"auto": N.DL_STEP_AUTO, "register": N.DL_STEP_REGISTER}
        N.call("dl_set_option", self._h, N.DL_OPT_STEP_KERNEL, vals[kind])

    def set_host_prefetch(self, on):
        """Let step_host upload inputs on the handle's copy stream ahead of the
        caller's stream (the host inputs must be ready when step_host is called)."""
        N.call("dl_set_option", self._h, N.DL_OPT_HOST_PREFETCH, 1 if on else 0)

    def set_pdl(self, on):
        """Programmatic dependent launch of steps that follow an append (default on)."""
        N.call("dl_set_option", self._h, N.DL_OPT_PDL, 1 if on else 0)

    def set_prefill_kernel(self, kind):
        """``"auto"`` (default), ``"recurrent"`` or ``"chunked"``: which kernel runs prefill."""
        vals = {"auto": N.DL_PREFILL_AUTO, "recurrent": N.DL_PREFILL_RECURRENT, "chunked": N.DL_PREFILL_CHUNKED}
        N.call("dl_set_option", self._h, N.DL_OPT_PREFILL_KERNEL, vals[kind])

    @property
    def last_prefill_kernel(self):
        """Kernel used by the most recent prefill: ``"recurrent"``, ``"chunked"`` or ``None``."""
        k = ctypes.c_int()
        N.call("dl_last_prefill_kernel", self._h, ctypes.byref(k))
        return {N.DL_PREFILL_RECURRENT: "recurrent", N.DL_PREFILL_CHUNKED: "chunked"}.get(k.value)

    def set_log_b_bf16(self, on):
        """Store GDN/KDA log value factors b_i in bf16 (bf16 handles, empty log)."""
        N.call("dl_set_option", self._h, N.DL_OPT_LOG_B_BF16, 1 if on else 0)

    def set_test_stall_log(self, on):
        """Test of the error path only: steps arm their log barrier but copy
        nothing, so every unit with a non-empty log times out (20 us), writes
        nothing and raises DL_DEVERR_WAIT_TIMEOUT."""
        N.call("dl_set_option", self._h, N.DL_OPT_TEST_STALL_LOG, 1 if on else 0)

    def set_log_lam_f16(self, on):
        """Store KDA/RWKV6 per-key decay metadata as fp16 log-gates (bf16 handles, empty log)."""
        N.call("dl_set_option", self._h, N.DL_OPT_LOG_LAM_F16, 1 if on else 0)

    def set_value_tiles(self, n):
        """0 (automatic), 1, 2 or 4 value tiles (CTAs) per head in the register-tile step kernel."""
        N.call("dl_set_option", self._h, N.DL_OPT_VALUE_TILES, int(n))

    @property
    def last_step_kernel(self):
        """Kernel used by the most recent step: ``"register"`` or ``None``."""
        k = ctypes.c_int()
        N.call("dl_last_step_kernel", self._h, ctypes.byref(k))
        return {N.DL_STEP_REGISTER: "register"}.get(k.value)

    @property
    def log_len(self):
        """Common log length of all slots (raises DeltaLogError when slots differ)."""
        n = ctypes.c_int()
        N.call("dl_log_len", self._h, ctypes.byref(n))
        return n.value

    # -- per-slot lifecycle (serving) ------------------------------------------
    def _slot_state_shape(self):
        return (self.H, self.d_k, self.d_v)

    def slot_load(self, slot, S=None, stream=None):
        """Admit a sequence into `slot`: state S [H, d_k, d_v] (None = zeros), empty log."""
        if S is not None:
            self._check("S", S, self._slot_state_shape(), torch.float32)
        N.call("dl_slot_load", self._h, int(slot), _ptr(S), self._stream(stream))

    def slot_merge(self, slot, stream=None):
        """Fold `slot`'s log into its base now (eviction / checkpoint)."""
        N.call("dl_slot_merge", self._h, int(slot), self._stream(stream))

    def slot_read(self, slot, out=None, stream=None):
        """Logical state of `slot` as [H, d_k, d_v] fp32 (the handle is unchanged)."""
        if out is None:
            out = torch.empty(self._slot_state_shape(), dtype=torch.float32, device=self.device)
        self._check("out", out, self._slot_state_shape(), torch.float32)
        N.call("dl_slot_read", self._h, int(slot), _ptr(out), self._stream(stream))
        return out

    def check_device(self, stream=None):
        N.call("dl_check_device", self._h, self._stream(stream))

    def close(self):
        if self._h:
            N.call("dl_destroy", self._h)
            self._h = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()
