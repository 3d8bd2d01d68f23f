"""Thin ctypes binding of libfwpkm.so (declared in include/fwpkm.h).

Argument marshalling only: every step of the memory read and write runs in
the library's CUDA kernels.  PyTorch supplies device memory and streams.  If
the library is missing the import of a state fails loudly -- there is no CPU
or library fallback.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfwpkm.so")

FWPKM_OK, FWPKM_EINVAL, FWPKM_ESHAPE, FWPKM_ENOMEM, FWPKM_ECUDA, FWPKM_EUNSUPPORTED = (
    0, -1, -2, -3, -4, -5)
FWPKM_F32, FWPKM_BF16 = 0, 1
FWPKM_LOOKAHEAD = 1
FWPKM_HEADS_SUM, FWPKM_AGG_COUNT, FWPKM_AGG_SUM, FWPKM_SCORE_DOT = 1, 2, 4, 8
STATUS_NAMES = {0: "OK", -1: "EINVAL", -2: "ESHAPE", -3: "ENOMEM", -4: "ECUDA",
                -5: "EUNSUPPORTED"}

_lib = None
_vp = ctypes.c_void_p


class FwpkmError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


def load_library():
    """Load libfwpkm.so (built by ``python -m sparse_weight_memory_b200.build``)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                           "`python -m sparse_weight_memory_b200.build` (nvcc, sm_100a)")
    L = ctypes.CDLL(LIB_PATH)
    i32, i64, f32, u32p = ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.POINTER(ctypes.c_uint32)
    i64p = ctypes.POINTER(ctypes.c_int64)
    L.fwpkm_last_error.restype = ctypes.c_char_p
    L.fwpkm_state_init.argtypes = [i64, i32, i32, i32, i32, i32, ctypes.POINTER(_vp)]
    L.fwpkm_state_init_batched.argtypes = [i64, i32, i32, i32, i32, i32, i32,
                                           ctypes.POINTER(_vp)]
    L.fwpkm_state_free.argtypes = [_vp]
    L.fwpkm_state_free.restype = None
    L.fwpkm_state_set_eps.argtypes = [_vp, f32]
    L.fwpkm_step.argtypes = [_vp, i32, i32, _vp, i32, _vp, i32, _vp, f32, f32, _vp, _vp]
    L.fwpkm_step_host.argtypes = [_vp, i32, i32, _vp, i32, _vp, i32, _vp, f32, f32, _vp, _vp]
    L.fwpkm_step_ex.argtypes = [_vp, i32, i32, _vp, i32, _vp, i32, _vp, _vp, i32, f32, f32, _vp,
                                _vp]
    L.fwpkm_step_host_ex.argtypes = L.fwpkm_step_ex.argtypes
    L.fwpkm_state_get.argtypes = [_vp, _vp, _vp, _vp]
    L.fwpkm_state_set.argtypes = [_vp, _vp, _vp, _vp]
    L.fwpkm_record_selection.argtypes = [_vp, _vp, _vp]
    L.fwpkm_force_selection.argtypes = [_vp, _vp, _vp]
    L.fwpkm_set_profiling.argtypes = [_vp, i32]
    L.fwpkm_set_graphs.argtypes = [_vp, i32]
    L.fwpkm_profile_read.argtypes = [_vp, ctypes.POINTER(ctypes.c_char_p),
                                     ctypes.POINTER(ctypes.c_double), i64p, i32,
                                     ctypes.POINTER(i32), _vp]
    L.fwpkm_read_stats.argtypes = [_vp, i64p, i64p, i64p, i64p, u32p, i32, _vp]
    L.fwpkm_select_noalloc.argtypes = [_vp, i32, i32, _vp, i32, _vp, _vp, _vp, _vp]
    L.fwpkm_set_wait_limits.argtypes = [_vp, i64, i64]
    L.fwpkm_state_set_options.argtypes = [_vp, ctypes.c_uint]
    L.fwpkm_inject_alloc_failures.argtypes = [i32]
    L.fwpkm_inject_alloc_failures.restype = None
    for name in ("fwpkm_state_init", "fwpkm_state_init_batched", "fwpkm_state_set_eps",
                 "fwpkm_step", "fwpkm_step_host",
                 "fwpkm_step_ex", "fwpkm_step_host_ex",
                 "fwpkm_state_get", "fwpkm_state_set", "fwpkm_record_selection",
                 "fwpkm_force_selection", "fwpkm_set_profiling", "fwpkm_profile_read",
                 "fwpkm_read_stats", "fwpkm_select_noalloc", "fwpkm_set_graphs",
                 "fwpkm_set_wait_limits", "fwpkm_state_set_options"):
        getattr(L, name).restype = i32
    _lib = L
    return L


def inject_alloc_failures(count: int):
    """Make the library's next ``count`` device allocations fail (ENOMEM)."""
    load_library().fwpkm_inject_alloc_failures(int(count))


def _check(rc: int):
    if rc != FWPKM_OK:
        raise FwpkmError(rc, load_library().fwpkm_last_error().decode())


def _ptr(t) -> Optional[int]:
    """Device (torch) or host (numpy) buffer address; None passes NULL."""
    if t is None:
        return None
    if isinstance(t, np.ndarray):
        assert t.flags["C_CONTIGUOUS"], "host arrays must be C-contiguous"
        return t.ctypes.data
    assert t.is_contiguous(), "tensors must be contiguous"
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return getattr(stream, "cuda_stream", stream)


def _dtype_code(t) -> int:
    import torch
    if isinstance(t, np.ndarray):
        if t.dtype == np.float32:
            return FWPKM_F32
        if t.dtype == np.uint16:  # bfloat16 bit patterns
            return FWPKM_BF16
        raise TypeError(f"unsupported host dtype {t.dtype}")
    if t.dtype == torch.float32:
        return FWPKM_F32
    if t.dtype == torch.bfloat16:
        return FWPKM_BF16
    raise TypeError(f"unsupported dtype {t.dtype}")


class FwPKMState:
    """One fast-weight product-key memory (sub-key tables + value table).

    Mirrors fwpkm_state_init / step / get / set of include/fwpkm.h.  With
    ``memories`` > 1 the state holds one memory per sequence
    (fwpkm_state_init_batched): a step's B must equal ``memories``.
    """

    def __init__(self, N: int, dq: int, dv: int, topk: int, chunk: int, heads: int = 1,
                 eps: float = 1e-3, memories: int = 1):
        L = load_library()
        h = _vp()
        if memories == 1:
            _check(L.fwpkm_state_init(N, dq, dv, topk, chunk, heads, ctypes.byref(h)))
        else:
            _check(L.fwpkm_state_init_batched(N, dq, dv, topk, chunk, heads, memories,
                                              ctypes.byref(h)))
        self._h = h
        self.N, self.dq, self.dv, self.topk, self.chunk, self.heads = N, dq, dv, topk, chunk, heads
        self.memories = memories
        self.n = int(round(N ** 0.5))
        if eps != 1e-3:
            _check(L.fwpkm_state_set_eps(h, eps))
        self.eps = eps

    def close(self):
        if getattr(self, "_h", None):
            load_library().fwpkm_state_free(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # -- tables ------------------------------------------------------------
    def set_tables(self, subkeys=None, values=None, stream=None):
        _check(load_library().fwpkm_state_set(self._h, _ptr(subkeys), _ptr(values),
                                              _stream(stream)))

    def get_tables(self, subkeys=None, values=None, stream=None):
        """Copy the tables into the given buffers (allocates CUDA tensors if None)."""
        import torch
        lead = (self.memories,) if self.memories > 1 else ()
        if subkeys is None:
            subkeys = torch.empty(lead + (self.heads, 2, self.n, self.dq // 2),
                                  dtype=torch.float32, device="cuda")
        if values is None:
            values = torch.empty(lead + (self.N, self.dv), dtype=torch.float32, device="cuda")
        _check(load_library().fwpkm_state_get(self._h, _ptr(subkeys), _ptr(values),
                                              _stream(stream)))
        return subkeys, values

    # -- the step ----------------------------------------------------------
    def step(self, Q, Vt, gate, eta: float, lam: float = 0.0, out=None, stream=None,
             omega=None, lookahead: bool = False):
        """Device step: Q [B,T,H*dq], Vt [B,T,dv] (fp32 or bf16), gate [B,T] fp32.
        ``omega`` [B,T] fp32: the tokens' MSE weights (default: the gate);
        ``lookahead``: query t is written towards the target of token t+1."""
        import torch
        B, T = gate.shape
        if out is None:
            out = torch.empty((B, T, self.dv), dtype=torch.float32, device=gate.device)
        L = load_library()
        if omega is None and not lookahead:
            _check(L.fwpkm_step(self._h, B, T, _ptr(Q), _dtype_code(Q), _ptr(Vt),
                                _dtype_code(Vt), _ptr(gate), eta, lam, _ptr(out),
                                _stream(stream)))
        else:
            _check(L.fwpkm_step_ex(self._h, B, T, _ptr(Q), _dtype_code(Q), _ptr(Vt),
                                   _dtype_code(Vt), _ptr(gate), _ptr(omega),
                                   FWPKM_LOOKAHEAD if lookahead else 0, eta, lam, _ptr(out),
                                   _stream(stream)))
        return out

    def step_host(self, Q: np.ndarray, Vt: np.ndarray, gate: np.ndarray, eta: float,
                  lam: float = 0.0, out: Optional[np.ndarray] = None, stream=None,
                  omega: Optional[np.ndarray] = None, lookahead: bool = False):
        """Host-buffer step (copies in and out inside the call; synchronous)."""
        B, T = gate.shape
        if out is None:
            out = np.empty((B, T, self.dv), dtype=np.float32)
        L = load_library()
        if omega is None and not lookahead:
            _check(L.fwpkm_step_host(self._h, B, T, _ptr(Q), _dtype_code(Q), _ptr(Vt),
                                     _dtype_code(Vt), _ptr(gate), eta, lam, _ptr(out),
                                     _stream(stream)))
        else:
            _check(L.fwpkm_step_host_ex(self._h, B, T, _ptr(Q), _dtype_code(Q), _ptr(Vt),
                                        _dtype_code(Vt), _ptr(gate), _ptr(omega),
                                        FWPKM_LOOKAHEAD if lookahead else 0, eta, lam,
                                        _ptr(out), _stream(stream)))
        return out

    # -- selection record / replay ---------------------------------------
    def record_selection(self, slots=None, weights=None):
        _check(load_library().fwpkm_record_selection(self._h, _ptr(slots), _ptr(weights)))

    def force_selection(self, slots=None, mask=None):
        _check(load_library().fwpkm_force_selection(self._h, _ptr(slots), _ptr(mask)))

    def select_noalloc(self, Q, slots, weights, errors=None, stream=None):
        """Selection only (slots, weights) into caller buffers; allocates nothing.
        ``errors``: optional one-element uint32 buffer (device tensor or host
        array) that receives the call's device error bits."""
        B, T = Q.shape[0], Q.shape[1]
        _check(load_library().fwpkm_select_noalloc(self._h, B, T, _ptr(Q), _dtype_code(Q),
                                                   _ptr(slots), _ptr(weights), _ptr(errors),
                                                   _stream(stream)))
        return slots, weights

    def set_options(self, heads: str = "mean", agg: str = "weight", score: str = "idw"):
        """Readings of the step: ``heads`` "mean" or "sum"; ``agg`` (divisor
        of a value row's gradient) "weight", "count" or "sum"; ``score``
        (sub-key score) "idw" or "dot"."""
        opts = {"mean": 0, "sum": FWPKM_HEADS_SUM}[heads] | \
            {"weight": 0, "count": FWPKM_AGG_COUNT, "sum": FWPKM_AGG_SUM}[agg] | \
            {"idw": 0, "dot": FWPKM_SCORE_DOT}[score]
        _check(load_library().fwpkm_state_set_options(self._h, opts))

    def set_wait_limits(self, mbar_polls: int = -1, scan_polls: int = -1):
        """Bounds of the device-side waits (negative = the default)."""
        _check(load_library().fwpkm_set_wait_limits(self._h, mbar_polls, scan_polls))

    def set_graphs(self, enable: bool):
        """Replay repeated calls as CUDA graphs (default on)."""
        _check(load_library().fwpkm_set_graphs(self._h, int(bool(enable))))

    # -- measurement -------------------------------------------------------
    def set_profiling(self, enable: bool):
        _check(load_library().fwpkm_set_profiling(self._h, int(bool(enable))))

    def profile_read(self, stream=None) -> dict:
        names = (ctypes.c_char_p * 16)()
        ms = (ctypes.c_double * 16)()
        n = (ctypes.c_int64 * 16)()
        cnt = ctypes.c_int(0)
        _check(load_library().fwpkm_profile_read(self._h, names, ms, n, 16, ctypes.byref(cnt),
                                                 _stream(stream)))
        return {names[i].decode(): (ms[i], n[i]) for i in range(cnt.value)}

    def read_stats(self, reset: bool = False, stream=None) -> dict:
        c, v, k, r = ctypes.c_int64(), ctypes.c_int64(), ctypes.c_int64(), ctypes.c_int64()
        err = ctypes.c_uint32()
        _check(load_library().fwpkm_read_stats(self._h, ctypes.byref(c), ctypes.byref(v),
                                               ctypes.byref(k), ctypes.byref(r), ctypes.byref(err),
                                               int(reset), _stream(stream)))
        return {"chunks": c.value, "value_rows": v.value, "key_rows": k.value, "records": r.value,
                "device_errors": err.value}
