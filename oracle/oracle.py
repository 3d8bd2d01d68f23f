"""ctypes front end of the fp64 CPU oracle (``fwpkm_oracle.c``).

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py``.  The library path never imports it.

Every array is handed to C as contiguous float64 (inputs widened exactly from
fp32 / bf16) or int64.  See ``fwpkm_oracle.c`` for the method, its sources and
the readings taken where the pages are silent.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "fwpkm_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

_dp = ctypes.POINTER(ctypes.c_double)
_ip = ctypes.POINTER(ctypes.c_int64)
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (fp64, OpenMP over token-heads)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-std=c11", "-shared", "-fPIC",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    if _lib is None:
        # FWPKM_ORACLE_LIB lets the mutation tests load a deliberately broken
        # copy of the oracle in a child process.
        path = os.environ.get("FWPKM_ORACLE_LIB") or build()
        L = ctypes.CDLL(path)
        i32, i64, f64 = ctypes.c_int, ctypes.c_int64, ctypes.c_double
        L.orc_num_threads.restype = i32
        L.orc_half_scores.argtypes = [_dp, _dp, i32, i32, f64, _dp, _dp]
        L.orc_half_scores_dot.argtypes = [_dp, _dp, i32, i32, _dp]
        L.orc_topk.argtypes = [_dp, i32, i32, _ip, _dp]
        L.orc_pk_select.argtypes = [_dp, _dp, i32, i32, _ip, _dp, _ip, _ip]
        L.orc_brute_select.argtypes = [_dp, _dp, i32, i32, _ip, _dp]
        L.orc_softmax.argtypes = [_dp, i32, _dp]
        L.orc_step.argtypes = [i64, i32, i32, i32, i32, i32, i32, f64, i32, _dp, _dp, i32,
                               i32, _dp, _dp, _dp, _dp, f64, f64, _dp, _ip, _dp, _dp, _ip, i32]
        L.orc_chunk_grads.argtypes = [i64, i32, i32, i32, i32, i32, i32, f64, i32, _dp, _dp,
                                      i32, i32, i32, i32, _dp, _dp, _dp, _dp, f64, _dp, _dp,
                                      _dp, _dp, _ip, _dp]
        L.orc_chunk_loss.argtypes = [i64, i32, i32, i32, i32, i32, f64, i32, _dp, _dp, i32,
                                     i32, i32, i32, _dp, _dp, _dp, _dp, f64, _ip]
        L.orc_chunk_loss.restype = f64
        _lib = L
    return _lib


def num_threads() -> int:
    return int(lib().orc_num_threads())


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float64)


def _p(a: Optional[np.ndarray]):
    if a is None:
        return None
    if a.dtype == np.float64:
        return a.ctypes.data_as(_dp)
    if a.dtype == np.int64:
        return a.ctypes.data_as(_ip)
    raise TypeError(a.dtype)


def _check(rc: int, what: str):
    if rc != 0:
        raise RuntimeError(f"oracle {what} failed with status {rc}")


# --------------------------------------------------------------------------
# Building blocks (exposed for the pins)
# --------------------------------------------------------------------------
def half_scores(q, K, eps):
    q, K = _f64(q), _f64(K)
    n, dh = K.shape
    s = np.empty(n)
    d = np.empty(n)
    lib().orc_half_scores(_p(q), _p(K), n, dh, eps, _p(s), _p(d))
    return s, d


def half_scores_dot(q, K):
    """The dot-product score q . K of one query half against a sub-key table."""
    q, K = _f64(q), _f64(K)
    n, dh = K.shape
    s = np.empty(n)
    lib().orc_half_scores_dot(_p(q), _p(K), n, dh, _p(s))
    return s


def topk(s, k):
    s = _f64(s)
    idx = np.empty(k, np.int64)
    val = np.empty(k)
    _check(lib().orc_topk(_p(s), len(s), k, _p(idx), _p(val)), "topk")
    return idx, val


def pk_select(s1, s2, k):
    s1, s2 = _f64(s1), _f64(s2)
    slot = np.empty(k, np.int64)
    sc = np.empty(k)
    ia = np.empty(k, np.int64)
    jb = np.empty(k, np.int64)
    _check(lib().orc_pk_select(_p(s1), _p(s2), len(s1), k, _p(slot), _p(sc), _p(ia), _p(jb)),
           "pk_select")
    return slot, sc, ia, jb


def brute_select(s1, s2, k):
    s1, s2 = _f64(s1), _f64(s2)
    slot = np.empty(k, np.int64)
    sc = np.empty(k)
    _check(lib().orc_brute_select(_p(s1), _p(s2), len(s1), k, _p(slot), _p(sc)), "brute")
    return slot, sc


def softmax(s):
    s = _f64(s)
    w = np.empty_like(s)
    lib().orc_softmax(_p(s), len(s), _p(w))
    return w


def lookahead_targets(Vt, weight):
    """Targets and token weights of the lookahead pairing q_t -> v_{t+1}
    (gist.science section 2, lookahead targets): token t < T-1 takes the
    next token's target; the last token of the call has none, so its weight
    is 0 (it is still read)."""
    Vt, weight = _f64(Vt), _f64(weight)
    shifted = Vt.copy()
    shifted[:, :-1] = Vt[:, 1:]
    w = weight.copy()
    w[:, -1] = 0.0
    return shifted, w


# --------------------------------------------------------------------------
# Memory state and the step
# --------------------------------------------------------------------------
# Options of two readings (fwpkm_oracle.c): how head readouts combine and what
# a value row's gradient is divided by.
HEADS = {"mean": 0, "sum": 1}
AGG = {"weight": 0, "count": 2, "sum": 4}
SCORE = {"idw": 0, "dot": 8}


class State:
    """fp64 copy of the fast weights: K [H][2][n][dq/2], V [N][dv].

    ``heads``: "mean" (head readouts averaged, the default reading) or "sum".
    ``agg``: a value row's gradient divided by its row contribution C_i =
    sum of w/H ("weight", the default), by its access count ("count"), or not
    divided ("sum").  ``score``: the sub-key score, "idw" (-log(eps + |q -
    K|^2), the default) or "dot" (q . K)."""

    def __init__(self, subkeys, values, *, topk: int, chunk: int, eps: float = 1e-3,
                 heads: str = "mean", agg: str = "weight", score: str = "idw"):
        self.K = _f64(subkeys).copy()
        self.V = _f64(values).copy()
        self.H, two, self.n, self.dh = self.K.shape
        assert two == 2
        self.N, self.dv = self.V.shape
        self.dq = 2 * self.dh
        self.topk, self.chunk, self.eps = topk, chunk, eps
        self.variant = HEADS[heads] | AGG[agg] | SCORE[score]

    def copy(self) -> "State":
        s = State.__new__(State)
        s.__dict__.update(self.__dict__)
        s.K = self.K.copy()
        s.V = self.V.copy()
        return s

    def _dims(self):
        return (self.N, self.n, self.dq, self.dv, self.topk, self.chunk, self.H, self.eps,
                self.variant)

    def step(self, Q, Vt, gate, eta: float, lam: float, *, want_sel: bool = False,
             want_gap: bool = False, max_chunks: int = 0, omega=None,
             lookahead: bool = False) -> dict:
        """Run the chunk loop over one call; updates the state in place.

        Q [B][T][H*dq], Vt [B][T][dv], gate [B][T] (any float dtype; widened).
        ``max_chunks`` > 0 stops after that many chunks (outputs of later
        tokens stay zero).  ``omega`` [B][T]: the MSE weight of each token
        (default: the gate).  ``lookahead``: query q_t is written towards
        target v_{t+1} (gist.science section 2, lookahead targets); the last
        token of the call has no target and gets weight 0.
        """
        Q, Vt, gate = _f64(Q), _f64(Vt), _f64(gate)
        B, T = gate.shape
        omega = None if omega is None else _f64(omega).copy()
        if lookahead:
            Vt, omega = lookahead_targets(Vt, gate if omega is None else omega)
        assert Q.shape == (B, T, self.H * self.dq) and Vt.shape == (B, T, self.dv)
        out = np.zeros((B, T, self.dv))
        k, H = self.topk, self.H
        sel = np.full((B, T, H, k), -1, np.int64) if want_sel else None
        selw = np.zeros((B, T, H, k)) if want_sel else None
        gap = np.full((B, T, H), np.nan) if want_gap else None
        n_chunks = -(-T // self.chunk)
        touched = np.zeros(n_chunks, np.int64)
        rc = lib().orc_step(*self._dims(), _p(self.K), _p(self.V), B, T, _p(Q), _p(Vt),
                            _p(gate), _p(omega), eta, lam, _p(out), _p(sel), _p(selw),
                            _p(gap), _p(touched), max_chunks)
        _check(rc, "step")
        return {"out": out, "sel_slot": sel, "sel_w": selw, "gap": gap, "touched": touched}

    def chunk_grads(self, Q, Vt, gate, lam: float, t0: int, Tc: int, omega=None) -> dict:
        """Raw gradients of one chunk without updating (dense; tiny shapes)."""
        Q, Vt, gate = _f64(Q), _f64(Vt), _f64(gate)
        omega = None if omega is None else _f64(omega)
        B, T = gate.shape
        dLdV = np.zeros((self.N, self.dv))
        dLdK = np.zeros_like(self.K)
        pbar = np.zeros(self.N)
        loss = np.zeros(1)
        sel = np.full((B, Tc, self.H, self.topk), -1, np.int64)
        selw = np.zeros((B, Tc, self.H, self.topk))
        # orc_chunk writes the selection at [b][t0 + tl]; give it a full-T view.
        sel_full = np.full((B, T, self.H, self.topk), -1, np.int64)
        selw_full = np.zeros((B, T, self.H, self.topk))
        rc = lib().orc_chunk_grads(*self._dims(), _p(self.K), _p(self.V), B, T, t0, Tc,
                                   _p(Q), _p(Vt), _p(gate), _p(omega), lam, _p(dLdV), _p(dLdK),
                                   _p(pbar), _p(loss), _p(sel_full), _p(selw_full))
        _check(rc, "chunk_grads")
        sel[:] = sel_full[:, t0:t0 + Tc]
        selw[:] = selw_full[:, t0:t0 + Tc]
        return {"dLdV": dLdV, "dLdK": dLdK, "pbar": pbar, "loss": float(loss[0]),
                "sel_slot": sel, "sel_w": selw}

    def chunk_loss(self, Q, Vt, gate, lam: float, t0: int, Tc: int, slots,
                   omega=None) -> float:
        """Loss of one chunk for a frozen selection ``slots`` [B][Tc][H][k]."""
        Q, Vt, gate = _f64(Q), _f64(Vt), _f64(gate)
        omega = None if omega is None else _f64(omega)
        B, T = gate.shape
        slots = np.ascontiguousarray(slots, dtype=np.int64)
        return float(lib().orc_chunk_loss(self.N, self.n, self.dq, self.dv, self.topk, self.H,
                                          self.eps, self.variant, _p(self.K), _p(self.V), B,
                                          T, t0, Tc,
                                          _p(Q), _p(Vt), _p(gate), _p(omega), lam,
                                          _p(slots)))
