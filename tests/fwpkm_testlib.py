"""Helpers of the GPU-vs-oracle parity tests.

Tolerances (stated for the step as a whole):
  * selected slot sets identical for every token-head whose oracle gap between
    the k-th and (k+1)-th best slot score exceeds TIE_GAP = 1e-5 (IDW score,
    a log: a relative gap of the distances); with the dot-product score the
    gap is absolute, and the fp32 error of a dot product grows with the norms,
    so there the bound is TIE_GAP * max |q_half| * 2 max |K_row| of the
    inputs (the factor 2 for sub-keys that grow by their updates);
  * outputs: |out_gpu - out_ref| <= 1e-5 + 1e-4 |out_ref| element-wise;
  * tables:  |X_gpu - X_ref| <= tol |X_ref| + tol rms(X_ref) element-wise, tol =
    1e-4 after one chunk and 1e-3 after more (64 and beyond).

Near ties.  Where the oracle's gap is <= TIE_GAP both selections are correct,
and an fp32 path may take either.  For multi-chunk runs the GPU is told to
read the ORACLE's choice at exactly those token-heads (fwpkm_force_selection,
oracle -> GPU only), so both trajectories stay comparable; everywhere else the
GPU decides by itself and must agree.  The single-chunk tests run without any
forcing and check that a differing GPU choice is a valid one.
"""
from __future__ import annotations

import dataclasses
from typing import List, Optional

import numpy as np

from sparse_weight_memory_b200.workloads import BF16, Inputs, Workload, bf16_bits_to_f32

TIE_GAP = 1e-5
OUT_ATOL, OUT_RTOL = 1e-5, 1e-4


def widen(a: np.ndarray) -> np.ndarray:
    if a.dtype == np.uint16:
        return bf16_bits_to_f32(a).astype(np.float64)
    return a.astype(np.float64)


def to_dev(a: np.ndarray):
    import torch
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).cuda().view(torch.bfloat16)
    return torch.from_numpy(a).cuda()


def schedule(wl: Workload, inp: Inputs, omega=None):
    """The calls of one workload step: chained segments, each read `passes`
    times; (Q, Vt, gate, omega) per call (omega None unless given)."""
    calls = []
    for c in range(wl.calls):
        sl = slice(c * wl.T, (c + 1) * wl.T)
        seg = (inp.Q[:, sl], inp.Vt[:, sl], inp.gate[:, sl],
               None if omega is None else omega[:, sl])
        for _ in range(wl.passes):
            calls.append(seg)
    return calls


@dataclasses.dataclass
class RunResult:
    outs: List[np.ndarray]
    sels: List[np.ndarray]
    ws: List[np.ndarray]
    gaps: List[Optional[np.ndarray]]
    K: np.ndarray
    V: np.ndarray
    touched: Optional[int] = None


def oracle_run(wl: Workload, inp: Inputs, oracle, max_chunks: int = 0,
               state=None, omega=None, tables: bool = True) -> RunResult:
    """Oracle over the workload's calls; continues `state` in place if given.
    ``omega`` [B][T_total]: the tokens' MSE weights (default: the gate).
    ``tables=False``: K and V of the result are None (read them from `state`)."""
    st = state if state is not None else oracle.State(inp.subkeys, inp.values, topk=wl.topk,
                                                      chunk=wl.chunk, eps=wl.eps,
                                                      heads=wl.heads_mode, agg=wl.agg,
                                                      score=wl.score)
    outs, sels, ws, gaps, touched = [], [], [], [], 0
    for Q, Vt, g, om in schedule(wl, inp, omega):
        r = st.step(widen(Q), widen(Vt), g, wl.eta, wl.lam, want_sel=True, want_gap=True,
                    max_chunks=max_chunks, omega=om, lookahead=wl.lookahead)
        outs.append(r["out"])
        sels.append(r["sel_slot"])
        ws.append(r["sel_w"])
        gaps.append(r["gap"])
        touched += int(r["touched"].sum())
    K = V = None
    if tables:
        K, V = (st.K.copy(), st.V.copy()) if state is not None else (st.K, st.V)
    return RunResult(outs, sels, ws, gaps, K, V, touched)


def gpu_run(wl: Workload, inp: Inputs, ref: Optional[RunResult] = None, force: bool = True,
            K0=None, V0=None, with_stats: bool = False, omega=None, state=None,
            tables: bool = True) -> RunResult:
    """Run the workload through the C ABI.  With `ref` and `force`, token-heads
    where the oracle has a near tie read the oracle's slots.  ``omega`` as in
    oracle_run; the workload's lookahead flag is passed on.  ``state``: an
    existing FwPKMState with its tables already set (the caller keeps it);
    ``tables=False`` leaves the tables on the device (K and V are None)."""
    import torch

    from sparse_weight_memory_b200 import FwPKMState
    st = state
    if st is None:
        st = FwPKMState(wl.N, wl.dq, wl.dv, wl.topk, wl.chunk, wl.heads, eps=wl.eps)
        st.set_options(heads=wl.heads_mode, agg=wl.agg, score=wl.score)
        st.set_tables(to_dev(inp.subkeys if K0 is None else K0),
                      to_dev(inp.values if V0 is None else V0))
    if with_stats:
        st.read_stats(reset=True)
    outs, sels, ws, keep = [], [], [], []
    for i, (Q, Vt, g, om) in enumerate(schedule(wl, inp, omega)):
        B, T = g.shape
        rs = torch.empty((B, T, wl.heads, wl.topk), dtype=torch.int32, device="cuda")
        rw = torch.empty((B, T, wl.heads, wl.topk), dtype=torch.float32, device="cuda")
        st.record_selection(rs, rw)
        if ref is not None and force:
            mask = to_dev((ref.gaps[i] <= tie_gap(wl, inp)).astype(np.uint8))
            slots = to_dev(ref.sels[i].astype(np.int32))
            st.force_selection(slots, mask)
            keep += [mask, slots]
        om_d = None if om is None else to_dev(np.ascontiguousarray(om, dtype=np.float32))
        out = st.step(to_dev(Q), to_dev(Vt), to_dev(g), wl.eta, wl.lam, omega=om_d,
                      lookahead=wl.lookahead)
        keep += [rs, rw, out, om_d]
        outs.append(out)
        sels.append(rs)
        ws.append(rw)
    torch.cuda.synchronize()
    K = V = None
    if tables:
        K, V = st.get_tables()
        torch.cuda.synchronize()
        K, V = K.cpu().numpy(), V.cpu().numpy()
    touched = None
    if with_stats:
        stats = st.read_stats()
        assert stats["device_errors"] == 0
        touched = stats["value_rows"]
    res = RunResult([o.cpu().numpy() for o in outs], [s.cpu().numpy() for s in sels],
                    [w.cpu().numpy() for w in ws], [None] * len(outs), K, V, touched)
    if state is None:
        st.close()
    return res


# ---------------------------------------------------------------------------
# comparisons
# ---------------------------------------------------------------------------
def tie_gap(wl: Workload, inp: Inputs) -> float:
    """The near-tie bound of the workload's score (see the module docstring)."""
    if wl.score != "dot":
        return TIE_GAP
    q = inp.q_f32().reshape(-1, 2 * wl.heads, wl.dh)
    qmax = float(np.sqrt((q.astype(np.float64) ** 2).sum(-1)).max())
    kmax = float(np.sqrt((inp.subkeys.astype(np.float64) ** 2).sum(-1)).max())
    return TIE_GAP * qmax * 2.0 * kmax


def check_selection(sel_g, sel_o, gap_o, what="", gap=TIE_GAP):
    """Slot sets equal wherever the oracle gap exceeds ``gap``."""
    a = np.sort(sel_g.astype(np.int64), axis=-1)
    b = np.sort(sel_o, axis=-1)
    ok = gap_o > gap
    diff = (a != b).any(axis=-1)
    bad = diff & ok
    assert not bad.any(), (f"{what}: {int(bad.sum())} token-heads select different slots with "
                           f"gap > {gap}; first at {np.argwhere(bad)[0]}")
    return diff


def check_close(x_g, x_o, atol, rtol, what=""):
    err = np.abs(x_g.astype(np.float64) - x_o)
    lim = atol + rtol * np.abs(x_o)
    bad = err > lim
    assert not bad.any(), (f"{what}: {int(bad.sum())} of {bad.size} elements outside "
                           f"{atol} + {rtol}|ref|; worst err {err.max():.3g} at "
                           f"{np.unravel_index(np.argmax(err - lim), err.shape)}")


def check_table(x_g, x_o, tol, what="", exclude_rows=None):
    x_o2 = x_o.reshape(-1, x_o.shape[-1])
    x_g2 = x_g.reshape(-1, x_g.shape[-1]).astype(np.float64)
    rms = float(np.sqrt(np.mean(x_o2 ** 2)))
    err = np.abs(x_g2 - x_o2)
    bad = err > tol * np.abs(x_o2) + tol * rms
    if exclude_rows is not None and len(exclude_rows):
        bad[np.asarray(sorted(exclude_rows))] = False
    assert not bad.any(), (f"{what}: {int(bad.any(axis=1).sum())} rows outside tol {tol}; "
                           f"worst abs err {err.max():.3g} (rms {rms:.3g})")


def update_rel_error(x_g, x_o, x0):
    """Relative Frobenius error of the update X_after - X_before."""
    du_o = x_o - x0.astype(np.float64)
    du_g = x_g.astype(np.float64) - x0.astype(np.float64)
    den = np.linalg.norm(du_o)
    return float(np.linalg.norm(du_g - du_o) / den) if den > 0 else 0.0


def table_tol(wl: Workload, T: int) -> float:
    chunks = wl.n_chunks(T) * wl.calls * wl.passes
    return 1e-4 if chunks <= 1 else 1e-3


def compare_runs(wl: Workload, inp: Inputs, g: RunResult, o: RunResult, what: str = ""):
    T = inp.gate.shape[1] // wl.calls
    tg = tie_gap(wl, inp)
    for i in range(len(o.outs)):
        check_selection(g.sels[i], o.sels[i], o.gaps[i], f"{what} call {i} selection", tg)
        check_close(g.outs[i], o.outs[i], OUT_ATOL, OUT_RTOL, f"{what} call {i} out")
    tol = table_tol(wl, T)
    check_table(g.V, o.V, tol, f"{what} values")
    check_table(g.K, o.K, tol, f"{what} sub-keys")
    info = {"dV_rel": update_rel_error(g.V, o.V, inp.values),
            "dK_rel": update_rel_error(g.K, o.K, inp.subkeys),
            "near_ties": int(sum((x <= tg).sum() for x in o.gaps))}
    # the achieved errors, so that a drift shows long before it reaches a bound
    out_ratio = max(float((np.abs(g.outs[i].astype(np.float64) - o.outs[i]) /
                           (OUT_ATOL + OUT_RTOL * np.abs(o.outs[i]))).max())
                    for i in range(len(o.outs)))
    print(f"{what}: worst out err / bound {out_ratio:.3f}, update rel err V {info['dV_rel']:.2e} "
          f"K {info['dK_rel']:.2e}, near ties {info['near_ties']}")
    return info
