"""The oracle against hand-worked examples stored under ``tests/golden/``.

Each fixture states its inputs and every expected value as exact fractions,
with the derivation written out in its comments, so that the values come from
arithmetic done by hand, not from any code.  The oracle is fp64, so it must
agree to rounding.
"""
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import yaml

from oracle import oracle

HERE = os.path.join(os.path.dirname(__file__), "golden")


def _f(x) -> float:
    return float(Fraction(str(x)))


def _arr(x) -> np.ndarray:
    if isinstance(x, list):
        return np.array([_arr(v) for v in x])
    return np.float64(_f(x))


def _key(s: str):
    return tuple(int(v) for v in s.split(","))


def _load(name):
    with open(os.path.join(HERE, name)) as fh:
        return yaml.safe_load(fh)


@pytest.fixture(scope="module")
def three_tokens():
    g = _load("hand_step_three_tokens.yaml")
    sh = g["shape"]
    H, n, dv = sh["heads"], sh["n"], sh["dv"]
    K = _arr(g["inputs"]["subkeys"])
    assert K.shape == (H, 2, n, sh["dq"] // 2)
    V = np.array([[float(r), 1.0] for r in range(n * n)])
    for r, row in g["inputs"]["values_read"].items():
        V[int(r)] = _arr(row)
    return g, K, V


def _state(g, K, V):
    sh = g["shape"]
    return oracle.State(K, V, topk=sh["topk"], chunk=sh["chunk"], eps=_f(sh["eps"]))


def _inputs(g):
    i = g["inputs"]
    return _arr(i["Q"]), _arr(i["Vtarget"]), _arr(i["gate"])


RTOL = 1e-12


def test_hand_step_selection_readout_and_update(three_tokens):
    g, K, V = three_tokens
    exp = g["expected"]
    st = _state(g, K, V)
    Q, Vt, gate = _inputs(g)
    res = st.step(Q, Vt, gate, _f(g["eta"]), _f(g["lambda"]), want_sel=True, want_gap=True)

    assert np.array_equal(res["sel_slot"], np.array(exp["sel_slot"]))
    np.testing.assert_allclose(res["sel_w"], _arr(exp["sel_w"]), rtol=RTOL)
    gap = np.vectorize(math.log)(_arr(exp["gap_log"]))
    np.testing.assert_allclose(res["gap"], gap, rtol=RTOL)
    np.testing.assert_allclose(res["out"], _arr(exp["out"]), rtol=RTOL)

    V_after = V.copy()
    for r, row in exp["values_after"].items():
        V_after[int(r)] = _arr(row)
    np.testing.assert_allclose(st.V, V_after, rtol=RTOL, atol=0)
    K_after = K.copy()
    for key, row in exp["subkeys_after"].items():
        K_after[_key(key)] = _arr(row)
    np.testing.assert_allclose(st.K, K_after, rtol=RTOL, atol=1e-15)


def test_hand_step_gradients_loss_and_marginal(three_tokens):
    g, K, V = three_tokens
    exp = g["expected"]
    st = _state(g, K, V)
    Q, Vt, gate = _inputs(g)
    gr = st.chunk_grads(Q, Vt, gate, _f(g["lambda"]), 0, g["shape"]["chunk"])

    assert gr["loss"] == pytest.approx(sum(_f(x) for x in exp["loss"]), rel=RTOL)
    pbar = np.zeros(st.N)
    for r, p in exp["pbar"].items():
        pbar[int(r)] = _f(p)
    np.testing.assert_allclose(gr["pbar"], pbar, rtol=RTOL, atol=0)
    dK = np.zeros_like(K)
    for key, row in exp["dLdK"].items():
        dK[_key(key)] = _arr(row)
    np.testing.assert_allclose(gr["dLdK"], dK, rtol=RTOL, atol=1e-15)
    # the state is not touched by the gradient query
    assert np.array_equal(st.K, K) and np.array_equal(st.V, V)


def _log_sum(terms) -> float:
    return sum(_f(c) * math.log(_f(p)) for c, p in terms)


def test_hand_step_entropy_term(three_tokens):
    g, K, V = three_tokens
    ent = g["entropy"]
    lam = _f(ent["lambda"])
    Q, Vt, gate = _inputs(g)
    chunk = g["shape"]["chunk"]
    gr0 = _state(g, K, V).chunk_grads(Q, Vt, gate, 0.0, 0, chunk)
    gr = _state(g, K, V).chunk_grads(Q, Vt, gate, lam, 0, chunk)

    delta = np.zeros_like(K)
    for key, coords in ent["dLdK_per_lambda"].items():
        delta[_key(key)] = [lam * _log_sum(t) for t in coords]
    np.testing.assert_allclose(gr["dLdK"] - gr0["dLdK"], delta, rtol=1e-10, atol=1e-15)
    assert gr["loss"] - gr0["loss"] == pytest.approx(
        lam * _log_sum(ent["loss_per_lambda"]), rel=1e-10)
    # the entropy term reaches the sub-keys only
    np.testing.assert_array_equal(gr["dLdV"], gr0["dLdV"])

    st = _state(g, K, V)
    st.step(Q, Vt, gate, _f(g["eta"]), lam)
    V_after = V.copy()
    for r, row in g["expected"]["values_after"].items():
        V_after[int(r)] = _arr(row)
    np.testing.assert_allclose(st.V, V_after, rtol=RTOL, atol=0)
