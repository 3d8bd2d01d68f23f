"""The oracle against hand-worked examples stored under ``tests/golden/``.

Each fixture states its inputs and every expected value as exact fractions,
with the derivation written out in its comments, so that the values come from
arithmetic done by hand, not from any code.  The oracle is fp64, so it must
agree to rounding.
"""
import math

import numpy as np
import pytest

from oracle import oracle

from golden_lib import arr, frac, load_hand_step, log_sum, row_key

RTOL = 1e-12


FIXTURES = ["hand_step_three_tokens.yaml", "hand_step_two_heads.yaml"]


@pytest.fixture(scope="module", params=FIXTURES)
def hs(request):
    return load_hand_step(request.param)


def _state(hs):
    return oracle.State(hs.K, hs.V, topk=hs.topk, chunk=hs.chunk, eps=hs.eps)


def test_hand_step_selection_readout_and_update(hs):
    exp = hs.expected
    st = _state(hs)
    res = st.step(hs.Q, hs.Vt, hs.gate, hs.eta, frac(hs.raw["lambda"]), want_sel=True,
                  want_gap=True)

    assert np.array_equal(res["sel_slot"], np.array(exp["sel_slot"]))
    np.testing.assert_allclose(res["sel_w"], arr(exp["sel_w"]), rtol=RTOL)
    gap = np.vectorize(math.log)(arr(exp["gap_log"]))
    np.testing.assert_allclose(res["gap"], gap, rtol=RTOL)
    np.testing.assert_allclose(res["out"], arr(exp["out"]), rtol=RTOL)
    np.testing.assert_allclose(st.V, hs.values_after(), rtol=RTOL, atol=0)
    np.testing.assert_allclose(st.K, hs.subkeys_after(), rtol=RTOL, atol=1e-15)


def test_hand_step_gradients_loss_and_marginal(hs):
    exp = hs.expected
    st = _state(hs)
    gr = st.chunk_grads(hs.Q, hs.Vt, hs.gate, frac(hs.raw["lambda"]), 0, hs.chunk)

    assert gr["loss"] == pytest.approx(sum(frac(x) for x in exp["loss"]), rel=RTOL)
    np.testing.assert_allclose(gr["pbar"], hs.pbar(), rtol=RTOL, atol=0)
    np.testing.assert_allclose(gr["dLdK"], hs.dLdK(), rtol=RTOL, atol=1e-15)
    # the state is not touched by the gradient query
    assert np.array_equal(st.K, hs.K) and np.array_equal(st.V, hs.V)


def test_hand_step_entropy_term(hs):
    ent = hs.raw["entropy"]
    lam = frac(ent["lambda"])
    gr0 = _state(hs).chunk_grads(hs.Q, hs.Vt, hs.gate, 0.0, 0, hs.chunk)
    gr = _state(hs).chunk_grads(hs.Q, hs.Vt, hs.gate, lam, 0, hs.chunk)

    np.testing.assert_allclose(gr["dLdK"] - gr0["dLdK"], lam * hs.dLdK_per_lambda(),
                               rtol=1e-10, atol=1e-15)
    assert gr["loss"] - gr0["loss"] == pytest.approx(lam * log_sum(ent["loss_per_lambda"]),
                                                     rel=1e-10)
    # the entropy term reaches the sub-keys only
    np.testing.assert_array_equal(gr["dLdV"], gr0["dLdV"])

    st = _state(hs)
    st.step(hs.Q, hs.Vt, hs.gate, hs.eta, lam)
    np.testing.assert_allclose(st.V, hs.values_after(), rtol=RTOL, atol=0)
    np.testing.assert_allclose(st.K, hs.subkeys_after(lam), rtol=1e-10, atol=1e-15)


def test_hand_step_lookahead(hs):
    """The same step with the lookahead pairing q_t -> v_{t+1}: the reads are
    unchanged, the writes follow the hand-worked values."""
    la = hs.raw.get("lookahead")
    if la is None:
        pytest.skip("this example has no lookahead part")
    st = _state(hs)
    res = st.step(hs.Q, hs.Vt, hs.gate, hs.eta, 0.0, want_sel=True, lookahead=True)
    np.testing.assert_allclose(res["out"], arr(hs.expected["out"]), rtol=RTOL)
    V = hs.V.copy()
    for r, row in la["values_after"].items():
        V[int(r)] = arr(row)
    np.testing.assert_allclose(st.V, V, rtol=RTOL, atol=0)
    K = hs.K.copy()
    for key, row in la["subkeys_after"].items():
        K[row_key(key)] = arr(row)
    np.testing.assert_allclose(st.K, K, rtol=RTOL, atol=1e-15)
    # the raw gradient and the loss, through the targets and weights the pairing gives
    Vt, om = oracle.lookahead_targets(hs.Vt, hs.gate)
    gr = _state(hs).chunk_grads(hs.Q, Vt, hs.gate, 0.0, 0, hs.chunk, omega=om)
    assert gr["loss"] == pytest.approx(sum(frac(x) for x in la["loss"]), rel=RTOL)
    dK = np.zeros_like(hs.K)
    for key, row in la["dLdK"].items():
        dK[row_key(key)] = arr(row)
    np.testing.assert_allclose(gr["dLdK"], dK, rtol=RTOL, atol=1e-15)


@pytest.mark.parametrize("agg", ["count", "sum"])
def test_hand_step_other_row_divisors(hs, agg):
    """A value row's gradient divided by its access count, or not divided:
    reads and sub-keys as in the main step, value rows as worked by hand."""
    part = hs.raw.get("aggregation")
    if part is None:
        pytest.skip("this example has no aggregation part")
    st = oracle.State(hs.K, hs.V, topk=hs.topk, chunk=hs.chunk, eps=hs.eps, agg=agg)
    res = st.step(hs.Q, hs.Vt, hs.gate, hs.eta, 0.0)
    np.testing.assert_allclose(res["out"], arr(hs.expected["out"]), rtol=RTOL)
    V = hs.V.copy()
    for r, row in part[agg]["values_after"].items():
        V[int(r)] = arr(row)
    np.testing.assert_allclose(st.V, V, rtol=RTOL, atol=0)
    np.testing.assert_allclose(st.K, hs.subkeys_after(), rtol=RTOL, atol=1e-15)


def test_hand_step_summed_heads(hs):
    """The head readouts summed, not averaged (the 1/H of the readout, of its
    gradients and of C_i goes): read, loss, dL/dK and both updated tables."""
    part = hs.raw.get("heads_sum")
    if part is None:
        pytest.skip("this example has no summed-heads part")
    st = oracle.State(hs.K, hs.V, topk=hs.topk, chunk=hs.chunk, eps=hs.eps, heads="sum")
    gr = st.chunk_grads(hs.Q, hs.Vt, hs.gate, 0.0, 0, hs.chunk)
    assert gr["loss"] == pytest.approx(sum(frac(x) for x in part["loss"]), rel=RTOL)
    dK = np.zeros_like(hs.K)
    for key, row in part["dLdK"].items():
        dK[row_key(key)] = arr(row)
    np.testing.assert_allclose(gr["dLdK"], dK, rtol=RTOL, atol=1e-15)
    res = st.step(hs.Q, hs.Vt, hs.gate, hs.eta, 0.0, want_sel=True)
    assert np.array_equal(res["sel_slot"], np.array(hs.expected["sel_slot"]))
    np.testing.assert_allclose(res["out"], arr(part["out"]), rtol=RTOL)
    V = hs.V.copy()
    for r, row in part["values_after"].items():
        V[int(r)] = arr(row)
    np.testing.assert_allclose(st.V, V, rtol=RTOL, atol=0)
    K = hs.K.copy()
    for key, row in part["subkeys_after"].items():
        K[row_key(key)] = arr(row)
    np.testing.assert_allclose(st.K, K, rtol=RTOL, atol=1e-15)


def test_hand_step_dot_product_score(hs):
    """The dot-product sub-key score: selection (ties by slot), gap, read,
    loss, dL/dK (ds/dK = q) and both updated tables, as worked by hand."""
    part = hs.raw.get("dot_score")
    if part is None:
        pytest.skip("this example has no dot-product part")
    Q = arr(part["Q"])
    st = oracle.State(hs.K, hs.V, topk=hs.topk, chunk=hs.chunk, eps=hs.eps, score="dot")
    gr = st.chunk_grads(Q, hs.Vt, hs.gate, 0.0, 0, hs.chunk)
    assert gr["loss"] == pytest.approx(sum(frac(x) for x in part["loss"]), rel=RTOL)
    dK = np.zeros_like(hs.K)
    for key, row in part["dLdK"].items():
        dK[row_key(key)] = arr(row)
    np.testing.assert_allclose(gr["dLdK"], dK, rtol=RTOL, atol=1e-15)
    res = st.step(Q, hs.Vt, hs.gate, hs.eta, 0.0, want_sel=True, want_gap=True)
    assert np.array_equal(res["sel_slot"], np.array(part["sel_slot"]))
    np.testing.assert_allclose(res["sel_w"], 0.5, rtol=RTOL)
    np.testing.assert_allclose(res["gap"], arr(part["gap"]), rtol=RTOL, atol=1e-15)
    np.testing.assert_allclose(res["out"], arr(part["out"]), rtol=RTOL)
    V = hs.V.copy()
    for r, row in part["values_after"].items():
        V[int(r)] = arr(row)
    np.testing.assert_allclose(st.V, V, rtol=RTOL, atol=0)
    K = hs.K.copy()
    for key, row in part["subkeys_after"].items():
        K[row_key(key)] = arr(row)
    np.testing.assert_allclose(st.K, K, rtol=RTOL, atol=1e-15)
