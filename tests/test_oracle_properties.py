"""Randomised properties of the oracle over small shapes and every option.

Each example draws a shape (heads, sub-keys per half, half width, value
width, top-k, chunk), the step's scalars and the readings' options (score,
head mode, divisor), then checks what holds for any input:
  * the selection is the top-k over all N slots of s1(i) + s2(j), with the
    half scores computed here with numpy from their definitions, and the
    weights are their softmax;
  * eta = 0 leaves both tables bit-unchanged;
  * only the selected value rows and the sub-key rows of the selected pairs
    change;
  * a chunk's outputs do not depend on later tokens;
  * the marginal p_bar over the chunk's token-heads sums to one.
"""
import numpy as np
import pytest

hypothesis = pytest.importorskip("hypothesis")
from hypothesis import given, settings, strategies as hs  # noqa: E402

from oracle import oracle  # noqa: E402

SETTINGS = settings(max_examples=25, deadline=None, derandomize=True)


@hs.composite
def cases(draw):
    H = draw(hs.integers(1, 3))
    n = draw(hs.integers(3, 9))
    dh = draw(hs.sampled_from([2, 3, 4]))
    dv = draw(hs.integers(1, 4))
    k = draw(hs.integers(1, min(6, n)))
    chunk = draw(hs.integers(1, 5))
    T = draw(hs.integers(chunk, 3 * chunk))
    B = draw(hs.integers(1, 2))
    opts = {"score": draw(hs.sampled_from(["idw", "dot"])),
            "heads": draw(hs.sampled_from(["mean", "sum"])),
            "agg": draw(hs.sampled_from(["weight", "count", "sum"]))}
    eta = draw(hs.sampled_from([0.1, 0.5, 1.0]))
    lam = draw(hs.sampled_from([0.0, 0.2]))
    seed = draw(hs.integers(0, 2**31 - 1))
    return dict(H=H, n=n, dh=dh, dv=dv, k=k, chunk=chunk, T=T, B=B, opts=opts, eta=eta,
                lam=lam, seed=seed)


def make(c):
    rng = np.random.default_rng(c["seed"])
    K = rng.standard_normal((c["H"], 2, c["n"], c["dh"]))
    V = rng.standard_normal((c["n"] * c["n"], c["dv"]))
    Q = rng.standard_normal((c["B"], c["T"], c["H"] * 2 * c["dh"]))
    Vt = rng.standard_normal((c["B"], c["T"], c["dv"]))
    g = rng.uniform(0.1, 1.0, (c["B"], c["T"]))
    return K, V, Q, Vt, g


def state(c, K, V):
    return oracle.State(K, V, topk=c["k"], chunk=c["chunk"], eps=1e-3, **c["opts"])


def half_scores(q, Kh, score):
    if score == "dot":
        return Kh @ q
    return -np.log(1e-3 + ((Kh - q) ** 2).sum(axis=1))


@SETTINGS
@given(cases())
def test_selection_is_the_top_k_over_all_slots(c):
    K, V, Q, Vt, g = make(c)
    res = state(c, K, V).step(Q, Vt, g, 0.0, 0.0, want_sel=True)  # eta = 0: one table
    n, dh, k = c["n"], c["dh"], c["k"]
    for b in range(c["B"]):
        for t in range(c["T"]):
            for h in range(c["H"]):
                q = Q[b, t, h * 2 * dh:(h + 1) * 2 * dh]
                s1 = half_scores(q[:dh], K[h, 0], c["opts"]["score"])
                s2 = half_scores(q[dh:], K[h, 1], c["opts"]["score"])
                full = (s1[:, None] + s2[None, :]).ravel()
                order = np.lexsort((np.arange(n * n), -full))[:k]
                got = res["sel_slot"][b, t, h]
                assert np.array_equal(np.sort(got), np.sort(order))
                w = np.exp(full[order] - full[order].max())
                w /= w.sum()
                gw = dict(zip(got, res["sel_w"][b, t, h]))
                assert np.allclose([gw[s] for s in order], w, rtol=1e-12, atol=0)


@SETTINGS
@given(cases())
def test_eta_zero_changes_nothing(c):
    K, V, Q, Vt, g = make(c)
    st = state(c, K, V)
    st.step(Q, Vt, g, 0.0, c["lam"])
    assert np.array_equal(st.K, K) and np.array_equal(st.V, V)


@SETTINGS
@given(cases())
def test_only_selected_rows_change(c):
    K, V, Q, Vt, g = make(c)
    c = dict(c, T=c["chunk"])  # one chunk: the selection is read with the initial tables
    Q, Vt, g = Q[:, :c["T"]], Vt[:, :c["T"]], g[:, :c["T"]]
    st = state(c, K, V)
    res = st.step(Q, Vt, g, c["eta"], c["lam"], want_sel=True)
    sel = res["sel_slot"]
    vrows = set(np.unique(sel).tolist())
    changed_v = set(np.nonzero((st.V != V).any(axis=1))[0].tolist())
    assert changed_v <= vrows
    n = c["n"]
    krows = set()
    for h in range(c["H"]):
        slots = sel[:, :, h, :].ravel()
        krows |= {(h, 0, int(s) // n) for s in slots} | {(h, 1, int(s) % n) for s in slots}
    changed_k = {tuple(int(x) for x in idx) for idx in np.argwhere((st.K != K).any(axis=-1))}
    assert changed_k <= krows


@SETTINGS
@given(cases())
def test_outputs_do_not_depend_on_later_tokens(c):
    K, V, Q, Vt, g = make(c)
    cut = c["chunk"]  # everything from the second chunk on is changed
    if c["T"] <= cut:
        return
    out_a = state(c, K, V).step(Q, Vt, g, c["eta"], c["lam"])["out"]
    Q2, Vt2, g2 = Q.copy(), Vt.copy(), g.copy()
    Q2[:, cut:] += 1.0
    Vt2[:, cut:] -= 2.0
    g2[:, cut:] = 0.5
    out_b = state(c, K, V).step(Q2, Vt2, g2, c["eta"], c["lam"])["out"]
    assert np.array_equal(out_a[:, :cut], out_b[:, :cut])


@SETTINGS
@given(cases())
def test_marginal_sums_to_one(c):
    K, V, Q, Vt, g = make(c)
    gr = state(c, K, V).chunk_grads(Q, Vt, g, c["lam"], 0, min(c["chunk"], c["T"]))
    assert gr["pbar"].sum() == pytest.approx(1.0, rel=1e-12)
