"""Pins of the fp64 oracle to facts other than itself.

Each test checks the oracle against something the pages or the mathematics fix:
brute force over all N slots, a library brute force, finite differences of the
loss written from its definition, closed forms (IDW weights, single-access and
two-writer updates, one-slot loss), invariants (eta = 0, untouched rows,
causality, chaining, sum of the marginal = 1) and a head-duplication
reduction.  A plausible mistake anywhere in the oracle (a dropped term, a
wrong sign or index, a transposed operand) fails at least one of them.
"""
import numpy as np
import pytest
from scipy.spatial.distance import cdist

EPS = 1e-3


def tiny_case(rng, B=2, T=8, H=2, dq=8, n=6, dv=5, k=3, gate="rand"):
    dh = dq // 2
    K = rng.standard_normal((H, 2, n, dh)) * dh ** -0.25
    V = rng.standard_normal((n * n, dv)) * 0.3
    Q = rng.standard_normal((B, T, H * dq))
    Vt = rng.standard_normal((B, T, dv))
    g = rng.uniform(0.2, 1.0, (B, T)) if gate == "rand" else np.ones((B, T))
    return K, V, Q, Vt, g


def make_state(oracle, K, V, k, chunk, **opts):
    return oracle.State(K, V, topk=k, chunk=chunk, eps=EPS, **opts)


# ---------------------------------------------------------------------------
# Selection
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("n,k", [(4, 1), (4, 4), (7, 3), (16, 8), (32, 32), (20, 11)])
def test_product_key_topk_equals_bruteforce(oracle, n, k):
    """Product-key top-k over k*k candidates == top-k over all N = n^2 slots."""
    rng = np.random.default_rng(100 + n * 37 + k)
    for trial in range(30):
        s1 = rng.standard_normal(n)
        s2 = rng.standard_normal(n)
        if trial % 3 == 1:       # forced ties inside each half
            s1 = np.round(s1 * 2) / 2
            s2 = np.round(s2 * 2) / 2
        elif trial % 3 == 2:     # all equal: pure index order decides
            s1[:] = 0.25
            s2[:] = -0.5
        pk, pks, ia, jb = oracle.pk_select(s1, s2, k)
        bf, bfs = oracle.brute_select(s1, s2, k)
        assert np.array_equal(pk, bf)
        assert np.array_equal(pks, bfs)
        assert np.array_equal(ia * n + jb, pk)


def test_ties_resolve_to_lower_index(oracle):
    """Equal scores are ordered by index (per half) and by slot (merged)."""
    idx, val = oracle.topk(np.array([1.0, 3.0, 3.0, 2.0, 3.0]), 4)
    assert list(idx) == [1, 2, 4, 3]
    slot, sc, ia, jb = oracle.pk_select(np.full(5, 0.5), np.full(5, 0.25), 3)
    assert list(slot) == [0, 1, 2]
    # through the whole step: identical sub-key rows make every slot score equal
    rng = np.random.default_rng(1)
    n, dh, k = 6, 3, 4
    K = np.broadcast_to(rng.standard_normal(dh), (1, 2, n, dh)).copy()
    V = rng.standard_normal((n * n, 2))
    Q = rng.standard_normal((1, 2, 2 * dh))
    st = make_state(oracle, K, V, k, 2)
    res = st.step(Q, rng.standard_normal((1, 2, 2)), np.ones((1, 2)), 0.0, 0.0,
                  want_sel=True)
    assert list(res["sel_slot"][0, 0, 0]) == [0, 1, 2, 3]
    assert np.allclose(res["sel_w"][0, 0, 0], 0.25, rtol=0, atol=1e-15)


def test_selection_matches_library_bruteforce(oracle):
    """Step selection == numpy/scipy brute force of -log(eps+d1)-log(eps+d2)."""
    rng = np.random.default_rng(7)
    K, V, Q, Vt, g = tiny_case(rng, B=1, T=6, H=2, dq=10, n=9, dv=4, k=5)
    st = make_state(oracle, K, V, 5, 6)
    res = st.step(Q, Vt, g, eta=0.0, lam=0.0, want_sel=True)
    dh = 5
    for t in range(6):
        for h in range(2):
            q = Q[0, t, h * 10:(h + 1) * 10]
            d1 = cdist(q[None, :dh], K[h, 0], "sqeuclidean")[0]
            d2 = cdist(q[None, dh:], K[h, 1], "sqeuclidean")[0]
            s = (-np.log(EPS + d1))[:, None] + (-np.log(EPS + d2))[None, :]
            flat = s.reshape(-1)
            order = np.lexsort((np.arange(flat.size), -flat))
            assert np.array_equal(res["sel_slot"][0, t, h], order[:5])


def test_idw_exact_hit_and_closed_form_weights(oracle):
    """q_h == K_h,i gives score -log(eps); weights are prop. to 1/((eps+d1)(eps+d2))."""
    rng = np.random.default_rng(3)
    n, dh = 8, 4
    K1 = rng.standard_normal((n, dh))
    q = K1[5].copy()
    s, d = oracle.half_scores(q, K1, EPS)
    assert s[5] == -np.log(EPS) and d[5] == 0.0
    # known distance: K row = q + delta * e_0  -> d = delta^2
    K1[2] = q.copy()
    K1[2, 0] += 0.75
    s, d = oracle.half_scores(q, K1, EPS)
    assert d[2] == 0.5625 and np.isclose(s[2], -np.log(EPS + 0.5625), rtol=0, atol=1e-15)

    K, V, Q, Vt, g = tiny_case(rng, B=1, T=4, H=1, dq=8, n=7, dv=3, k=4)
    st = make_state(oracle, K, V, 4, 4)
    res = st.step(Q, Vt, g, eta=0.0, lam=0.0, want_sel=True)
    for t in range(4):
        q = Q[0, t]
        d1 = cdist(q[None, :4], K[0, 0], "sqeuclidean")[0]
        d2 = cdist(q[None, 4:], K[0, 1], "sqeuclidean")[0]
        sl = res["sel_slot"][0, t, 0]
        inv = 1.0 / ((EPS + d1[sl // 7]) * (EPS + d2[sl % 7]))
        assert np.allclose(res["sel_w"][0, t, 0], inv / inv.sum(), rtol=1e-12, atol=0)


def test_gap_is_kth_minus_next(oracle):
    rng = np.random.default_rng(11)
    K, V, Q, Vt, g = tiny_case(rng, B=1, T=5, H=1, dq=6, n=5, dv=2, k=3)
    st = make_state(oracle, K, V, 3, 5)
    res = st.step(Q, Vt, g, 0.0, 0.0, want_gap=True)
    for t in range(5):
        q = Q[0, t]
        d1 = cdist(q[None, :3], K[0, 0], "sqeuclidean")[0]
        d2 = cdist(q[None, 3:], K[0, 1], "sqeuclidean")[0]
        s = np.sort(((-np.log(EPS + d1))[:, None] - np.log(EPS + d2)[None, :]).ravel())[::-1]
        assert np.isclose(res["gap"][0, t, 0], s[2] - s[3], rtol=0, atol=1e-13)


# ---------------------------------------------------------------------------
# Gradients: central finite differences of the loss definition
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("lam,H,gate,own_weight,heads", [
    (0.0, 1, "one", False, "mean"), (0.0, 2, "rand", False, "mean"),
    (0.3, 2, "rand", False, "mean"), (1.5, 1, "rand", False, "mean"),
    (0.3, 2, "rand", True, "mean"), (0.0, 3, "rand", False, "sum"),
    (0.4, 2, "rand", True, "sum"), (0.0, 2, "rand", False, "dot"),
    (0.5, 1, "rand", True, "dot")])
def test_gradients_match_finite_differences(oracle, lam, H, gate, own_weight, heads):
    rng = np.random.default_rng(int(lam * 10) + H + (7 if own_weight else 0))
    B, T, dq, n, dv, k = 2, 6, 8, 6, 5, 3
    K, V, Q, Vt, g = tiny_case(rng, B=B, T=T, H=H, dq=dq, n=n, dv=dv, k=k, gate=gate)
    # a per-token MSE weight of its own (some tokens 0), else the gate
    om = rng.uniform(0.0, 1.5, (B, T)) * (rng.random((B, T)) > 0.3) if own_weight else None
    # "dot": heads averaged, the dot-product sub-key score
    opts = {"score": "dot"} if heads == "dot" else {"heads": heads}
    st = make_state(oracle, K, V, k, T, **opts)
    gr = st.chunk_grads(Q, Vt, g, lam, 0, T, omega=om)
    slots = gr["sel_slot"]
    L0 = st.chunk_loss(Q, Vt, g, lam, 0, T, slots, omega=om)
    assert np.isclose(L0, gr["loss"], rtol=1e-13, atol=0)
    h = 1e-6
    # values
    fdV = np.zeros_like(st.V)
    for idx in np.ndindex(*st.V.shape):
        s2 = st.copy()
        s2.V[idx] += h
        lp = s2.chunk_loss(Q, Vt, g, lam, 0, T, slots, omega=om)
        s2.V[idx] -= 2 * h
        lm = s2.chunk_loss(Q, Vt, g, lam, 0, T, slots, omega=om)
        fdV[idx] = (lp - lm) / (2 * h)
    assert np.allclose(gr["dLdV"], fdV, rtol=1e-6, atol=1e-8)
    # sub-keys
    fdK = np.zeros_like(st.K)
    for idx in np.ndindex(*st.K.shape):
        s2 = st.copy()
        s2.K[idx] += h
        lp = s2.chunk_loss(Q, Vt, g, lam, 0, T, slots, omega=om)
        s2.K[idx] -= 2 * h
        lm = s2.chunk_loss(Q, Vt, g, lam, 0, T, slots, omega=om)
        fdK[idx] = (lp - lm) / (2 * h)
    assert np.allclose(gr["dLdK"], fdK, rtol=1e-6, atol=1e-8)
    # both gradients are non-trivial, so the comparison above has teeth
    assert np.abs(fdK).max() > 0 and np.abs(fdV).max() > 0


def test_one_slot_loss_closed_form(oracle):
    """k=1, one token: L = g ||V_slot - v||^2; two tokens on distinct slots add
    lam * log(1/2) (marginal p_bar = (1/2, 1/2))."""
    rng = np.random.default_rng(5)
    K, V, Q, Vt, g = tiny_case(rng, B=1, T=2, H=1, dq=4, n=3, dv=3, k=1)
    st = make_state(oracle, K, V, 1, 2)
    gr = st.chunk_grads(Q, Vt, g, 0.0, 0, 1)
    sl = gr["sel_slot"][0, 0, 0, 0]
    assert np.isclose(gr["loss"], g[0, 0] * np.sum((V[sl] - Vt[0, 0]) ** 2), rtol=1e-14)
    gr2 = st.chunk_grads(Q, Vt, g, 0.7, 0, 2)
    s0, s1 = gr2["sel_slot"][0, :, 0, 0]
    if s0 != s1:
        mse = sum(g[0, t] * np.sum((V[gr2['sel_slot'][0, t, 0, 0]] - Vt[0, t]) ** 2)
                  for t in range(2))
        assert np.isclose(gr2["loss"], mse + 0.7 * np.log(0.5), rtol=1e-13)
        assert np.isclose(gr2["pbar"][s0], 0.5) and np.isclose(gr2["pbar"][s1], 0.5)


def test_marginal_sums_to_one(oracle):
    rng = np.random.default_rng(21)
    K, V, Q, Vt, g = tiny_case(rng, B=3, T=5, H=2, dq=6, n=5, dv=2, k=4)
    st = make_state(oracle, K, V, 4, 5)
    gr = st.chunk_grads(Q, Vt, g, 0.2, 0, 5)
    assert np.isclose(gr["pbar"].sum(), 1.0, rtol=0, atol=1e-14)
    assert (gr["pbar"] >= 0).all()


# ---------------------------------------------------------------------------
# Update rule: closed forms and invariants
# ---------------------------------------------------------------------------
def test_single_access_update_closed_form(oracle):
    """A row written by exactly one token-head moves by -2 eta g (yhat - v),
    whatever its weight and the head count."""
    rng = np.random.default_rng(9)
    for H in (1, 2, 3):
        K, V, Q, Vt, g = tiny_case(rng, B=1, T=1, H=H, dq=8, n=12, dv=4, k=3)
        st = make_state(oracle, K, V, 3, 1)
        st0 = st.copy()
        eta = 0.37
        res = st.step(Q, Vt, g, eta, 0.0, want_sel=True)
        yhat = res["out"][0, 0] / g[0, 0]
        sl = res["sel_slot"][0, 0].ravel()
        uniq, cnt = np.unique(sl, return_counts=True)
        for s_, c_ in zip(uniq, cnt):
            if c_ == 1:
                expect = st0.V[s_] - 2 * eta * g[0, 0] * (yhat - Vt[0, 0])
                assert np.allclose(st.V[s_], expect, rtol=1e-12, atol=1e-14)


def test_k1_half_step_memorises_target(oracle):
    """k=1, g=1, eta=1/2: the single selected row becomes the target exactly."""
    rng = np.random.default_rng(2)
    K, V, Q, Vt, g = tiny_case(rng, B=1, T=1, H=1, dq=6, n=4, dv=3, k=1, gate="one")
    st = make_state(oracle, K, V, 1, 1)
    res = st.step(Q, Vt, g, 0.5, 0.0, want_sel=True)
    sl = res["sel_slot"][0, 0, 0, 0]
    assert np.allclose(st.V[sl], Vt[0, 0], rtol=0, atol=1e-15)


def test_two_writers_average_targets(oracle):
    """Two identical queries with different targets: every selected row moves
    by -2 eta (yhat - mean(v_a, v_b)) -- the averaged (consensus) write."""
    rng = np.random.default_rng(4)
    K, V, Q, Vt, g = tiny_case(rng, B=1, T=2, H=1, dq=8, n=6, dv=3, k=3, gate="one")
    Q[0, 1] = Q[0, 0]
    st = make_state(oracle, K, V, 3, 2)
    st0 = st.copy()
    eta = 0.25
    res = st.step(Q, Vt, g, eta, 0.0, want_sel=True)
    yhat = res["out"][0, 0]
    for s_ in res["sel_slot"][0, 0, 0]:
        expect = st0.V[s_] - 2 * eta * (yhat - 0.5 * (Vt[0, 0] + Vt[0, 1]))
        assert np.allclose(st.V[s_], expect, rtol=1e-12, atol=1e-14)


def test_eta_zero_leaves_state_and_reads(oracle):
    rng = np.random.default_rng(12)
    K, V, Q, Vt, g = tiny_case(rng, B=2, T=12, H=2, dq=8, n=6, dv=4, k=3)
    st = make_state(oracle, K, V, 3, 4)
    res = st.step(Q, Vt, g, 0.0, 0.9)
    assert np.array_equal(st.K, K) and np.array_equal(st.V, V)
    # every chunk reads the initial tables: same as reading the whole call at once
    st_once = make_state(oracle, K, V, 3, 12)
    res_once = st_once.step(Q, Vt, g, 0.0, 0.0)
    assert np.array_equal(res["out"], res_once["out"])


@pytest.mark.parametrize("lam", [0.0, 0.4])
def test_only_selected_rows_change(oracle, lam):
    rng = np.random.default_rng(13)
    K, V, Q, Vt, g = tiny_case(rng, B=2, T=4, H=2, dq=8, n=7, dv=4, k=3)
    st = make_state(oracle, K, V, 3, 4)
    res = st.step(Q, Vt, g, 0.8, lam, want_sel=True)
    sel = np.unique(res["sel_slot"])
    changed_v = np.where((st.V != V).any(axis=1))[0]
    assert set(changed_v) <= set(sel) and len(changed_v) > 0
    n = 7
    for h in range(2):
        used_i = np.unique(res["sel_slot"][:, :, h] // n)
        used_j = np.unique(res["sel_slot"][:, :, h] % n)
        ch1 = np.where((st.K[h, 0] != K[h, 0]).any(axis=1))[0]
        ch2 = np.where((st.K[h, 1] != K[h, 1]).any(axis=1))[0]
        assert set(ch1) <= set(used_i) and set(ch2) <= set(used_j)
        assert len(ch1) > 0 and len(ch2) > 0


def test_causality(oracle):
    """Perturbing tokens of chunk 2 leaves the outputs of chunks 0 and 1 unchanged."""
    rng = np.random.default_rng(14)
    K, V, Q, Vt, g = tiny_case(rng, B=2, T=16, H=1, dq=8, n=6, dv=4, k=2)
    st_a = make_state(oracle, K, V, 2, 4)
    ra = st_a.step(Q, Vt, g, 0.6, 0.2)
    Q2, Vt2 = Q.copy(), Vt.copy()
    Q2[:, 8:12] += rng.standard_normal(Q2[:, 8:12].shape)
    Vt2[:, 8:12] += 1.0
    st_b = make_state(oracle, K, V, 2, 4)
    rb = st_b.step(Q2, Vt2, g, 0.6, 0.2)
    assert np.array_equal(ra["out"][:, :8], rb["out"][:, :8])
    assert not np.array_equal(ra["out"][:, 8:], rb["out"][:, 8:])


def test_chaining_equals_one_long_call(oracle):
    rng = np.random.default_rng(15)
    K, V, Q, Vt, g = tiny_case(rng, B=2, T=24, H=2, dq=8, n=6, dv=4, k=3)
    one = make_state(oracle, K, V, 3, 4)
    r1 = one.step(Q, Vt, g, 0.5, 0.1)
    ch = make_state(oracle, K, V, 3, 4)
    outs = [ch.step(Q[:, s:s + 8], Vt[:, s:s + 8], g[:, s:s + 8], 0.5, 0.1)["out"]
            for s in (0, 8, 16)]
    assert np.array_equal(np.concatenate(outs, axis=1), r1["out"])
    assert np.array_equal(one.K, ch.K) and np.array_equal(one.V, ch.V)


def test_second_pass_equals_a_fresh_state_from_the_first(oracle):
    """Iterative reading: pass 2 over the same sequence equals a step started
    from a new state holding pass 1's tables (the tables are the whole state)."""
    rng = np.random.default_rng(18)
    K, V, Q, Vt, g = tiny_case(rng, B=2, T=12, H=2, dq=8, n=6, dv=4, k=3)
    a = make_state(oracle, K, V, 3, 4)
    a.step(Q, Vt, g, 0.5, 0.2)
    b = make_state(oracle, a.K, a.V, 3, 4)
    r2 = a.step(Q, Vt, g, 0.5, 0.2)
    rb = b.step(Q, Vt, g, 0.5, 0.2)
    assert np.array_equal(r2["out"], rb["out"])
    assert np.array_equal(a.K, b.K) and np.array_equal(a.V, b.V)
    # and the second pass reads differently from the first
    r1 = make_state(oracle, K, V, 3, 4).step(Q, Vt, g, 0.5, 0.2)
    assert not np.array_equal(r1["out"], r2["out"])


def test_zero_weight_tokens_are_read_but_write_nothing(oracle):
    """Tokens whose MSE weight is 0 still read (out = g * yhat) but leave both
    tables unchanged; with every weight 0 the step is a pure read."""
    rng = np.random.default_rng(19)
    K, V, Q, Vt, g = tiny_case(rng, B=2, T=8, H=2, dq=8, n=6, dv=4, k=3)
    a = make_state(oracle, K, V, 3, 4)
    ra = a.step(Q, Vt, g, 0.6, 0.0, omega=np.zeros_like(g))
    assert np.array_equal(a.K, K) and np.array_equal(a.V, V)
    rb = make_state(oracle, K, V, 3, 4).step(Q, Vt, g, 0.0, 0.0)
    assert np.array_equal(ra["out"], rb["out"])


def test_lookahead_pairs_each_query_with_the_next_target(oracle):
    """k = 1, one head: each token reads one slot with weight 1, so a slot read
    once by token t moves by -2 eta g_t (V[slot] - v_{t+1}), and the last token
    (no target in the call) leaves its slot unchanged.  The keys do not move
    (with k = 1 the softmax Jacobian is 0), and the outputs are the plain read."""
    rng = np.random.default_rng(23)
    for _ in range(20):
        K, V, Q, Vt, g = tiny_case(rng, B=1, T=3, H=1, dq=4, n=5, dv=3, k=1)
        st = make_state(oracle, K, V, 1, 3)
        r = st.step(Q, Vt, g, 0.4, 0.0, want_sel=True, lookahead=True)
        sl = r["sel_slot"][0, :, 0, 0]
        if len(set(sl.tolist())) < 3:
            continue  # a shared slot: the closed form below needs distinct rows
        for t in range(3):
            assert np.allclose(r["out"][0, t], g[0, t] * V[sl[t]], rtol=1e-14, atol=0)
        for t in range(2):
            want = V[sl[t]] - 2 * 0.4 * g[0, t] * (V[sl[t]] - Vt[0, t + 1])
            assert np.allclose(st.V[sl[t]], want, rtol=1e-13, atol=1e-15)
        assert np.array_equal(st.V[sl[2]], V[sl[2]])
        assert np.array_equal(st.K, K)
        return
    pytest.fail("no draw with three distinct slots")


def test_ragged_last_chunk(oracle):
    """T = 10 with chunk 4: chunks of 4, 4, 2; the split is the same as three calls."""
    rng = np.random.default_rng(16)
    K, V, Q, Vt, g = tiny_case(rng, B=1, T=10, H=1, dq=8, n=6, dv=4, k=2)
    a = make_state(oracle, K, V, 2, 4)
    ra = a.step(Q, Vt, g, 0.5, 0.3)
    b = make_state(oracle, K, V, 2, 4)
    outs = [b.step(Q[:, s:e], Vt[:, s:e], g[:, s:e], 0.5, 0.3)["out"]
            for s, e in ((0, 4), (4, 8), (8, 10))]
    assert np.array_equal(np.concatenate(outs, axis=1), ra["out"])
    assert np.array_equal(a.V, b.V) and np.array_equal(a.K, b.K)


@pytest.mark.parametrize("lam", [0.0, 0.5])
def test_duplicated_heads_reduce_to_one_head(oracle, lam):
    """H=2 with identical queries and sub-keys per head == H=1: same reads and
    value update; each head's sub-keys take half the single-head key step."""
    rng = np.random.default_rng(17)
    K1, V, Q1, Vt, g = tiny_case(rng, B=2, T=4, H=1, dq=8, n=6, dv=4, k=3)
    K2 = np.concatenate([K1, K1], axis=0)
    Q2 = np.concatenate([Q1, Q1], axis=2)
    a = make_state(oracle, K1, V, 3, 4)
    ra = a.step(Q1, Vt, g, 0.7, lam)
    b = make_state(oracle, K2, V, 3, 4)
    rb = b.step(Q2, Vt, g, 0.7, lam)
    assert np.allclose(ra["out"], rb["out"], rtol=1e-13, atol=1e-15)
    assert np.allclose(a.V, b.V, rtol=1e-12, atol=1e-15)
    for h in range(2):
        assert np.allclose(b.K[h] - K1[0], 0.5 * (a.K[0] - K1[0]), rtol=1e-9, atol=1e-15)


# ---------------------------------------------------------------------------
# Options of two readings: the divisor of a value row's gradient, and summed
# heads (each against a closed form or a reduction, like the defaults above)
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("agg", ["count", "sum"])
def test_single_access_update_without_row_contribution(oracle, agg):
    """A row written once: divided by its access count (1) or not divided, it
    moves by the raw gradient -eta (2 g / H) w (yhat - v) -- the weight w no
    longer cancels as it does under the default divisor."""
    rng = np.random.default_rng(31)
    for H in (1, 2):
        K, V, Q, Vt, g = tiny_case(rng, B=1, T=1, H=H, dq=8, n=12, dv=4, k=3)
        st = make_state(oracle, K, V, 3, 1, agg=agg)
        st0 = st.copy()
        eta = 0.37
        res = st.step(Q, Vt, g, eta, 0.0, want_sel=True)
        yhat = res["out"][0, 0] / g[0, 0]
        sl = res["sel_slot"][0, 0].ravel()
        w = res["sel_w"][0, 0].ravel()
        uniq, cnt = np.unique(sl, return_counts=True)
        checked = 0
        for s_, c_ in zip(uniq, cnt):
            if c_ == 1:
                wi = w[sl == s_][0]
                expect = st0.V[s_] - eta * (2 * g[0, 0] / H) * wi * (yhat - Vt[0, 0])
                assert np.allclose(st.V[s_], expect, rtol=1e-12, atol=1e-14)
                checked += 1
        assert checked > 0


@pytest.mark.parametrize("agg,factor", [("count", 1.0), ("sum", 2.0)])
def test_two_writers_without_row_contribution(oracle, agg, factor):
    """Two identical queries (same slots, same weights w) with targets v_a,
    v_b: G = 2 w (2 yhat - v_a - v_b); divided by the count 2 the row moves by
    -2 eta w (yhat - mean v), undivided by twice that."""
    rng = np.random.default_rng(4)
    K, V, Q, Vt, g = tiny_case(rng, B=1, T=2, H=1, dq=8, n=6, dv=3, k=3, gate="one")
    Q[0, 1] = Q[0, 0]
    st = make_state(oracle, K, V, 3, 2, agg=agg)
    st0 = st.copy()
    eta = 0.25
    res = st.step(Q, Vt, g, eta, 0.0, want_sel=True)
    yhat = res["out"][0, 0]
    for s_, w_ in zip(res["sel_slot"][0, 0, 0], res["sel_w"][0, 0, 0]):
        expect = st0.V[s_] - factor * 2 * eta * w_ * (yhat - 0.5 * (Vt[0, 0] + Vt[0, 1]))
        assert np.allclose(st.V[s_], expect, rtol=1e-12, atol=1e-14)


def test_summed_duplicated_heads_read_twice_one_head(oracle):
    """H = 2 with identical queries and sub-keys per head, readouts summed:
    every read is twice the single head's (eta = 0, so every chunk reads the
    same tables)."""
    rng = np.random.default_rng(19)
    K1, V, Q1, Vt, g = tiny_case(rng, B=2, T=6, H=1, dq=8, n=6, dv=4, k=3)
    a = make_state(oracle, K1, V, 3, 3)
    ra = a.step(Q1, Vt, g, 0.0, 0.0)
    b = make_state(oracle, np.concatenate([K1, K1], axis=0), V, 3, 3, heads="sum")
    rb = b.step(np.concatenate([Q1, Q1], axis=2), Vt, g, 0.0, 0.0)
    assert np.allclose(rb["out"], 2.0 * ra["out"], rtol=1e-13, atol=1e-15)


def test_dot_product_selection_is_the_brute_force_top_k(oracle):
    """With the dot-product score, the product-key selection equals the top-k
    over all N slots of q1.K1[i] + q2.K2[j], computed here with numpy (ties
    by slot), and the weights are their softmax."""
    rng = np.random.default_rng(23)
    for n, k in ((6, 3), (9, 5), (12, 12)):
        K, V, Q, Vt, g = tiny_case(rng, B=1, T=5, H=1, dq=8, n=n, dv=3, k=k)
        st = make_state(oracle, K, V, k, 5, score="dot")
        res = st.step(Q, Vt, g, 0.0, 0.0, want_sel=True)
        for t in range(5):
            s1 = K[0, 0] @ Q[0, t, :4]
            s2 = K[0, 1] @ Q[0, t, 4:]
            full = (s1[:, None] + s2[None, :]).ravel()
            order = np.lexsort((np.arange(n * n), -full))[:k]
            assert np.array_equal(np.sort(res["sel_slot"][0, t, 0]), np.sort(order))
            w = np.exp(full[order] - full[order].max())
            got = dict(zip(res["sel_slot"][0, t, 0], res["sel_w"][0, t, 0]))
            for sl, wi in zip(order, w / w.sum()):
                assert np.isclose(got[sl], wi, rtol=1e-12)
        assert np.allclose(oracle.half_scores_dot(Q[0, 0, :4], K[0, 0]), K[0, 0] @ Q[0, 0, :4])
