"""GPU (C ABI, sm_100a kernels) vs the fp64 oracle on the same seeded inputs.

Sizes here finish in seconds on the oracle yet span several chunks and score
tiles with a ragged last chunk; test_gpu_fullsize.py runs the full workload
sizes.  Tolerances and the near-tie policy are in fwpkm_testlib.
"""
import numpy as np
import pytest

from sparse_weight_memory_b200.workloads import WORKLOADS, Workload, make_inputs

from fwpkm_testlib import (OUT_ATOL, OUT_RTOL, TIE_GAP, check_close, check_selection,
                           check_table, compare_runs, gpu_run, oracle_run, to_dev, widen)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from sparse_weight_memory_b200 import build
    build.build()


REDUCED = {
    # every workload shape, T cut to a few chunks plus a ragged tail
    "tiny": WORKLOADS["tiny"],
    "library": WORKLOADS["library"].replace(T=3 * 256 + 77),
    "multihead": WORKLOADS["multihead"].replace(B=2, T=2 * 512 + 131),
    "longctx": WORKLOADS["longctx"].replace(T=3 * 1024 + 211, plant_frac=0.01),
    "iterative": WORKLOADS["iterative"].replace(B=2, T=2 * 512 + 45),
}


@pytest.mark.parametrize("name", sorted(REDUCED))
def test_workload_parity_forced_near_ties(oracle, name):
    wl = REDUCED[name]
    inp = make_inputs(wl)
    o = oracle_run(wl, inp, oracle)
    g = gpu_run(wl, inp, o, force=True, with_stats=True)
    info = compare_runs(wl, inp, g, o, name)
    # identical selections => identical count of distinct rows written
    assert g.touched == o.touched, (g.touched, o.touched)
    assert info["dV_rel"] < 1e-3 and info["dK_rel"] < 1e-3, info


@pytest.mark.parametrize("name", sorted(REDUCED))
def test_single_chunk_unforced(oracle, name):
    """One chunk from the initial tables, GPU deciding every selection itself.

    Slot sets must match wherever the oracle gap > 1e-5; a differing choice at
    a near tie must be valid (every chosen slot within 1e-5 of the k-th best
    oracle score).  Outputs and tables are compared away from such choices.
    """
    wl0 = REDUCED[name]
    wl = wl0.replace(T=wl0.chunk, calls=1, passes=1)
    inp = make_inputs(wl)
    o = oracle_run(wl, inp, oracle)
    g = gpu_run(wl, inp, None, force=False)
    diff = check_selection(g.sels[0], o.sels[0], o.gaps[0], name)
    Q = widen(inp.Q)
    excl_v, excl_k = set(), set()
    for b, t, h in np.argwhere(diff):
        q = Q[b, t, h * wl.dq:(h + 1) * wl.dq]
        s1, _ = oracle.half_scores(q[:wl.dh], inp.subkeys[h, 0], wl.eps)
        s2, _ = oracle.half_scores(q[wl.dh:], inp.subkeys[h, 1], wl.eps)
        kth = (s1[o.sels[0][b, t, h] // wl.n] + s2[o.sels[0][b, t, h] % wl.n]).min()
        for sl in g.sels[0][b, t, h]:
            assert s1[sl // wl.n] + s2[sl % wl.n] >= kth - TIE_GAP
        # rows this token wrote (either side) are affected by the choice
        for hh in range(wl.heads):
            for sl in list(g.sels[0][b, t, hh]) + list(o.sels[0][b, t, hh]):
                excl_v.add(int(sl))
                excl_k.add((hh * 2 + 0) * wl.n + int(sl) // wl.n)
                excl_k.add((hh * 2 + 1) * wl.n + int(sl) % wl.n)
    tok_ok = ~diff.any(axis=-1)
    check_close(g.outs[0][tok_ok], o.outs[0][tok_ok], OUT_ATOL, OUT_RTOL, f"{name} out")
    if not diff.any():  # same slot sets: compare the weights slot by slot
        og = np.argsort(g.sels[0], axis=-1)
        oo = np.argsort(o.sels[0], axis=-1)
        check_close(np.take_along_axis(g.ws[0], og, -1), np.take_along_axis(o.ws[0], oo, -1),
                    1e-6, 1e-5, f"{name} weights")
    check_table(g.V, o.V, 1e-4, f"{name} values", exclude_rows=excl_v)
    check_table(g.K, o.K, 1e-4, f"{name} sub-keys", exclude_rows=excl_k)


def test_determinism_bit_identical():
    wl = REDUCED["multihead"]
    inp = make_inputs(wl)
    a = gpu_run(wl, inp, None, force=False)
    b = gpu_run(wl, inp, None, force=False)
    assert np.array_equal(a.outs[0], b.outs[0])
    assert np.array_equal(a.V, b.V) and np.array_equal(a.K, b.K)
    assert np.array_equal(a.sels[0], b.sels[0])


@pytest.mark.parametrize("name", ["library", "multihead"])
def test_graph_replay_matches_direct_launches(name):
    """Calls repeated over fixed buffers are replayed as captured CUDA graphs
    (from the second sighting on); the results must be bit-identical to
    kernel-by-kernel launches of the same calls."""
    import torch

    from sparse_weight_memory_b200 import FwPKMState
    wl = REDUCED[name]
    inp = make_inputs(wl)
    Q, Vt, g = to_dev(inp.Q[:, :wl.T]), to_dev(inp.Vt[:, :wl.T]), to_dev(inp.gate[:, :wl.T])
    results = []
    for graphs in (False, True):
        st = FwPKMState(wl.N, wl.dq, wl.dv, wl.topk, wl.chunk, wl.heads, eps=wl.eps)
        st.set_graphs(graphs)
        st.set_tables(to_dev(inp.subkeys), to_dev(inp.values))
        out = torch.empty((wl.B, wl.T, wl.dv), dtype=torch.float32, device="cuda")
        outs = []
        for _ in range(4):  # direct, capture + replay, replay, replay
            st.step(Q, Vt, g, wl.eta, wl.lam, out=out)
            outs.append(out.cpu().numpy())
        K, V = st.get_tables()
        torch.cuda.synchronize()
        results.append((outs, K.cpu().numpy(), V.cpu().numpy()))
        st.close()
    (o0, K0, V0), (o1, K1, V1) = results
    for a, b in zip(o0, o1):
        assert np.array_equal(a, b)
    assert np.array_equal(K0, K1) and np.array_equal(V0, V1)


def test_eta_zero_leaves_tables_and_reads(oracle):
    wl = REDUCED["library"].replace(eta=0.0, calls=1)
    inp = make_inputs(wl)
    g = gpu_run(wl, inp, None, force=False)
    assert np.array_equal(g.V, inp.values) and np.array_equal(g.K, inp.subkeys)
    o = oracle_run(wl, inp, oracle)
    check_selection(g.sels[0], o.sels[0], o.gaps[0], "eta=0")
    diff = (np.sort(g.sels[0], -1) != np.sort(o.sels[0], -1)).any(-1).any(-1)
    check_close(g.outs[0][~diff], o.outs[0][~diff], OUT_ATOL, OUT_RTOL, "eta=0 out")


def test_chaining_equals_one_call():
    """Three chained calls over T == one call over 3T (chunk-aligned), bit-exact."""
    wl = WORKLOADS["library"].replace(T=512, calls=3)
    inp = make_inputs(wl)
    chained = gpu_run(wl, inp, None, force=False)
    one = gpu_run(wl.replace(T=3 * 512, calls=1), inp, None, force=False)
    assert np.array_equal(np.concatenate(chained.outs, axis=1), one.outs[0])
    assert np.array_equal(chained.V, one.V) and np.array_equal(chained.K, one.K)


def test_second_pass_equals_step_from_pass1_state():
    """Iterative reading: pass 2 == a fresh state loaded with the pass-1 tables."""
    wl = REDUCED["iterative"]
    inp = make_inputs(wl)
    two = gpu_run(wl, inp, None, force=False)
    one = gpu_run(wl.replace(passes=1), inp, None, force=False)
    again = gpu_run(wl.replace(passes=1), inp, None, force=False, K0=one.K, V0=one.V)
    assert np.array_equal(two.outs[1], again.outs[0])
    assert np.array_equal(two.V, again.V) and np.array_equal(two.K, again.K)


@pytest.mark.parametrize("case", ["library", "multihead", "ragged", "read_only"])
def test_host_buffer_step_equals_device_step(case):
    """Host buffers (copied in and out chunk by chunk, overlapping the step)
    give the device call's results bit for bit: several sequences, bf16
    inputs, a ragged last chunk."""
    import torch

    from sparse_weight_memory_b200 import FwPKMState
    if case == "ragged":
        base = REDUCED["library"]
        wl = base.replace(calls=1, B=3, T=3 * base.chunk + 7)
    elif case == "read_only":
        wl = REDUCED["iterative"].replace(calls=1, passes=1, eta=0.0)
    else:
        wl = REDUCED[case].replace(calls=1, passes=1)
    inp = make_inputs(wl)
    res = []
    for host in (False, True):
        st = FwPKMState(wl.N, wl.dq, wl.dv, wl.topk, wl.chunk, wl.heads)
        st.set_tables(to_dev(inp.subkeys), to_dev(inp.values))
        if host:
            out = st.step_host(inp.Q, inp.Vt, inp.gate, wl.eta, wl.lam)
        else:
            out = st.step(to_dev(inp.Q), to_dev(inp.Vt), to_dev(inp.gate), wl.eta,
                          wl.lam).cpu().numpy()
        torch.cuda.synchronize()
        K, V = st.get_tables()
        res.append((out, K.cpu().numpy(), V.cpu().numpy()))
        st.close()
    for a, b in zip(*res):
        assert np.array_equal(a, b)


EDGE = {
    "T_below_chunk": Workload("e1", B=3, T=5, chunk=32, heads=1, dq=32, n=16, dv=8, topk=4,
                              eta=0.7, lam=0.2, gate="uniform"),
    "k1": Workload("e2", B=2, T=40, chunk=16, heads=2, dq=16, n=8, dv=4, topk=1, eta=0.5,
                   lam=0.0, gate="uniform"),
    "k_equals_n": Workload("e3", B=1, T=33, chunk=8, heads=1, dq=32, n=4, dv=12, topk=4,
                           eta=0.4, lam=0.3, gate="beta25"),
    "k32_n32": Workload("e4", B=2, T=70, chunk=32, heads=1, dq=64, n=32, dv=64, topk=32,
                        eta=0.5, lam=0.1, gate="uniform"),
    "n_not_pow2": Workload("e5", B=2, T=100, chunk=48, heads=3, dq=48, n=48, dv=20, topk=7,
                           eta=0.6, lam=0.05, gate="uniform"),
    "wide_dv": Workload("e6", B=1, T=64, chunk=32, heads=1, dq=64, n=16, dv=2048, topk=8,
                        eta=0.3, lam=0.0, gate="one"),
    "many_heads_big_k": Workload("e7", B=1, T=40, chunk=20, heads=4, dq=32, n=64, dv=1024,
                                 topk=32, eta=0.2, lam=0.01, gate="uniform"),
    # 16 heads x k = 32 rows of 4 KB (8 KB) per token: 2 MB (4 MB) of rows, so
    # the read splits each token over a cluster of 2 (4) CTAs
    "heads16_cluster2_read": Workload("e8", B=1, T=24, chunk=12, heads=16, dq=32, n=32,
                                      dv=1024, topk=32, eta=0.2, lam=0.0, gate="uniform"),
    "heads16_cluster4_read_entropy": Workload("e9", B=1, T=20, chunk=10, heads=16, dq=32,
                                              n=32, dv=2048, topk=32, eta=0.2, lam=0.05,
                                              gate="uniform"),
    # dq/2 = 1024: 32 k-blocks in the score ring and 8 chunk norms per sub-key row
    "dq2048": Workload("e10", B=2, T=40, chunk=16, heads=1, dq=2048, n=16, dv=8, topk=4,
                       eta=0.05, lam=0.1, gate="uniform"),
    "heads16_small_dv": Workload("e11", B=2, T=30, chunk=16, heads=16, dq=32, n=8, dv=8,
                                 topk=4, eta=0.3, lam=0.02, gate="beta25"),
}


def read_cluster_size(wl) -> int:
    """The read kernel's sizing rule: one CTA per token, doubled into a
    cluster of G <= 8 CTAs while a CTA's share of the H*k rows exceeds 1 MB."""
    HK, row = wl.heads * wl.topk, wl.dv * 4
    G = 1
    while G < 8 and G < HK and -(-HK // G) * row > 1024 * 1024:
        G *= 2
    return G


def test_edge_table_reaches_the_cluster_read():
    assert read_cluster_size(EDGE["heads16_cluster2_read"]) == 2
    assert read_cluster_size(EDGE["heads16_cluster4_read_entropy"]) == 4
    assert read_cluster_size(EDGE["many_heads_big_k"]) == 1


@pytest.mark.parametrize("name", sorted(EDGE))
def test_edge_shapes(oracle, name):
    wl = EDGE[name]
    inp = make_inputs(wl)
    o = oracle_run(wl, inp, oracle)
    g = gpu_run(wl, inp, o, force=True)
    compare_runs(wl, inp, g, o, name)


@pytest.mark.parametrize("T,chunk", [(96, 96), (1100, 1100), (5000, 5000)])
def test_degenerate_identical_queries(oracle, T, chunk):
    """Every token reads the same slots: one group per slot with T members.
    Covers groups split into blocks with partials (> 32 members), buckets
    sorted by the whole CTA (> 32) and buckets merged through global memory
    (> 4096)."""
    wl = Workload("deg", B=1, T=T, chunk=chunk, heads=1, dq=32, n=8, dv=16, topk=4, eta=0.5,
                  lam=0.3, gate="uniform")
    inp = make_inputs(wl)
    inp.Q[:] = inp.Q[:, :1]
    o = oracle_run(wl, inp, oracle)
    g = gpu_run(wl, inp, o, force=True)
    compare_runs(wl, inp, g, o, "degenerate")


def test_invalid_arguments_launch_nothing():
    import torch

    from sparse_weight_memory_b200 import FwPKMState, FwpkmError
    from sparse_weight_memory_b200.fwpkm import FWPKM_EINVAL, FWPKM_ESHAPE
    wl = WORKLOADS["tiny"]
    inp = make_inputs(wl)
    st = FwPKMState(wl.N, wl.dq, wl.dv, wl.topk, wl.chunk)
    st.set_tables(to_dev(inp.subkeys), to_dev(inp.values))
    Q, Vt, g = to_dev(inp.Q), to_dev(inp.Vt), to_dev(inp.gate)
    with pytest.raises(FwpkmError) as e:
        st.step(Q, Vt, g, -1.0)
    assert e.value.status == FWPKM_EINVAL
    with pytest.raises(FwpkmError) as e:
        st.step(Q, Vt, g, float("nan"))
    assert e.value.status == FWPKM_EINVAL
    buf = torch.zeros(Q.numel() + 4, device="cuda")
    with pytest.raises(FwpkmError) as e:  # misaligned Q
        st.step(buf[1:1 + Q.numel()].view(Q.shape), Vt, g, 0.5)
    assert e.value.status == FWPKM_EINVAL
    torch.cuda.synchronize()
    K, V = st.get_tables()
    torch.cuda.synchronize()
    assert np.array_equal(V.cpu().numpy(), inp.values)
    with pytest.raises(FwpkmError) as e:
        FwPKMState(1000, 64, 64, 4, 32)
    assert e.value.status == FWPKM_ESHAPE
    st.close()


def test_eta_zero_runs_the_read_alone():
    """eta = 0 changes no table, so the step is the read alone: the write
    kernels do not launch, the first chunk's outputs equal those of a step
    with a tiny eta bit for bit (the read is the same), and the tables stay."""
    import torch

    from sparse_weight_memory_b200 import FwPKMState
    wl = REDUCED["multihead"].replace(calls=1)
    inp = make_inputs(wl)
    Q, Vt, g = to_dev(inp.Q), to_dev(inp.Vt), to_dev(inp.gate)
    outs = []
    for eta in (0.0, 1e-30):
        st = FwPKMState(wl.N, wl.dq, wl.dv, wl.topk, wl.chunk, wl.heads, eps=wl.eps)
        st.set_tables(to_dev(inp.subkeys), to_dev(inp.values))
        st.set_profiling(True)
        out = st.step(Q, Vt, g, eta, wl.lam)
        prof = st.profile_read()
        outs.append(out[:, :wl.chunk].cpu().numpy())
        if eta == 0.0:
            for kind in ("fwpkm_scan", "fwpkm_bsort", "fwpkm_apply", "fwpkm_pgrad"):
                assert prof[kind][1] == 0, (kind, prof[kind])
            assert prof["fwpkm_read"][1] == wl.n_chunks()
            K, V = st.get_tables()
            torch.cuda.synchronize()
            assert np.array_equal(K.cpu().numpy(), inp.subkeys)
            assert np.array_equal(V.cpu().numpy(), inp.values)
        st.close()
    assert np.array_equal(outs[0], outs[1])
