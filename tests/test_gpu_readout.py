"""Iterative readout with the lookahead pairing and token weights of their own,
on the GPU (fwpkm_step_ex) against the fp64 oracle.

gist.science "Fast-weight Product Key Memory", section 2 (lookahead targets:
query q_t is written towards v_{t+1}) and section 4 (iterative reading: the
same sequence read 2-4 times with the memory carried over); sciencestack
table of contents (the MSE loss weighted by token importance).  Tolerances
and the near-tie policy are those of fwpkm_testlib.
"""
import numpy as np
import pytest

from sparse_weight_memory_b200.workloads import WORKLOADS, make_inputs

from fwpkm_testlib import compare_runs, gpu_run, oracle_run, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from sparse_weight_memory_b200 import build
    build.build()


ITER = WORKLOADS["iterative"].replace(B=2, T=2 * 512 + 45)


@pytest.mark.parametrize("name,wl", [
    ("iterative_lookahead_2pass", ITER.replace(lookahead=True)),
    ("library_lookahead_chained", WORKLOADS["library"].replace(T=2 * 256 + 31,
                                                               lookahead=True)),
    ("longctx_lookahead", WORKLOADS["longctx"].replace(T=2 * 1024 + 100, lookahead=True)),
])
def test_lookahead_parity(oracle, name, wl):
    inp = make_inputs(wl)
    o = oracle_run(wl, inp, oracle)
    g = gpu_run(wl, inp, o, force=True, with_stats=True)
    info = compare_runs(wl, inp, g, o, name)
    assert g.touched == o.touched
    assert info["dV_rel"] < 1e-3 and info["dK_rel"] < 1e-3, info


def test_token_weights_apart_from_the_gate(oracle):
    """omega != gate, a quarter of the tokens at weight 0 (read, write nothing
    of their own); bf16 inputs and the entropy term on."""
    wl = WORKLOADS["multihead"].replace(B=2, T=512 + 77)
    inp = make_inputs(wl)
    rng = np.random.default_rng(11)
    omega = rng.random(inp.gate.shape).astype(np.float32) * 2.0
    omega[rng.random(omega.shape) < 0.25] = 0.0
    o = oracle_run(wl, inp, oracle, omega=omega)
    g = gpu_run(wl, inp, o, force=True, with_stats=True, omega=omega)
    info = compare_runs(wl, inp, g, o, "omega")
    assert info["dV_rel"] < 1e-3 and info["dK_rel"] < 1e-3, info


def test_four_passes_with_lookahead(oracle):
    """The same sequence read four times, the memory carried across passes
    (2-4 reads on the pages), each pass with the lookahead pairing."""
    wl = ITER.replace(passes=4, lookahead=True)
    inp = make_inputs(wl)
    o = oracle_run(wl, inp, oracle)
    g = gpu_run(wl, inp, o, force=True)
    info = compare_runs(wl, inp, g, o, "4 passes")
    assert info["dV_rel"] < 1e-3 and info["dK_rel"] < 1e-3, info


def test_weight_zero_everywhere_writes_nothing():
    """omega = 0 for every token: reads as usual, tables bit-unchanged."""
    import torch

    from sparse_weight_memory_b200 import FwPKMState
    wl = WORKLOADS["library"].replace(T=300, calls=1)
    inp = make_inputs(wl)
    st = FwPKMState(wl.N, wl.dq, wl.dv, wl.topk, wl.chunk, wl.heads, eps=wl.eps)
    st.set_tables(to_dev(inp.subkeys), to_dev(inp.values))
    zero = torch.zeros(inp.gate.shape, dtype=torch.float32, device="cuda")
    st.step(to_dev(inp.Q), to_dev(inp.Vt), to_dev(inp.gate), wl.eta, 0.0, omega=zero)
    torch.cuda.synchronize()
    K, V = st.get_tables()
    torch.cuda.synchronize()
    assert np.array_equal(K.cpu().numpy(), inp.subkeys)
    assert np.array_equal(V.cpu().numpy(), inp.values)
    st.close()


def test_lookahead_graph_replay_matches_direct_launches():
    import torch

    from sparse_weight_memory_b200 import FwPKMState
    wl = ITER.replace(lookahead=True)
    inp = make_inputs(wl)
    Q, Vt, g = to_dev(inp.Q), to_dev(inp.Vt), to_dev(inp.gate)
    res = []
    for graphs in (False, True):
        st = FwPKMState(wl.N, wl.dq, wl.dv, wl.topk, wl.chunk, wl.heads, eps=wl.eps)
        st.set_graphs(graphs)
        st.set_tables(to_dev(inp.subkeys), to_dev(inp.values))
        out = torch.empty((wl.B, wl.T, wl.dv), dtype=torch.float32, device="cuda")
        outs = []
        for _ in range(3):
            st.step(Q, Vt, g, wl.eta, wl.lam, out=out, lookahead=True)
            outs.append(out.cpu().numpy())
        K, V = st.get_tables()
        torch.cuda.synchronize()
        res.append((outs, K.cpu().numpy(), V.cpu().numpy()))
        st.close()
    for a, b in zip(res[0][0], res[1][0]):
        assert np.array_equal(a, b)
    assert np.array_equal(res[0][1], res[1][1]) and np.array_equal(res[0][2], res[1][2])


def test_unknown_flags_are_rejected():
    import ctypes

    import torch

    from sparse_weight_memory_b200 import FwPKMState
    from sparse_weight_memory_b200.fwpkm import FWPKM_EINVAL, load_library
    wl = WORKLOADS["tiny"]
    inp = make_inputs(wl)
    st = FwPKMState(wl.N, wl.dq, wl.dv, wl.topk, wl.chunk, wl.heads)
    Q, Vt, g = to_dev(inp.Q), to_dev(inp.Vt), to_dev(inp.gate)
    out = torch.empty((wl.B, wl.T, wl.dv), dtype=torch.float32, device="cuda")
    rc = load_library().fwpkm_step_ex(st._h, wl.B, wl.T, Q.data_ptr(), 0, Vt.data_ptr(), 0,
                                      g.data_ptr(), None, 2, 0.5, 0.0, out.data_ptr(),
                                      ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == FWPKM_EINVAL
    st.close()


def test_host_buffers_with_lookahead_and_weights_equal_the_device_step():
    """fwpkm_step_host_ex (host buffers, copies pipelined per chunk; the
    lookahead read waits for the next chunk's inputs) gives the device
    call's results bit for bit."""
    import torch

    from sparse_weight_memory_b200 import FwPKMState
    wl = WORKLOADS["library"].replace(B=3, T=3 * 256 + 7, calls=1)
    inp = make_inputs(wl)
    omega = (np.random.default_rng(5).random(inp.gate.shape) * 1.5).astype(np.float32)
    res = []
    for host in (False, True):
        st = FwPKMState(wl.N, wl.dq, wl.dv, wl.topk, wl.chunk, wl.heads)
        st.set_tables(to_dev(inp.subkeys), to_dev(inp.values))
        if host:
            out = st.step_host(inp.Q, inp.Vt, inp.gate, wl.eta, wl.lam, omega=omega,
                               lookahead=True)
        else:
            out = st.step(to_dev(inp.Q), to_dev(inp.Vt), to_dev(inp.gate), wl.eta, wl.lam,
                          omega=to_dev(omega), lookahead=True).cpu().numpy()
        torch.cuda.synchronize()
        K, V = st.get_tables()
        res.append((out, K.cpu().numpy(), V.cpu().numpy()))
        st.close()
    for a, b in zip(*res):
        assert np.array_equal(a, b)
