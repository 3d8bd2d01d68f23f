"""One memory per sequence in one state (fwpkm_state_init_batched), on the GPU.

The other reading of how memories relate to sequences: each of the B
sequences of a call reads and writes a memory of its own (the package page
chains one memory per call, pypi.org fast-weight-product-key-memory, Usage),
all B in the same launches.  Two references:
  * the oracle, as B separate fp64 states, one sequence each (parity at the
    tolerances of fwpkm_testlib);
  * a plain GPU state stepping that sequence alone: every per-memory sum
    runs in the same order, so the results must agree bit for bit.
"""
import numpy as np
import pytest

from sparse_weight_memory_b200.workloads import WORKLOADS, make_inputs

from fwpkm_testlib import (OUT_ATOL, OUT_RTOL, TIE_GAP, check_close, check_selection,
                           check_table, to_dev, widen)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from sparse_weight_memory_b200 import build
    build.build()


def memory_tables(wl, B):
    """B independent initial memories (the workload's recipe, seeds 100 + b)."""
    one = wl.replace(B=1)
    ins = [make_inputs(one, seed=100 + b) for b in range(B)]
    return np.stack([i.subkeys for i in ins]), np.stack([i.values for i in ins])


def run_batched(wl, inp, K0, V0, steps=1, force=None):
    import torch

    from sparse_weight_memory_b200 import FwPKMState
    B = inp.gate.shape[0]
    st = FwPKMState(wl.N, wl.dq, wl.dv, wl.topk, wl.chunk, wl.heads, eps=wl.eps, memories=B)
    st.set_tables(to_dev(K0), to_dev(V0))
    outs, sels = [], []
    for _ in range(steps):
        rs = torch.empty((B, wl.T, wl.heads, wl.topk), dtype=torch.int32, device="cuda")
        rw = torch.empty_like(rs, dtype=torch.float32)
        st.record_selection(rs, rw)
        if force is not None:
            st.force_selection(*force)
        out = st.step(to_dev(inp.Q), to_dev(inp.Vt), to_dev(inp.gate), wl.eta, wl.lam)
        outs.append(out.cpu().numpy())
        sels.append(rs.cpu().numpy())
    K, V = st.get_tables()
    torch.cuda.synchronize()
    res = (outs, sels, K.cpu().numpy(), V.cpu().numpy())
    st.close()
    return res


def run_single(wl, inp, b, K0, V0, steps=1):
    import torch

    from sparse_weight_memory_b200 import FwPKMState
    st = FwPKMState(wl.N, wl.dq, wl.dv, wl.topk, wl.chunk, wl.heads, eps=wl.eps)
    st.set_tables(to_dev(K0[b]), to_dev(V0[b]))
    sl = slice(b, b + 1)
    outs = []
    for _ in range(steps):
        out = st.step(to_dev(inp.Q[sl]), to_dev(inp.Vt[sl]), to_dev(inp.gate[sl]), wl.eta, wl.lam)
        outs.append(out.cpu().numpy()[0])
    K, V = st.get_tables()
    torch.cuda.synchronize()
    res = (outs, K.cpu().numpy(), V.cpu().numpy())
    st.close()
    return res


CASES = {
    # 3 memories of the library shape, a ragged last chunk (256-row chunks: no padding)
    "library_3": WORKLOADS["library"].replace(B=3, T=2 * 256 + 41, calls=1),
    # chunks of 100 rows: every sequence padded to a 128-row score tile; 2 heads, entropy
    "iterative_2_padded": WORKLOADS["iterative"].replace(B=2, T=230, chunk=100, passes=1),
    # bf16 queries and targets, 4 heads, entropy
    "multihead_2": WORKLOADS["multihead"].replace(B=2, T=512 + 19),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_batched_equals_one_state_per_sequence(name):
    """Bit for bit: memory b of the batched state after two calls equals a
    plain state that stepped sequence b alone, and so do the outputs."""
    wl = CASES[name]
    inp = make_inputs(wl)
    B = wl.B
    K0, V0 = memory_tables(wl, B)
    outs, _, K, V = run_batched(wl, inp, K0, V0, steps=2)
    for b in range(B):
        s_outs, sK, sV = run_single(wl, inp, b, K0, V0, steps=2)
        for step in range(2):
            assert np.array_equal(outs[step][b], s_outs[step]), (name, b, step)
        assert np.array_equal(K[b], sK) and np.array_equal(V[b], sV), (name, b)


@pytest.mark.parametrize("name", sorted(CASES))
def test_batched_parity_with_separate_oracle_states(oracle, name):
    """Against B oracle states, one sequence each; near ties forced to the
    oracle's choice (slots of the token's own memory)."""
    wl = CASES[name]
    inp = make_inputs(wl)
    B = wl.B
    K0, V0 = memory_tables(wl, B)
    refs = []
    for b in range(B):
        st = oracle.State(K0[b], V0[b], topk=wl.topk, chunk=wl.chunk, eps=wl.eps)
        r = st.step(widen(inp.Q[b:b + 1]), widen(inp.Vt[b:b + 1]), inp.gate[b:b + 1], wl.eta,
                    wl.lam, want_sel=True, want_gap=True)
        refs.append((r, st))
    sel_o = np.concatenate([r["sel_slot"] for r, _ in refs])
    gap_o = np.concatenate([r["gap"] for r, _ in refs])
    mask = to_dev((gap_o <= TIE_GAP).astype(np.uint8))
    slots = to_dev(sel_o.astype(np.int32))
    outs, sels, K, V = run_batched(wl, inp, K0, V0, force=(slots, mask))
    check_selection(sels[0], sel_o, gap_o, f"{name} selection")
    tol = 1e-4 if wl.n_chunks() <= 1 else 1e-3
    for b, (r, st) in enumerate(refs):
        check_close(outs[0][b], r["out"][0], OUT_ATOL, OUT_RTOL, f"{name} memory {b} out")
        check_table(V[b], st.V, tol, f"{name} memory {b} values")
        check_table(K[b], st.K, tol, f"{name} memory {b} sub-keys")


def test_batch_must_match_the_memories():
    import torch

    from sparse_weight_memory_b200 import FwPKMState, FwpkmError
    from sparse_weight_memory_b200.fwpkm import FWPKM_ESHAPE
    wl = WORKLOADS["tiny"]
    st = FwPKMState(wl.N, wl.dq, wl.dv, wl.topk, wl.chunk, memories=3)
    inp = make_inputs(wl.replace(B=2))
    with pytest.raises(FwpkmError) as e:
        st.step(to_dev(inp.Q), to_dev(inp.Vt), to_dev(inp.gate), 0.5)
    assert e.value.status == FWPKM_ESHAPE
    torch.cuda.synchronize()
    st.close()
