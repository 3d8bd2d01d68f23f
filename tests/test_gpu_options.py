"""The step's other readings on the GPU (fwpkm_state_set_options) against the
fp64 oracle with the same options: summed heads (the pypi page's multi-head
variant read the other way), two other divisors of a value row's gradient
(the averaging of repeated-slot gradients, gist.science section 2: by the
access count, or none), and the dot-product sub-key score (gist.science
section 2, Key Technical Choices: the score IDW is chosen over).  Tolerances
and the near-tie policy of fwpkm_testlib.
"""
import numpy as np
import pytest

from sparse_weight_memory_b200.workloads import WORKLOADS, make_inputs

from fwpkm_testlib import compare_runs, gpu_run, oracle_run

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from sparse_weight_memory_b200 import build
    build.build()


ITER = WORKLOADS["iterative"].replace(B=2, T=2 * 512 + 45)
MH = WORKLOADS["multihead"].replace(B=2, T=512 + 77)


@pytest.mark.parametrize("name,wl", [
    ("summed_heads_iterative", ITER.replace(heads_mode="sum", eta=0.1)),
    ("summed_heads_multihead_bf16", MH.replace(heads_mode="sum", eta=0.1)),
    ("count_iterative", ITER.replace(agg="count")),
    ("count_longctx", WORKLOADS["longctx"].replace(T=2 * 1024 + 100, agg="count")),
    ("plain_sum_multihead_bf16", MH.replace(agg="sum", eta=0.05)),
    ("summed_heads_and_count", ITER.replace(heads_mode="sum", agg="count", eta=0.1)),
    ("dot_iterative", ITER.replace(score="dot", eta=0.05)),
    ("dot_multihead_bf16", MH.replace(score="dot", eta=0.05)),
    # The dot-product score's sub-key gradient has no 1/(eps + d) factor: at
    # the long-context eta = 1 one chunk multiplies the key norms several-fold,
    # the scores' absolute fp32 error grows with them and the softmax passes it
    # on, so the dot-score cases take a step of 0.05.
    ("dot_longctx", WORKLOADS["longctx"].replace(T=2 * 1024 + 100, score="dot", eta=0.05)),
    ("dot_entropy", ITER.replace(score="dot", lam=0.3, eta=0.05)),
    ("dot_summed_heads_count_bf16", MH.replace(score="dot", heads_mode="sum", agg="count",
                                               eta=0.05)),
])
def test_options_parity(oracle, name, wl):
    inp = make_inputs(wl)
    o = oracle_run(wl, inp, oracle)
    g = gpu_run(wl, inp, o, force=True, with_stats=True)
    info = compare_runs(wl, inp, g, o, name)
    assert g.touched == o.touched
    assert info["dV_rel"] < 1e-3 and info["dK_rel"] < 1e-3, info


def test_exclusive_divisors_are_rejected():
    from sparse_weight_memory_b200 import FwPKMState, FwpkmError
    from sparse_weight_memory_b200.fwpkm import (FWPKM_AGG_COUNT, FWPKM_AGG_SUM, FWPKM_EINVAL,
                                                 load_library)
    wl = WORKLOADS["tiny"]
    st = FwPKMState(wl.N, wl.dq, wl.dv, wl.topk, wl.chunk)
    L = load_library()
    assert L.fwpkm_state_set_options(st._h, FWPKM_AGG_COUNT | FWPKM_AGG_SUM) == FWPKM_EINVAL
    assert L.fwpkm_state_set_options(st._h, 64) == FWPKM_EINVAL
    st.close()


def test_dot_selection_without_allocation_is_the_steps():
    """fwpkm_select_noalloc on a state with the dot-product score selects what
    the dot-product step reads (eta = 0), and that is the oracle's dot-product
    selection away from near ties."""
    import torch

    from sparse_weight_memory_b200 import FwPKMState

    from fwpkm_testlib import check_selection, tie_gap, to_dev
    wl = WORKLOADS["iterative"].replace(B=2, T=700, score="dot", eta=0.0)
    inp = make_inputs(wl)
    shape = (wl.B, wl.T, wl.heads, wl.topk)

    def state():
        st = FwPKMState(wl.N, wl.dq, wl.dv, wl.topk, wl.chunk, wl.heads, eps=wl.eps)
        st.set_options(score="dot")
        st.set_tables(to_dev(inp.subkeys), to_dev(inp.values))
        return st

    st = state()
    slots = torch.empty(shape, dtype=torch.int32, device="cuda")
    weights = torch.empty(shape, dtype=torch.float32, device="cuda")
    errors = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    st.select_noalloc(to_dev(inp.Q), slots, weights, errors)
    torch.cuda.synchronize()
    assert errors.item() == 0
    st.close()

    st = state()
    rs = torch.empty(shape, dtype=torch.int32, device="cuda")
    rw = torch.empty(shape, dtype=torch.float32, device="cuda")
    st.record_selection(rs, rw)
    st.step(to_dev(inp.Q), to_dev(inp.Vt), to_dev(inp.gate), 0.0, 0.0)
    torch.cuda.synchronize()
    st.close()
    assert np.array_equal(slots.cpu().numpy(), rs.cpu().numpy())
    assert np.array_equal(weights.cpu().numpy(), rw.cpu().numpy())

    from oracle import oracle
    o = oracle.State(inp.subkeys, inp.values, topk=wl.topk, chunk=wl.chunk, eps=wl.eps,
                     score="dot").step(inp.Q, inp.Vt, inp.gate, 0.0, 0.0, want_sel=True,
                                       want_gap=True)
    check_selection(slots.cpu().numpy(), o["sel_slot"], o["gap"], "dot selection",
                    tie_gap(wl, inp))


def test_dot_score_long_run_stays_finite():
    """With the dot-product score the top-k scores can lie hundreds apart, so
    some fp32 softmax weights are denormal, and a value row written only by
    such pairs has a denormal divisor C.  Scaling by eta / C overflowed there
    (NaN in the outputs within a 128-chunk long-context call).  The update
    divides G by C first: every output and table entry stays finite over the
    whole call, as the oracle's do (max |K| about 50 by its last chunk)."""
    import torch

    from sparse_weight_memory_b200 import FwPKMState

    from fwpkm_testlib import to_dev
    wl = WORKLOADS["longctx"].replace(score="dot", eta=0.05)
    inp = make_inputs(wl)
    st = FwPKMState(wl.N, wl.dq, wl.dv, wl.topk, wl.chunk, wl.heads, eps=wl.eps)
    st.set_options(score="dot")
    st.set_tables(to_dev(inp.subkeys), to_dev(inp.values))
    out = st.step(to_dev(inp.Q), to_dev(inp.Vt), to_dev(inp.gate), wl.eta, wl.lam)
    K, V = st.get_tables()
    torch.cuda.synchronize()
    assert bool(torch.isfinite(out).all()), "non-finite outputs"
    assert bool(torch.isfinite(K).all()) and bool(torch.isfinite(V).all()), "non-finite tables"
    st.close()
