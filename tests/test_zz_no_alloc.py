"""fwpkm_select_noalloc: the selection entry point for callers that cannot
allocate device memory at call time (a server with a pre-planned, fixed
device-memory budget, or a plugin whose host framework owns the allocator).

Its slots and weights must equal what the existing fwpkm_step reads (eta = 0,
recorded with fwpkm_record_selection) for the same tables and queries, on two
calls in a row, and the calls must not take device memory.  Its error word
stays 0 on those calls, and reports a bounded wait that gives up.  Kept in a
file of its own that runs last.
"""
import numpy as np
import pytest

from sparse_weight_memory_b200.workloads import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch_cuda():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from sparse_weight_memory_b200 import build
    build.build()
    return torch


def to_dev(torch, a):
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).cuda().view(torch.bfloat16)
    return torch.from_numpy(a).cuda()


def reference_selection(torch, wl, inp, Q):
    """Slots and weights fwpkm_step reads with eta = 0 (tables unchanged)."""
    from sparse_weight_memory_b200 import FwPKMState
    st = FwPKMState(wl.N, wl.dq, wl.dv, wl.topk, wl.chunk, wl.heads, eps=wl.eps)
    st.set_tables(to_dev(torch, inp.subkeys), to_dev(torch, inp.values))
    B, T = Q.shape[0], Q.shape[1]
    slots = torch.empty((B, T, wl.heads, wl.topk), dtype=torch.int32, device="cuda")
    weights = torch.empty((B, T, wl.heads, wl.topk), dtype=torch.float32, device="cuda")
    st.record_selection(slots, weights)
    vt = torch.zeros((B, T, wl.dv), dtype=torch.float32, device="cuda")
    gate = torch.ones((B, T), dtype=torch.float32, device="cuda")
    st.step(Q, vt, gate, 0.0, 0.0)
    torch.cuda.synchronize()
    st.close()
    return slots.cpu().numpy(), weights.cpu().numpy()


@pytest.mark.parametrize("name,B,T", [("iterative", 4, 1000), ("multihead", 2, 300)])
def test_select_noalloc_matches_step_twice(torch_cuda, name, B, T):
    torch = torch_cuda
    from sparse_weight_memory_b200 import FwPKMState
    wl = WORKLOADS[name].replace(B=B, T=T)
    inp = make_inputs(wl)
    inp2 = make_inputs(wl, seed=wl.seed + 7)
    queries = [to_dev(torch, inp.Q), to_dev(torch, inp2.Q)]

    st = FwPKMState(wl.N, wl.dq, wl.dv, wl.topk, wl.chunk, wl.heads, eps=wl.eps)
    st.set_tables(to_dev(torch, inp.subkeys), to_dev(torch, inp.values))
    shape = (B, T, wl.heads, wl.topk)
    slots = torch.empty(shape, dtype=torch.int32, device="cuda")
    weights = torch.empty(shape, dtype=torch.float32, device="cuda")
    errors = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    for call, Q in enumerate(queries):
        slots.fill_(-1)
        weights.fill_(float("nan"))
        errors.fill_(-1)
        torch.cuda.synchronize()
        free_before = torch.cuda.mem_get_info()[0]
        st.select_noalloc(Q, slots, weights, errors)
        torch.cuda.synchronize()
        assert errors.item() == 0, f"call {call}: device error bits {errors.item():#x}"
        free_after = torch.cuda.mem_get_info()[0]
        if call > 0:  # the first call on a device may map the library's image
            assert free_after >= free_before - (1 << 20), (free_before, free_after)
        ref_s, ref_w = reference_selection(torch, wl, inp, Q)
        got_s, got_w = slots.cpu().numpy(), weights.cpu().numpy()
        assert np.array_equal(got_s, ref_s), f"call {call}: slots differ"
        err = np.abs(got_w.astype(np.float64) - ref_w)
        assert (err <= 1e-6 + 1e-5 * np.abs(ref_w)).all(), f"call {call}: weights {err.max()}"
    # the tables are read only
    K, V = st.get_tables()
    torch.cuda.synchronize()
    assert np.array_equal(K.cpu().numpy(), inp.subkeys)
    st.close()


def test_select_noalloc_rejects_oversized_batch(torch_cuda):
    torch = torch_cuda
    from sparse_weight_memory_b200 import FwPKMState, FwpkmError
    from sparse_weight_memory_b200.fwpkm import FWPKM_ESHAPE
    wl = WORKLOADS["longctx"].replace(T=1)
    st = FwPKMState(wl.N, wl.dq, wl.dv, wl.topk, wl.chunk, wl.heads)
    B = 4096  # 4096 rows x ~10 KB of per-row scratch > 16 MiB
    Q = torch.zeros((B, 1, wl.dq), dtype=torch.float32, device="cuda")
    slots = torch.empty((B, 1, 1, wl.topk), dtype=torch.int32, device="cuda")
    weights = torch.empty((B, 1, 1, wl.topk), dtype=torch.float32, device="cuda")
    with pytest.raises(FwpkmError) as e:
        st.select_noalloc(Q, slots, weights)
    assert e.value.status == FWPKM_ESHAPE and "static scratch" in str(e.value)
    st.close()


def test_select_noalloc_reports_a_wait_that_gives_up(torch_cuda):
    """With the state's wait bound at 0 the score kernel gives up before it
    issues a copy: the call's error word gets bit 8, the slots stay in range,
    nothing faults; with the bound restored the next call is clean and
    matches the step's selection again."""
    torch = torch_cuda
    from sparse_weight_memory_b200 import FwPKMState
    wl = WORKLOADS["iterative"].replace(B=2, T=100)
    inp = make_inputs(wl)
    Q = to_dev(torch, inp.Q)
    st = FwPKMState(wl.N, wl.dq, wl.dv, wl.topk, wl.chunk, wl.heads, eps=wl.eps)
    st.set_tables(to_dev(torch, inp.subkeys), to_dev(torch, inp.values))
    shape = (wl.B, wl.T, wl.heads, wl.topk)
    slots = torch.empty(shape, dtype=torch.int32, device="cuda")
    weights = torch.empty(shape, dtype=torch.float32, device="cuda")
    errors = torch.zeros((1,), dtype=torch.int32, device="cuda")
    st.set_wait_limits(mbar_polls=0)
    st.select_noalloc(Q, slots, weights, errors)
    torch.cuda.synchronize()
    assert errors.item() & 8, errors.item()
    got = slots.cpu().numpy()
    assert got.min() >= 0 and got.max() < wl.N
    st.set_wait_limits()
    st.select_noalloc(Q, slots, weights, errors)
    torch.cuda.synchronize()
    assert errors.item() == 0
    ref_s, _ = reference_selection(torch, wl, inp, Q)
    assert np.array_equal(slots.cpu().numpy(), ref_s)
    st.close()


def test_select_noalloc_rejects_tables_too_large_for_the_scratch(torch_cuda):
    """n = 1024 sub-keys of dq/2 = 1024 need ~17 MB for their split alone:
    no batch size fits, and the message says so."""
    torch = torch_cuda
    from sparse_weight_memory_b200 import FwPKMState, FwpkmError
    from sparse_weight_memory_b200.fwpkm import FWPKM_ESHAPE
    st = FwPKMState(1024 * 1024, 2048, 4, 4, 16, 1)
    Q = torch.zeros((1, 1, 2048), dtype=torch.float32, device="cuda")
    slots = torch.empty((1, 1, 1, 4), dtype=torch.int32, device="cuda")
    weights = torch.empty((1, 1, 1, 4), dtype=torch.float32, device="cuda")
    with pytest.raises(FwpkmError) as e:
        st.select_noalloc(Q, slots, weights)
    assert e.value.status == FWPKM_ESHAPE and "no batch size fits" in str(e.value)
    st.close()
