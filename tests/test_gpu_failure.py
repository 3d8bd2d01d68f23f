"""Failure detection on the GPU without a GPU fault.

Every device-side wait of the step is bounded (fwpkm_set_wait_limits).  A
bound of 0 makes a wait give up at once: the kernel sets its error bit,
still lets its own copies in flight land, and returns.  The kernels after the
bucket scan then skip the rest of the call, so the tables keep the values of
the last complete chunk, and fwpkm_read_stats reports the bits with
FWPKM_ECUDA.  Allocation failures are injected on the host
(fwpkm_inject_alloc_failures).  Nothing here traps, faults or hangs a GPU,
and after each failure the state is shown to be usable again.
"""
import ctypes

import numpy as np
import pytest

from sparse_weight_memory_b200.workloads import WORKLOADS, Workload, make_inputs

from fwpkm_testlib import to_dev

pytestmark = pytest.mark.gpu

ERR_SCAN_TIMEOUT, ERR_SCORE_TIMEOUT = 4, 8


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from sparse_weight_memory_b200 import build
    build.build()


def device_errors(st, reset=True):
    """(status, error bits) of fwpkm_read_stats, without raising."""
    import torch

    from sparse_weight_memory_b200.fwpkm import load_library
    err = ctypes.c_uint32()
    rc = load_library().fwpkm_read_stats(st._h, None, None, None, None, ctypes.byref(err),
                                         int(reset), torch.cuda.current_stream().cuda_stream)
    return rc, err.value


def fresh_state(wl, inp):
    from sparse_weight_memory_b200 import FwPKMState
    st = FwPKMState(wl.N, wl.dq, wl.dv, wl.topk, wl.chunk, wl.heads, eps=wl.eps)
    st.set_tables(to_dev(inp.subkeys), to_dev(inp.values))
    return st


def run_and_tables(st, wl, inp):
    import torch
    out = st.step(to_dev(inp.Q), to_dev(inp.Vt), to_dev(inp.gate), wl.eta, wl.lam)
    torch.cuda.synchronize()
    K, V = st.get_tables()
    torch.cuda.synchronize()
    return out.cpu().numpy(), K.cpu().numpy(), V.cpu().numpy()


def check_recovers(st, wl, inp):
    """With the limits restored and the bits reset, the state gives exactly
    the results of a fresh state on the same inputs."""
    st.set_wait_limits()
    st.set_tables(to_dev(inp.subkeys), to_dev(inp.values))
    got = run_and_tables(st, wl, inp)
    rc, bits = device_errors(st)
    assert rc == 0 and bits == 0
    ref_st = fresh_state(wl, inp)
    ref = run_and_tables(ref_st, wl, inp)
    ref_st.close()
    for a, b in zip(got, ref):
        assert np.array_equal(a, b)


# A shape whose bucket scan spans several CTAs (2048 buckets each): 128 x 128
# slots, 2048 rows per chunk with 32 pairs each, so 16,384 value buckets plus
# 256 sub-key rows.  The first CTA never waits; the later ones give up at once
# with a bound of 0, which the error bit then proves.
SCAN2 = Workload("scan2", B=1, T=4096, chunk=2048, heads=1, dq=16, n=128, dv=4, topk=32,
                 eta=0.5, lam=0.0, gate="uniform")


def test_scan_wait_gives_up_and_the_write_is_skipped():
    from sparse_weight_memory_b200.fwpkm import FWPKM_ECUDA
    wl = SCAN2
    inp = make_inputs(wl)
    st = fresh_state(wl, inp)
    st.set_wait_limits(scan_polls=0)
    _, K, V = run_and_tables(st, wl, inp)
    rc, bits = device_errors(st)
    assert rc == FWPKM_ECUDA
    assert bits & ERR_SCAN_TIMEOUT, bits
    # nothing after the give-up wrote the tables: they hold the initial values
    assert np.array_equal(K, inp.subkeys) and np.array_equal(V, inp.values)
    check_recovers(st, wl, inp)
    st.close()


def test_score_wait_gives_up_and_the_write_is_skipped():
    from sparse_weight_memory_b200.fwpkm import FWPKM_ECUDA
    wl = WORKLOADS["library"].replace(T=2 * 256, calls=1)
    inp = make_inputs(wl)
    st = fresh_state(wl, inp)
    st.set_wait_limits(mbar_polls=0)
    _, K, V = run_and_tables(st, wl, inp)
    rc, bits = device_errors(st)
    assert rc == FWPKM_ECUDA
    assert bits & ERR_SCORE_TIMEOUT, bits
    assert np.array_equal(K, inp.subkeys) and np.array_equal(V, inp.values)
    check_recovers(st, wl, inp)
    st.close()


def test_scratch_allocation_failure_leaves_the_state_usable():
    """A step that needs a larger scratch arena meets an (injected) failed
    allocation: ENOMEM, nothing enqueued, the state unchanged; the same call
    then succeeds."""
    import torch

    from sparse_weight_memory_b200 import FwpkmError
    from sparse_weight_memory_b200.fwpkm import FWPKM_ENOMEM, inject_alloc_failures
    wl = WORKLOADS["library"].replace(B=2, T=256, calls=1)
    inp = make_inputs(wl)
    st = fresh_state(wl.replace(B=1), inp)  # the arena starts at one chunk of 1 sequence
    inject_alloc_failures(1)
    try:
        with pytest.raises(FwpkmError) as e:
            st.step(to_dev(inp.Q), to_dev(inp.Vt), to_dev(inp.gate), wl.eta, wl.lam)
    finally:
        inject_alloc_failures(0)
    assert e.value.status == FWPKM_ENOMEM
    torch.cuda.synchronize()
    K, V = st.get_tables()
    torch.cuda.synchronize()
    assert np.array_equal(K.cpu().numpy(), inp.subkeys)
    assert np.array_equal(V.cpu().numpy(), inp.values)
    got = run_and_tables(st, wl, inp)
    ref_st = fresh_state(wl, inp)
    ref = run_and_tables(ref_st, wl, inp)
    ref_st.close()
    for a, b in zip(got, ref):
        assert np.array_equal(a, b)
    st.close()


def test_staging_allocation_failure_is_enomem():
    from sparse_weight_memory_b200 import FwpkmError
    from sparse_weight_memory_b200.fwpkm import FWPKM_ENOMEM, inject_alloc_failures
    wl = WORKLOADS["tiny"]
    inp = make_inputs(wl)
    st = fresh_state(wl, inp)
    inject_alloc_failures(1)
    try:
        with pytest.raises(FwpkmError) as e:
            st.step_host(inp.Q, inp.Vt, inp.gate, wl.eta, wl.lam)
    finally:
        inject_alloc_failures(0)
    assert e.value.status == FWPKM_ENOMEM
    out = st.step_host(inp.Q, inp.Vt, inp.gate, wl.eta, wl.lam)
    assert np.isfinite(out).all()
    st.close()
