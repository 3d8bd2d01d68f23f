"""The step's other readings on the GPU (fwpkm_state_set_options) against the
fp64 oracle with the same options: summed heads (the pypi page's multi-head
variant read the other way) and two other divisors of a value row's gradient
(the averaging of repeated-slot gradients, gist.science section 2: by the
access count, or none).  Tolerances and the near-tie policy of fwpkm_testlib.
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
