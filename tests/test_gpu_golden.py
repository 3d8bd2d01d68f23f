"""The CUDA path against the hand-worked example of ``tests/golden/``.

The example (H=1, n=4, dh=2, dv=2, k=2, eps=1, three tokens in one chunk) is
zero-padded to the library's alignment (dh=8, dv=4).  Zero coordinates change
no distance, dot product or residual, so the expected values stay the
hand-worked fractions, and the padded coordinates must stay exactly zero.
Tolerances are those of the oracle comparisons (fwpkm_testlib).
"""
import numpy as np
import pytest

from sparse_weight_memory_b200.workloads import Inputs, Workload

from fwpkm_testlib import OUT_ATOL, OUT_RTOL, check_close, check_table, gpu_run
from golden_lib import arr, frac, load_hand_step, pad_last, pad_queries

pytestmark = pytest.mark.gpu

DH_TO, DV_TO = 8, 4


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from sparse_weight_memory_b200 import build
    build.build()


def padded_case(hs, lam):
    B, T = hs.gate.shape
    wl = Workload("hand_step", B=B, T=T, chunk=hs.chunk, heads=hs.heads, dq=2 * DH_TO, n=hs.n,
                  dv=DV_TO, topk=hs.topk, eta=hs.eta, lam=lam, gate="one", eps=hs.eps)
    f32 = np.float32
    inp = Inputs(wl, pad_last(hs.K, DH_TO).astype(f32), pad_last(hs.V, DV_TO).astype(f32),
                 pad_queries(hs.Q, hs.heads, hs.dq // 2, DH_TO).astype(f32),
                 pad_last(hs.Vt, DV_TO).astype(f32), hs.gate.astype(f32),
                 np.zeros((0, 2), np.int64))
    return wl, inp


def check_against_hand_values(hs, res, lam):
    exp = hs.expected
    sel, w = res.sels[0].astype(np.int64), res.ws[0].astype(np.float64)
    sel_h, w_h = np.array(exp["sel_slot"]), arr(exp["sel_w"])
    # slot sets; within a token-head, each slot's weight (token C's two slots
    # are tied, so their order is not compared)
    assert np.array_equal(np.sort(sel, axis=-1), np.sort(sel_h, axis=-1)), (sel, sel_h)
    for idx in np.ndindex(sel_h.shape[:-1]):
        want = dict(zip(sel_h[idx].tolist(), w_h[idx].tolist()))
        got = dict(zip(sel[idx].tolist(), w[idx].tolist()))
        for s_, w_ in want.items():
            assert abs(got[s_] - w_) <= 1e-6, (idx, s_, got[s_], w_)
    out = res.outs[0]
    check_close(out[..., :hs.dv], arr(exp["out"]), OUT_ATOL, OUT_RTOL, "hand step out")
    assert not out[..., hs.dv:].any()
    check_table(res.V[:, :hs.dv], hs.values_after(), 1e-4, "hand step values")
    assert not res.V[:, hs.dv:].any()
    check_table(res.K[..., :hs.dq // 2], hs.subkeys_after(lam), 1e-4, "hand step sub-keys")
    assert not res.K[..., hs.dq // 2:].any()
    assert res.touched == len(exp["values_after"])


@pytest.mark.parametrize("entropy", [False, True], ids=["mse", "entropy"])
def test_hand_step_on_gpu(entropy):
    hs = load_hand_step()
    lam = frac(hs.raw["entropy"]["lambda"]) if entropy else 0.0
    wl, inp = padded_case(hs, lam)
    res = gpu_run(wl, inp, None, force=False, with_stats=True)
    check_against_hand_values(hs, res, lam)


def test_hand_step_lookahead_on_gpu():
    """The hand-worked step with the lookahead pairing q_t -> v_{t+1}: the
    reads are those of the plain step; the write follows the fixture's
    lookahead section (the last token, weight 0, pulls no row)."""
    hs = load_hand_step()
    la = hs.raw["lookahead"]
    wl, inp = padded_case(hs, 0.0)
    res = gpu_run(wl.replace(lookahead=True), inp, None, force=False, with_stats=True)
    exp = hs.expected
    assert np.array_equal(np.sort(res.sels[0].astype(np.int64), axis=-1),
                          np.sort(np.array(exp["sel_slot"]), axis=-1))
    out = res.outs[0]
    check_close(out[..., :hs.dv], arr(exp["out"]), OUT_ATOL, OUT_RTOL, "lookahead out")
    V = hs.V.copy()
    for r, row in la["values_after"].items():
        V[int(r)] = arr(row)
    check_table(res.V[:, :hs.dv], V, 1e-4, "lookahead values")
    assert not res.V[:, hs.dv:].any()
    K = hs.K.copy()
    for key, row in la["subkeys_after"].items():
        K[tuple(int(v) for v in key.split(","))] = arr(row)
    check_table(res.K[..., :hs.dq // 2], K, 1e-4, "lookahead sub-keys")
    assert not res.K[..., hs.dq // 2:].any()


@pytest.mark.parametrize("agg", ["count", "sum"])
def test_hand_step_other_row_divisors_on_gpu(agg):
    """The fixture's value rows divided by their access count, or not at all."""
    hs = load_hand_step()
    wl, inp = padded_case(hs, 0.0)
    res = gpu_run(wl.replace(agg=agg), inp, None, force=False)
    V = hs.V.copy()
    for r, row in hs.raw["aggregation"][agg]["values_after"].items():
        V[int(r)] = arr(row)
    check_table(res.V[:, :hs.dv], V, 1e-4, f"{agg} values")
    assert not res.V[:, hs.dv:].any()
    check_table(res.K[..., :hs.dq // 2], hs.subkeys_after(), 1e-4, f"{agg} sub-keys")


def test_hand_step_two_heads_summed_on_gpu():
    """The two-head fixture with the head readouts summed."""
    hs = load_hand_step("hand_step_two_heads.yaml")
    part = hs.raw["heads_sum"]
    wl, inp = padded_case(hs, 0.0)
    res = gpu_run(wl.replace(heads_mode="sum"), inp, None, force=False)
    check_close(res.outs[0][..., :hs.dv], arr(part["out"]), OUT_ATOL, OUT_RTOL, "summed out")
    V = hs.V.copy()
    for r, row in part["values_after"].items():
        V[int(r)] = arr(row)
    check_table(res.V[:, :hs.dv], V, 1e-4, "summed values")
    K = hs.K.copy()
    for key, row in part["subkeys_after"].items():
        K[tuple(int(v) for v in key.split(","))] = arr(row)
    check_table(res.K[..., :hs.dq // 2], K, 1e-4, "summed sub-keys")
    assert not res.K[..., hs.dq // 2:].any()
