"""The bench's roofline arithmetic on the CPU: algorithmic work per kernel as
the design notes define it, achieved = work per launch / launch time,
frac = achieved / peak, and the tf32 peak derived from the bf16 one."""
import json
import os

import pytest

import bench
from sparse_weight_memory_b200.workloads import BF16, WORKLOADS


def test_algorithmic_work_matches_the_per_unit_definitions():
    wl = WORKLOADS["library"]  # fp32 inputs, H=1, k=8, dv=dq=512, n=256
    segments = 3
    tokens, U_v, U_k, records = segments * wl.B * wl.T, 3000, 400, 10000
    w = bench.algorithmic_work(wl, tokens, segments, U_v, U_k, records)
    # read, per token: H*k*dv*4 gathered + dv*4 target (fp32) + dv*4 out
    assert w["fwpkm_read"] == ("hbm", tokens * (1 * 8 * 512 * 4 + 512 * 4 + 512 * 4))
    # apply: read-modify-write of the written value rows and sub-key rows
    assert w["fwpkm_apply"] == ("hbm", 2 * U_v * 512 * 4 + 2 * U_k * 256 * 4)
    # score: 2 * n * dq fp32 flops per token-head
    assert w["fwpkm_score"] == ("tensor", 2.0 * tokens * 1 * 256 * 512)
    # topk, per token-head: both halves' n distances read, k (slot, weight) written
    assert w["fwpkm_topk"] == ("hbm", tokens * (2 * 256 * 4 + 8 * 8))
    # query halves per token-head: q read (4 B), hi + lo written (8 B), a norm per half
    halves = lambda t: t * (512 * (4 + 8) + 2 * 4)
    first = segments * wl.B * min(wl.chunk, wl.T)  # the first chunk of each call
    # prep: the first chunk's halves and, once per call, every sub-key row of
    # both halves split (fp32 read, hi + lo written, two 128-float chunk norms)
    assert w["fwpkm_prep"] == ("hbm", halves(first) + segments * 2 * 256 * (256 * 12 + 2 * 4))
    # sort: records read and written (32 B each), and the later chunks' halves
    assert w["fwpkm_bsort"] == ("hbm", 2 * 32 * records + halves(tokens - first))


def test_bf16_inputs_halve_the_streamed_target_bytes():
    wl = WORKLOADS["multihead"]
    assert wl.in_dtype == BF16
    tokens = 1000
    w = bench.algorithmic_work(wl, tokens, 1, 0, 0, 0)
    gather = tokens * wl.heads * wl.topk * wl.dv * 4
    assert w["fwpkm_read"][1] == gather + tokens * wl.dv * 2 + tokens * wl.dv * 4


def test_kernel_roofline_hbm_and_tensor():
    # 10 launches moving 2e6 bytes each in 1 ms total: 2e6 B / 100 us = 20 GB/s
    r = bench.kernel_roofline("k", ("hbm", 2e7), 1.0, 10, 6545.0, 1608.5, "measured", None)
    assert r["achieved"] == pytest.approx(20.0)
    assert r["frac"] == pytest.approx(20.0 / 6545.0)
    assert r["unit"] == "GB/s" and r["us_per_launch"] == pytest.approx(100.0)
    assert r["frac_vs_nominal_8000"] == pytest.approx(20.0 / 8000.0)
    # 4 launches of 1e9 flops in 2 ms: 1e9 / 0.5 ms = 2 TFLOP/s against tf32
    t = bench.kernel_roofline("s", ("tensor", 4e9), 2.0, 4, 6545.0, 1608.5, "measured", None)
    peak = 1608.5 * 1.1 / 2.25
    assert t["peak"] == pytest.approx(peak) and bench.tensor_peak_tf32(1608.5) == pytest.approx(peak)
    assert t["achieved"] == pytest.approx(2.0) and t["frac"] == pytest.approx(2.0 / peak)


def test_peaks_come_from_the_measured_file():
    path = os.path.join(bench.ROOT, "MEASURED_PEAKS.json")
    if not os.path.exists(path):
        pytest.skip("no measured peaks on this machine")
    with open(path) as f:
        p = json.load(f)
    assert bench.peaks() == (float(p["hbm_gbs"]), float(p["bf16_tflops"]), "measured")
