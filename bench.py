"""Benchmark of the FwPKM chunked read-then-write step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload longctx]
                    [--impl reference]

A step is one pass of the whole hot path over one batch of the workload: for
the default `longctx` workload (B=1, T=131,072, chunk 1024, N=1,048,576 slots
(a 2 GiB value table), dq=dv=512, topk 32, 1% planted recalls) that is one
call of 128 chunks = 131,072 tokens, each chunk read and then written.
Inputs are resident in HBM when the timed region starts; between steps
(untimed) the tables are reset to their initial values and L2 is flushed by
writing a 256 MiB buffer.  Every step is timed with CUDA events on the
launching stream.

Multi-GPU: the step does not shard (chunks are sequential and all token-heads
of a chunk write one shared table), so `--gpus N` runs N independent
replicas, one per GPU, with no collective on the data path (weak scaling);
torch.distributed only provides the barrier and the max-over-ranks time.

`--impl reference` times the fp64 CPU oracle (the only reference this method
has) on the host cores, on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from sparse_weight_memory_b200.workloads import (BF16, WORKLOADS, bf16_bits_to_f32,  # noqa: E402
                                                make_inputs)

METRIC = "FwPKM tokens/sec (read+write per chunk), 1xB200; % of HBM/tensor roofline"
UNIT = "tokens/s"


def describe(wl) -> str:
    s = (f"{wl.name}: B={wl.B} T={wl.T} chunk={wl.chunk} heads={wl.heads} dq={wl.dq} "
         f"n={wl.n} (N={wl.N}) dv={wl.dv} topk={wl.topk} eta={wl.eta} "
         f"lambda={wl.lam} gate={wl.gate} inputs={'bf16' if wl.in_dtype == BF16 else 'f32'}")
    if wl.calls > 1:
        s += f" x{wl.calls} chained calls"
    if wl.passes > 1:
        s += f" x{wl.passes} passes"
    if wl.lookahead:
        s += " lookahead (q_t written towards v_t+1)"
    if wl.per_sequence:
        s += f" one memory per sequence ({wl.B} memories)"
    if wl.score != "idw":
        s += f" score={wl.score}"
    return s


def config_for(wl, world: int) -> dict:
    """The `config` object both arms print for a workload."""
    return {"workload": describe(wl), "parallelism": f"replicas{world}",
            "l2": "flushed between steps (256 MiB write), tables reset untimed",
            "tokens_per_step": wl.tokens_per_step}


def max_over_ranks(x: float, device=None) -> float:
    """Max of a per-rank number over the process group (identity when there
    is no group).  Every rank must call it at the same point."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_step_per_rank: float, steps: int, world: int,
                   total_ms_max: float) -> float:
    """Units all ranks processed / the slowest rank's time (weak scaling)."""
    return units_per_step_per_rank * steps * world / (total_ms_max / 1e3)


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), "measured"
    except Exception:
        return 6650.0, 1590.0, "fallback"


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    """Polls the GPU's SM clock and clock-event reasons through NVML (read
    only) every few milliseconds while the timed region runs."""

    # NVML clock-event reason bits
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown"}

    def __init__(self, torch_device_index: int, period_s: float = 0.002):
        self.dev = torch_device_index
        self.period = period_s
        self.samples = []
        self.mx = None
        self._stop = None
        self._thread = None
        self.error = None

    def _handle(self, nv):
        import torch
        try:
            p = torch.cuda.get_device_properties(self.dev)
            bus = f"{p.pci_domain_id:08x}:{p.pci_bus_id:02x}:{p.pci_device_id:02x}.0"
            return nv.nvmlDeviceGetHandleByPciBusId(bus)
        except Exception:
            return nv.nvmlDeviceGetHandleByIndex(self.dev)

    def _run(self, nv, h):
        while not self._stop.is_set():
            try:
                sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                bits = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                self.samples.append((sm, bits))
            except Exception as e:  # keep the timed region going
                self.error = repr(e)
                return
            self._stop.wait(self.period)

    def __enter__(self):
        import threading
        try:
            import pynvml as nv
            nv.nvmlInit()
            h = self._handle(nv)
            self.mx = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
        except Exception as e:
            self.error = repr(e)
            return self
        self._stop = threading.Event()
        self._thread = threading.Thread(target=self._run, args=(nv, h), daemon=True)
        self._thread.start()
        return self

    def __exit__(self, *a):
        if self._thread is not None:
            self._stop.set()
            self._thread.join(timeout=5)

    def summary(self) -> dict:
        sm = [x for x, _ in self.samples]
        reasons = sorted({name for _, bits in self.samples
                          for bit, name in self.REASONS.items() if bits & bit})
        out = {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": self.mx,
               "reasons": reasons, "samples": len(sm), "source": "nvml"}
        if self.error:
            out["error"] = self.error
        return out


# ---------------------------------------------------------------------------
# oracle (CPU) arm
# ---------------------------------------------------------------------------
def widen_inputs(a) -> np.ndarray:
    """fp32, or bf16 bit patterns, widened exactly to fp64."""
    if a.dtype == np.uint16:
        return bf16_bits_to_f32(a).astype(np.float64)
    return a.astype(np.float64)


class OracleSampler:
    """Times the fp64 oracle on the workload step, chunk by chunk and in the
    step's order (calls, then passes, then chunks), one state carried across
    chunks exactly as one call carries it.  Each sample runs chunks until its
    budget of oracle time is spent; the next sample continues where it
    stopped, and the walk starts over from the initial tables after the last
    chunk of the step."""

    def __init__(self, wl, inp):
        self.wl, self.inp = wl, inp
        self.seq = [(c, t0) for c in range(wl.calls) for _ in range(wl.passes)
                    for t0 in range(0, wl.T, wl.chunk)]
        self.pos = 0
        self.state = None

    def _fresh(self):
        from oracle import oracle as orc
        wl, inp = self.wl, self.inp
        # one state shared by the sequences, or one per sequence (all starting
        # from the workload's tables)
        self.state = [orc.State(inp.subkeys, inp.values, topk=wl.topk, chunk=wl.chunk,
                                eps=wl.eps, heads=wl.heads_mode, agg=wl.agg, score=wl.score)
                      for _ in range(wl.B if wl.per_sequence else 1)]

    def sample(self, budget_s: float):
        from oracle import oracle as orc
        wl, inp = self.wl, self.inp
        tokens, elapsed, chunks = 0, 0.0, 0
        while elapsed < budget_s:
            if self.pos == 0 or self.state is None:
                self._fresh()
            c, t0 = self.seq[self.pos]
            lo, hi = c * wl.T + t0, c * wl.T + min(wl.T, t0 + wl.chunk)
            Q = widen_inputs(inp.Q[:, lo:hi])
            g = inp.gate[:, lo:hi]
            om = None
            if wl.lookahead:
                # the call's pairing q_t -> v_{t+1}; its last token has weight 0
                end = (c + 1) * wl.T
                Vt = widen_inputs(inp.Vt[:, lo + 1:min(hi + 1, end)])
                om = g.astype(np.float64).copy()
                if hi == end:
                    Vt = np.concatenate([Vt, np.zeros_like(Vt[:, :1])], axis=1)
                    om[:, -1] = 0.0
            else:
                Vt = widen_inputs(inp.Vt[:, lo:hi])
            t = time.perf_counter()
            if len(self.state) == 1:
                self.state[0].step(Q, Vt, g, wl.eta, wl.lam, omega=om)
            else:
                for b, st in enumerate(self.state):
                    st.step(Q[b:b + 1], Vt[b:b + 1], g[b:b + 1], wl.eta, wl.lam,
                            omega=None if om is None else om[b:b + 1])
            elapsed += time.perf_counter() - t
            tokens += wl.B * (hi - lo)
            chunks += 1
            self.pos = (self.pos + 1) % len(self.seq)
        desc = (f"{chunks} chunk(s) of the workload step in order ({tokens} tokens; "
                f"{len(self.seq)} chunks per step), fp64 oracle")
        return tokens / elapsed, elapsed, desc, orc.num_threads()


def run_reference(args, wl):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    inp = make_inputs(wl)
    vals = []
    info = None
    sampler = OracleSampler(wl, inp)
    for i in range(args.warmup + args.steps):
        v, el, sample, cores = sampler.sample(args.ref_budget)
        if i >= args.warmup:
            vals.append((v, el))
        info = (sample, cores)
    tok_s = statistics.median([v for v, _ in vals])
    ms = statistics.median([el for _, el in vals]) * 1e3
    line = {"impl": "reference", "metric": METRIC, "value": tok_s, "unit": UNIT,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_for(wl, args.gpus),
            "cpu_baseline": {"value": tok_s, "unit": UNIT, "cores": info[1], "kind": "oracle",
                             "sample": info[0]},
            "e2e": {"value": tok_s, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------
def algorithmic_work(wl, tokens, segments, value_rows, key_rows, records, memories=1):
    """Algorithmic bytes (HBM-bound kernels) or flops (score) over `tokens`
    tokens in `segments` step calls, whose chunks wrote `value_rows` /
    `key_rows` distinct rows and grouped `records` member records."""
    in_b = 2 if wl.in_dtype == BF16 else 4
    gather = tokens * wl.heads * wl.topk * wl.dv * 4
    dh = wl.dq // 2
    # query halves of `t` tokens: read, written as TF32 hi + lo, and a norm per half
    def halves(t):
        return t * wl.heads * (wl.dq * (in_b + 8) + 2 * 4)
    # the prep makes the first chunk's halves of each call and splits every
    # sub-key row once per call (hi + lo + its 128-float chunk norms); the
    # sort's extra CTAs make the halves of every later chunk
    first = segments * wl.B * min(wl.chunk, wl.T)
    split = segments * memories * 2 * wl.heads * wl.n * (dh * (4 + 8) + -(-dh // 128) * 4)
    return {
        # gathered value rows + Vtarget read + out written
        "fwpkm_read": ("hbm", gather + tokens * wl.dv * in_b + tokens * wl.dv * 4),
        # read-modify-write of every touched value row and sub-key row
        "fwpkm_apply": ("hbm", 2 * value_rows * wl.dv * 4 + 2 * key_rows * (wl.dq // 2) * 4),
        # q_half . K_row for every sub-key of both halves (fp32 products)
        "fwpkm_score": ("tensor", 2.0 * tokens * wl.heads * wl.n * wl.dq),
        # member records read in claim order and written grouped (32 bytes each),
        # and the next chunks' query halves
        "fwpkm_bsort": ("hbm", 2 * 32 * records + halves(tokens - first)),
        # distance matrix read once, slots + weights written
        "fwpkm_topk": ("hbm", tokens * wl.heads * (2 * wl.n * 4 + wl.topk * 8)),
        "fwpkm_prep": ("hbm", halves(first) + split),
    }


# Per-launch DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum, bytes)
# of the kernels as last captured with ncu (cold caches), keyed by workload and
# kernel; the captures and their commands are summarised in profiles/.
# Missing = no capture of the current kernel.
NCU_TRAFFIC = {
    # longctx: captures of commit a3bdd73 (fwpkm_apply: 3b2b6da), one chunk of 1024 tokens
    # (the unit of a launch at any call length) taken in a 32-chunk call, chunk 29 of the last
    # warm-up step; ncu flushes the caches before each pass, so these are cold-cache bytes
    "longctx": {"fwpkm_read": 17.811e6, "fwpkm_apply": 21.680e6, "fwpkm_bsort": 3.958e6,
                "fwpkm_topk": 8.496e6, "fwpkm_score": 8.485e6, "fwpkm_scan": 0.052e6},
}


def tensor_peak_tf32(bf16_tf):
    """Dense tf32 tensor peak: the measured bf16 figure x the nominal ratio
    1.1 / 2.25 PFLOP/s.  The score kernel issues three tf32 products per fp32
    product (hi*hi + hi*lo + lo*hi), so its fp32-equivalent ceiling is a third
    of this."""
    return bf16_tf * 1.1 / 2.25


def kernel_roofline(name, work, ms, launches, hbm_gbs, bf16_tf, peak_kind, traffic):
    bound, amount = work
    per_launch = amount / launches
    sec = ms / launches / 1e3
    if bound == "hbm":
        achieved, peak, unit = per_launch / sec / 1e9, hbm_gbs, "GB/s"
        note = f"{peak_kind} copy bandwidth"
    else:
        achieved, peak, unit = per_launch / sec / 1e12, tensor_peak_tf32(bf16_tf), "TFLOP/s"
        note = (f"{peak_kind} bf16 x 1.1/2.25 (tf32); achieved counts fp32 products once, "
                f"the 3xTF32 split issues 3 tf32 products each, so frac <= 1/3")
    out = {"kernel": name, "bound": bound, "achieved": achieved, "peak": peak, "unit": unit,
           "frac": achieved / peak, "traffic": traffic,
           "algorithmic_per_launch": per_launch, "us_per_launch": sec * 1e6, "peak_kind": note}
    if bound == "hbm":
        out["frac_vs_nominal_8000"] = achieved / 8000.0  # HBM3e nominal, GB/s
    return out


def run_gpu(args, wl):
    import torch
    import torch.distributed as dist

    from sparse_weight_memory_b200 import FwPKMState, load_library
    from sparse_weight_memory_b200 import build as fwbuild

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    if rank == 0:
        fwbuild.build()
    if world > 1:
        dist.barrier()
    load_library()

    dev = torch.device("cuda", local)
    inp = make_inputs(wl, seed=wl.seed + rank)  # independent replica per rank

    def to_dev(a):
        a = np.ascontiguousarray(a)
        if a.dtype == np.uint16:
            return torch.from_numpy(a.view(np.int16)).to(dev).view(torch.bfloat16)
        return torch.from_numpy(a).to(dev)

    mem = wl.B if wl.per_sequence else 1
    if mem > 1:  # every memory starts from the workload's tables
        K0 = to_dev(np.stack([inp.subkeys] * mem))
        V0 = to_dev(np.stack([inp.values] * mem))
    else:
        K0, V0 = to_dev(inp.subkeys), to_dev(inp.values)
    segs = []
    for c in range(wl.calls):
        sl = slice(c * wl.T, (c + 1) * wl.T)
        dq_, dv_, dg_ = to_dev(inp.Q[:, sl]), to_dev(inp.Vt[:, sl]), to_dev(inp.gate[:, sl])
        for _ in range(wl.passes):
            segs.append((dq_, dv_, dg_))
    outs = [torch.empty((wl.B, wl.T, wl.dv), dtype=torch.float32, device=dev) for _ in segs]
    st = FwPKMState(wl.N, wl.dq, wl.dv, wl.topk, wl.chunk, wl.heads, eps=wl.eps, memories=mem)
    st.set_options(heads=wl.heads_mode, agg=wl.agg, score=wl.score)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def reset():
        st.set_tables(K0, V0)
        flush.zero_()

    def one_step():
        for (q, v, g), o in zip(segs, outs):
            st.step(q, v, g, wl.eta, wl.lam, out=o, lookahead=wl.lookahead)

    for _ in range(args.warmup):
        reset()
        one_step()
    torch.cuda.synchronize()
    st.read_stats(reset=True)

    times = []
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        for _ in range(args.steps):
            reset()
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            one_step()
            b.record(stream)
            times.append((a, b))
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    step_ms = [a.elapsed_time(b) for a, b in times]
    recall = None
    if len(inp.plants):
        # Planted recalls (a position repeating an earlier (q, v) pair): the
        # squared error of the readout there against the planted target, next
        # to the same at all other positions, from the last timed step.
        pos = torch.from_numpy(inp.plants[:, 0]).to(dev)
        err = []
        for c in range(wl.calls):
            o = outs[c * wl.passes + wl.passes - 1]
            lo, hi = c * wl.T, (c + 1) * wl.T
            sel = pos[(pos >= lo) & (pos < hi)] - lo
            vt = torch.from_numpy(np.ascontiguousarray(inp.vt_f32()[:, lo:hi])).to(dev)
            se = ((o - vt) ** 2).mean(dim=-1)  # [B, T]
            mask = torch.zeros(wl.T, dtype=torch.bool, device=dev)
            mask[sel] = True
            err.append((se[:, mask].sum().item(), int(mask.sum().item()) * wl.B,
                        se[:, ~mask].sum().item(), int((~mask).sum().item()) * wl.B))
        recall = {"planted_mse": sum(e[0] for e in err) / max(1, sum(e[1] for e in err)),
                  "other_mse": sum(e[2] for e in err) / max(1, sum(e[3] for e in err)),
                  "planted_positions": int(sum(e[1] for e in err))}
    total_ms = sum(step_ms)
    stats = st.read_stats(reset=True)
    total_ms_max = max_over_ranks(total_ms, dev)
    tokens_per_step = wl.tokens_per_step
    value = whole_job_rate(tokens_per_step, args.steps, world, total_ms_max)

    # per-kernel event timing (separate, instrumented steps)
    st.set_profiling(True)
    prof_steps = max(1, min(args.steps, 3))
    for _ in range(prof_steps):
        reset()
        one_step()
    torch.cuda.synchronize()
    prof = st.profile_read()
    st.set_profiling(False)
    pstats = st.read_stats(reset=True)

    # end to end through the C ABI with pinned host buffers
    hsegs = []
    for c in range(wl.calls):
        sl = slice(c * wl.T, (c + 1) * wl.T)
        hq = torch.from_numpy(np.ascontiguousarray(inp.Q[:, sl])).pin_memory().numpy()
        hv = torch.from_numpy(np.ascontiguousarray(inp.Vt[:, sl])).pin_memory().numpy()
        hg = torch.from_numpy(np.ascontiguousarray(inp.gate[:, sl])).pin_memory().numpy()
        for _ in range(wl.passes):
            hsegs.append((hq, hv, hg))
    hout = torch.empty((wl.B, wl.T, wl.dv), dtype=torch.float32).pin_memory().numpy()
    h2d = sum(q.nbytes + v.nbytes + g.nbytes for q, v, g in hsegs)
    d2h = hout.nbytes * len(hsegs)
    e2e_ms = []
    for i in range(args.warmup + args.steps):
        reset()
        torch.cuda.synchronize()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for q, v, g in hsegs:
            st.step_host(q, v, g, wl.eta, wl.lam, out=hout, lookahead=wl.lookahead)
        b.record(stream)
        torch.cuda.synchronize()
        if i >= args.warmup:
            e2e_ms.append(a.elapsed_time(b))
    e2e_value = whole_job_rate(tokens_per_step, args.steps, world,
                               max_over_ranks(sum(e2e_ms), dev))

    if rank == 0:
        hbm_gbs, bf16_tf, peak_kind = peaks()
        rows_sum = wl.B * wl.T * wl.calls * wl.passes * prof_steps
        segs_sum = wl.calls * wl.passes * prof_steps
        work = algorithmic_work(wl, rows_sum, segs_sum, pstats["value_rows"], pstats["key_rows"],
                                pstats["records"], wl.B if wl.per_sequence else 1)
        traffic = NCU_TRAFFIC.get(wl.name, {})
        fracs = {k: kernel_roofline(k, work[k], ms, n, hbm_gbs, bf16_tf, peak_kind,
                                    traffic.get(k))
                 for k, (ms, n) in prof.items() if k in work and n > 0}
        dominant = max(prof.items(), key=lambda kv: kv[1][0])[0]
        roofline = fracs.get(dominant)
        if roofline is None:  # the longest kernel has no algorithmic-work model
            roofline = {"kernel": dominant, "bound": None, "achieved": None, "peak": None,
                        "unit": None, "frac": None, "traffic": None}
        # Events inside the timed steps would break the launch chaining and the
        # graph replay they measure, so kernels are timed in separate steps.
        roofline = dict(roofline, timing=(
            f"CUDA event pair around every launch on the launching stream, over {prof_steps} "
            "instrumented steps run after the timed ones (same inputs, no programmatic "
            "dependent launch, no graphs)"))
        kernels = {k: {"ms_per_step": v[0] / prof_steps, "launches_per_step": v[1] / prof_steps,
                       "share": v[0] / sum(x[0] for x in prof.values()),
                       "frac": fracs[k]["frac"] if k in fracs else None}
                   for k, v in prof.items()}
        # whole-step roofline: gathered + scattered + streamed bytes at HBM peak
        vrows = stats["value_rows"] / args.steps
        in_b = 2 if wl.in_dtype == BF16 else 4
        tok = wl.tokens_per_step
        step_bytes = (tok * wl.heads * wl.topk * wl.dv * 4 + 2 * vrows * wl.dv * 4 +
                      tok * (wl.heads * wl.dq * in_b + wl.dv * in_b + 4 + wl.dv * 4))
        step_flops = 2.0 * tok * wl.heads * wl.n * wl.dq
        t_roof = max(step_bytes / (hbm_gbs * 1e9),
                     step_flops / (tensor_peak_tf32(bf16_tf) / 3 * 1e12))
        clocks = clk.summary()
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            v, el, sample, cores = OracleSampler(wl, inp).sample(args.ref_budget)
            cpu = {"value": v, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample}
        launches = sum(int(round(x["launches_per_step"])) for x in kernels.values()) * args.steps
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": total_ms_max / args.steps,
            "step_ms": {"median": statistics.median(step_ms), "best": min(step_ms)},
            "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": config_for(wl, world),
            "roofline": roofline,
            "step_roofline": {"bytes_per_step": step_bytes, "flops_per_step": step_flops,
                              "t_roof_ms": t_roof * 1e3,
                              "frac": t_roof * 1e3 / (total_ms_max / args.steps),
                              "value_rows_per_step": vrows,
                              # the instrumented steps' kernel times, summed: above the
                              # timed step by what chaining and graphs hide
                              "instrumented_kernels_ms_per_step":
                                  sum(v[0] for v in prof.values()) / prof_steps},
            "kernels": kernels,
            "cpu_baseline": cpu,
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h},
            "gpu_launches": launches,
            "recall": recall,
            "clocks": clocks,
        }
        print(json.dumps(line), flush=True)
    st.close()
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="longctx", choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--ref-budget", type=float, default=5.0,
                    help="seconds of oracle time per reference sample (the chunks of "
                         "the step in order, continued by the next sample)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--tokens", type=int, default=0,
                    help="tokens per sequence and call (default: the workload's T); a "
                         "shorter run of the same shape, for profiler captures")
    ap.add_argument("--passes", type=int, default=0,
                    help="reads of each segment with the memory carried over (default: the "
                         "workload's)")
    ap.add_argument("--per-sequence", action="store_true",
                    help="one memory per sequence: the B sequences of a call each read and "
                         "write their own memory, in the same launches")
    ap.add_argument("--eta", type=float, default=None,
                    help="learning rate of the update (default: the workload's)")
    ap.add_argument("--score", choices=["idw", "dot"], default="idw",
                    help="sub-key score: -log(eps + |q - K|^2) (default) or the dot product")
    ap.add_argument("--lookahead", action="store_true",
                    help="write query t towards the target of token t+1 (each call's last "
                         "token has weight 0)")
    args = ap.parse_args()
    wl = WORKLOADS[args.workload]
    if args.tokens:
        wl = wl.replace(T=args.tokens)
    if args.passes:
        wl = wl.replace(passes=args.passes)
    if args.lookahead:
        wl = wl.replace(lookahead=True)
    if args.per_sequence:
        wl = wl.replace(per_sequence=True)
    if args.score != "idw":
        wl = wl.replace(score=args.score)
    if args.eta is not None:
        wl = wl.replace(eta=args.eta)
    if args.impl == "reference":
        run_reference(args, wl)
    else:
        run_gpu(args, wl)


if __name__ == "__main__":
    main()
