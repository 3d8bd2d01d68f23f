"""Seeded synthetic workloads for the FwPKM chunked read-then-write step.

This module only draws numbers: it holds none of the method's arithmetic, so
the CPU oracle (``oracle/``) and the CUDA path can both be fed from it.

Five workload shapes stand in for the ones the pages describe (no dataset is
used anywhere):

* ``tiny``       -- N=1024 slots, 8 chunks; small enough for brute force.
* ``library``    -- the usage example of the ``fast-weight-product-key-memory``
                    package page (Usage: dim 512, 256*256 memories, topk 8,
                    learning rate 1, chunk 256), at T=4096 with B=2 and the
                    memory chained over 3 consecutive calls.
* ``multihead``  -- 4 query heads sharing one memory, bf16 queries/targets,
                    marginal-entropy term on (gist.science, section 2 "Core
                    Architecture", addressing objective).
* ``longctx``    -- 128K tokens into N = 1,048,576 slots with 1% planted
                    recalls (stands in for the 128K Needle-in-a-Haystack
                    shape, gist.science section 4).
* ``iterative``  -- the same sequence read twice with the memory carried over
                    (iterative reading, gist.science section 4).

Draw order (numpy PCG64 ``default_rng(seed)``): sub-keys, values, Q, Vtarget,
gate, plants.  Distribution conventions:

* Q, Vtarget ~ N(0, 1) per element, drawn in float32; bf16 workloads round the
  float32 draw to bfloat16 with round-to-nearest-even.
* sub-keys ~ N(0, variance 1/sqrt(dq/2)), i.e. standard deviation
  (dq/2)**-0.25 (the "N(0, 1/sqrt(32))" of the tiny shape read as mean,
  variance -- the same convention as "N(0, 0.02^2)" for the values).
* values ~ N(0, 0.02^2).
* gate: 1, U(0, 1) or Beta(2, 5) per workload.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np

F32 = 0
BF16 = 1


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    T: int
    chunk: int
    heads: int
    dq: int
    n: int
    dv: int
    topk: int
    eta: float
    lam: float
    gate: str            # "one" | "uniform" | "beta25"
    in_dtype: int = F32  # dtype of Q and Vtarget (tables are always fp32)
    calls: int = 1       # consecutive chained calls over fresh segments
    passes: int = 1      # re-reads of the same sequence with the state carried
    plant_frac: float = 0.0
    seed: int = 0
    eps: float = 1e-3
    lookahead: bool = False  # each call writes query t towards the target of token t+1
    heads_mode: str = "mean"  # head readouts "mean" or "sum"
    agg: str = "weight"       # divisor of a value row's gradient: "weight", "count", "sum"
    score: str = "idw"        # sub-key score: "idw" (-log(eps + |q - K|^2)) or "dot" (q . K)
    per_sequence: bool = False  # one memory per sequence (B memories in one state)

    @property
    def N(self) -> int:
        return self.n * self.n

    @property
    def dh(self) -> int:
        return self.dq // 2

    @property
    def tokens_per_step(self) -> int:
        """Tokens processed by one full pass of the workload (all calls/passes)."""
        return self.B * self.T * self.calls * self.passes

    def n_chunks(self, T: Optional[int] = None) -> int:
        T = self.T if T is None else T
        return -(-T // self.chunk)

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    "tiny": Workload("tiny", B=1, T=256, chunk=32, heads=1, dq=64, n=32, dv=64, topk=4,
                     eta=0.5, lam=0.0, gate="one"),
    "library": Workload("library", B=2, T=4096, chunk=256, heads=1, dq=512, n=256, dv=512,
                        topk=8, eta=1.0, lam=0.0, gate="uniform", calls=3),
    "multihead": Workload("multihead", B=8, T=4096, chunk=512, heads=4, dq=512, n=512,
                          dv=512, topk=16, eta=0.5, lam=0.05, gate="uniform", in_dtype=BF16),
    "longctx": Workload("longctx", B=1, T=131072, chunk=1024, heads=1, dq=512, n=1024,
                        dv=512, topk=32, eta=1.0, lam=0.0, gate="one", plant_frac=0.01),
    "iterative": Workload("iterative", B=4, T=8192, chunk=512, heads=2, dq=256, n=512,
                          dv=256, topk=16, eta=0.5, lam=0.1, gate="beta25", passes=2),
}


def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round float32 -> bfloat16 (nearest-even); returns the uint16 bit patterns."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    rounded = (b + 0x7FFF + ((b >> 16) & 1)) >> 16
    return rounded.astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Widen bfloat16 bit patterns to float32 (exact)."""
    return (bits.astype(np.uint32) << 16).view(np.float32)


@dataclasses.dataclass
class Inputs:
    """Host arrays for one workload.

    ``subkeys`` [H][2][n][dq/2] fp32, ``values`` [N][dv] fp32,
    ``Q`` [B][T_total][H*dq] and ``Vt`` [B][T_total][dv] (fp32, or uint16
    bfloat16 bit patterns when ``in_dtype`` is BF16), ``gate`` [B][T_total]
    fp32.  ``T_total`` = calls * T: call c reads the segment
    [c*T, (c+1)*T).  ``plants`` lists (position, source) pairs.
    """
    wl: Workload
    subkeys: np.ndarray
    values: np.ndarray
    Q: np.ndarray
    Vt: np.ndarray
    gate: np.ndarray
    plants: np.ndarray

    def q_f32(self) -> np.ndarray:
        return bf16_bits_to_f32(self.Q) if self.wl.in_dtype == BF16 else self.Q

    def vt_f32(self) -> np.ndarray:
        return bf16_bits_to_f32(self.Vt) if self.wl.in_dtype == BF16 else self.Vt

    def segment(self, call: int):
        """(Q, Vt, gate) of chained call ``call`` (views)."""
        T = self.wl.T
        s = slice(call * T, (call + 1) * T)
        return self.Q[:, s], self.Vt[:, s], self.gate[:, s]


def make_inputs(wl: Workload, seed: Optional[int] = None) -> Inputs:
    rng = np.random.default_rng(wl.seed if seed is None else seed)
    H, n, dh, dv, B = wl.heads, wl.n, wl.dh, wl.dv, wl.B
    T_total = wl.T * wl.calls
    key_std = np.float32(dh ** -0.25)
    subkeys = rng.standard_normal((H, 2, n, dh), dtype=np.float32) * key_std
    values = rng.standard_normal((wl.N, dv), dtype=np.float32) * np.float32(0.02)
    Q = rng.standard_normal((B, T_total, H * wl.dq), dtype=np.float32)
    Vt = rng.standard_normal((B, T_total, dv), dtype=np.float32)
    if wl.gate == "one":
        gate = np.ones((B, T_total), dtype=np.float32)
    elif wl.gate == "uniform":
        gate = rng.random((B, T_total), dtype=np.float32)
    elif wl.gate == "beta25":
        gate = rng.beta(2.0, 5.0, size=(B, T_total)).astype(np.float32)
    else:
        raise ValueError(f"unknown gate distribution {wl.gate!r}")
    plants = np.zeros((0, 2), dtype=np.int64)
    if wl.plant_frac > 0.0:
        n_plant = int(wl.plant_frac * T_total)
        pos = np.sort(rng.choice(np.arange(1, T_total), size=n_plant, replace=False))
        src = np.empty_like(pos)
        for idx, p in enumerate(pos):
            src[idx] = rng.integers(0, p)
            Q[:, p] = Q[:, src[idx]]
            Vt[:, p] = Vt[:, src[idx]]
        plants = np.stack([pos, src], axis=1)
    if wl.in_dtype == BF16:
        Q = round_to_bf16(Q)
        Vt = round_to_bf16(Vt)
    return Inputs(wl, np.ascontiguousarray(subkeys), np.ascontiguousarray(values),
                  np.ascontiguousarray(Q), np.ascontiguousarray(Vt),
                  np.ascontiguousarray(gate), plants)
