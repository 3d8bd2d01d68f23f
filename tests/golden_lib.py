"""Reader of the hand-worked examples under ``tests/golden/``.

A fixture states its inputs and expected values as exact fractions (strings
such as "-155/256"); this module only parses them into float64 arrays.
"""
from __future__ import annotations

import dataclasses
import math
import os
from fractions import Fraction

import numpy as np
import yaml

GOLDEN_DIR = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def frac(x) -> float:
    return float(Fraction(str(x)))


def arr(x) -> np.ndarray:
    if isinstance(x, list):
        return np.array([arr(v) for v in x])
    return np.float64(frac(x))


def row_key(s: str):
    return tuple(int(v) for v in s.split(","))


def log_sum(terms) -> float:
    """sum of c * log(p) over [c, p] pairs."""
    return sum(frac(c) * math.log(frac(p)) for c, p in terms)


@dataclasses.dataclass
class HandStep:
    raw: dict
    heads: int
    n: int
    dq: int
    dv: int
    topk: int
    chunk: int
    eps: float
    eta: float
    K: np.ndarray        # [H][2][n][dq/2]
    V: np.ndarray        # [N][dv]
    Q: np.ndarray        # [B][T][H*dq]
    Vt: np.ndarray       # [B][T][dv]
    gate: np.ndarray     # [B][T]

    @property
    def expected(self) -> dict:
        return self.raw["expected"]

    def values_after(self) -> np.ndarray:
        V = self.V.copy()
        for r, row in self.expected["values_after"].items():
            V[int(r)] = arr(row)
        return V

    def subkeys_after(self, lam: float = 0.0) -> np.ndarray:
        K = self.K.copy()
        for key, row in self.expected["subkeys_after"].items():
            K[row_key(key)] = arr(row)
        if lam:
            K -= self.eta * lam * self.dLdK_per_lambda()
        return K

    def dLdK(self) -> np.ndarray:
        dK = np.zeros_like(self.K)
        for key, row in self.expected["dLdK"].items():
            dK[row_key(key)] = arr(row)
        return dK

    def dLdK_per_lambda(self) -> np.ndarray:
        d = np.zeros_like(self.K)
        for key, coords in self.raw["entropy"]["dLdK_per_lambda"].items():
            d[row_key(key)] = [log_sum(t) for t in coords]
        return d

    def pbar(self) -> np.ndarray:
        p = np.zeros(self.n * self.n)
        for r, v in self.expected["pbar"].items():
            p[int(r)] = frac(v)
        return p


def load_hand_step(name: str = "hand_step_three_tokens.yaml") -> HandStep:
    with open(os.path.join(GOLDEN_DIR, name)) as fh:
        g = yaml.safe_load(fh)
    sh, inp = g["shape"], g["inputs"]
    n, dv = sh["n"], sh["dv"]
    K = arr(inp["subkeys"])
    assert K.shape == (sh["heads"], 2, n, sh["dq"] // 2)
    # every row that the example does not read holds (r, 1)
    assert dv == 2
    V = np.array([[float(r), 1.0] for r in range(n * n)])
    for r, row in inp["values_read"].items():
        V[int(r)] = arr(row)
    return HandStep(g, sh["heads"], n, sh["dq"], dv, sh["topk"], sh["chunk"], frac(sh["eps"]),
                    frac(g["eta"]), K, V, arr(inp["Q"]), arr(inp["Vtarget"]), arr(inp["gate"]))


def pad_last(a: np.ndarray, width: int) -> np.ndarray:
    """Zero-pad the last axis to ``width`` (zeros change no distance, dot
    product or residual of the example)."""
    out = np.zeros(a.shape[:-1] + (width,), dtype=a.dtype)
    out[..., :a.shape[-1]] = a
    return out


def pad_queries(Q: np.ndarray, H: int, dh: int, dh_to: int) -> np.ndarray:
    """[B][T][H*2*dh] -> [B][T][H*2*dh_to]: each query half zero-padded."""
    B, T, _ = Q.shape
    halves = Q.reshape(B, T, H, 2, dh)
    return pad_last(halves, dh_to).reshape(B, T, H * 2 * dh_to)

