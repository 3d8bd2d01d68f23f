"""The seeded input generators shared by the oracle and the GPU path.

They hold no method arithmetic, but both sides read their output, so they are
pinned here against independent references: PyTorch's bfloat16 conversion,
the seed contract, the planted-recall recipe and the stated distributions.
"""
import numpy as np
import pytest

from sparse_weight_memory_b200.workloads import (WORKLOADS, bf16_bits_to_f32, make_inputs,
                                                 round_to_bf16)


def test_bf16_rounding_matches_torch():
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(3)
    x = np.concatenate([
        rng.standard_normal(100_000).astype(np.float32),
        (rng.standard_normal(10_000) * 1e-38).astype(np.float32),  # subnormals
        np.array([0.0, -0.0, 1.0, -1.0, 65504.0, 3.3895314e38, np.inf, -np.inf], np.float32),
        # exact ties between two bfloat16 neighbours (round half to even)
        np.array([1.00390625, 1.01171875, -1.00390625], np.float32),
    ])
    ours = round_to_bf16(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
    # and the widening back is exact
    assert np.array_equal(bf16_bits_to_f32(ours),
                          torch.from_numpy(x).to(torch.bfloat16).float().numpy())


def test_inputs_are_a_function_of_the_seed():
    wl = WORKLOADS["tiny"]
    a, b = make_inputs(wl), make_inputs(wl)
    for name in ("subkeys", "values", "Q", "Vt", "gate"):
        assert np.array_equal(getattr(a, name), getattr(b, name))
    c = make_inputs(wl, seed=wl.seed + 1)
    assert not np.array_equal(a.Q, c.Q)


def test_planted_recalls_repeat_an_earlier_pair():
    wl = WORKLOADS["longctx"].replace(T=8192)
    inp = make_inputs(wl)
    pos, src = inp.plants[:, 0], inp.plants[:, 1]
    assert len(pos) == int(wl.plant_frac * wl.T)
    assert np.all(np.diff(pos) > 0) and np.all(src < pos) and np.all(pos >= 1)
    assert np.array_equal(inp.Q[:, pos], inp.Q[:, src])
    assert np.array_equal(inp.Vt[:, pos], inp.Vt[:, src])


def test_stated_distributions():
    wl = WORKLOADS["library"]
    inp = make_inputs(wl)
    # sub-keys: variance 1/sqrt(dq/2), i.e. std (dq/2)^(-1/4); values: std 0.02
    assert abs(inp.subkeys.std() / (wl.dh ** -0.25) - 1) < 0.02
    assert abs(inp.values.std() / 0.02 - 1) < 0.01
    assert abs(inp.Q.std() - 1) < 0.01 and abs(inp.Q.mean()) < 0.01
    assert inp.gate.min() >= 0 and inp.gate.max() <= 1 and abs(inp.gate.mean() - 0.5) < 0.01
