"""The exact worked example in tests/golden/ (linear memory, d = 4, T = 5,
C = 2, rational inputs and outputs; see make_linear_exact.py there for the
rules it follows) against the float64 oracle and against the library's fp32
kernel. The expected values come from exact arithmetic, not from either
implementation."""
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle

HERE = os.path.dirname(os.path.abspath(__file__))
FIXTURE = os.path.join(HERE, "golden", "linear_d4_T5_C2.txt")
D, T, C = 4, 5, 2


def load():
    out = {}
    with open(FIXTURE) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            name, *vals = line.split()
            out[name] = [Fraction(v) for v in vals]
    return out


def as_f64(vals, shape):
    return np.array([float(v) for v in vals], dtype=np.float64).reshape(shape)


def inputs(g):
    return dict(k=as_f64(g["k"], (1, T, D)), v=as_f64(g["v"], (1, T, D)), q=as_f64(g["q"], (1, T, D)),
                theta=as_f64(g["theta"], (1, T)), eta=as_f64(g["eta"], (1, T)),
                alpha=as_f64(g["alpha"], (1, T)), W0=as_f64(g["W0"], (1, D * D)),
                S0=as_f64(g["S0"], (1, D * D)))


def test_fixture_inputs_are_exact_in_float32():
    g = load()
    for name in ("k", "v", "q", "theta", "eta", "alpha", "W0", "S0"):
        for v in g[name]:
            assert Fraction(float(np.float32(float(v)))) == v, (name, v)


def test_oracle_matches_exact_example():
    g = load()
    p = inputs(g)
    r = oracle.run([D, D], C, p["k"], p["v"], p["q"], p["theta"], p["eta"], p["alpha"], p["W0"], p["S0"])
    for name, got in (("y", r["y"][0].reshape(-1)), ("W_end", r["W_end"][0]), ("S_end", r["S_end"][0])):
        want = as_f64(g[name], (-1,))
        np.testing.assert_allclose(got, want, rtol=1e-13, atol=1e-16, err_msg=name)


@pytest.mark.gpu
@pytest.mark.parametrize("path", ["simt", "auto"])
def test_library_matches_exact_example(path):
    """fp32 arithmetic on a handful of terms: within 1e-5 normwise of the exact
    values (float32 resolution is 6e-8 per operation)."""
    from test_trained_neural_b200 import NeuralMemory

    g = load()
    p = inputs(g)
    dev = {k: torch.from_numpy(v.astype(np.float32)).reshape(1, 1, *v.shape[1:]).cuda().contiguous()
           for k, v in p.items()}
    mem = NeuralMemory(1, D, 1, path=path)
    y, We, Se = mem.run(dev["k"], dev["v"], dev["q"], dev["theta"], dev["eta"], dev["alpha"], dev["W0"],
                        dev["S0"], C, sync=True)
    torch.cuda.synchronize()
    for name, got in (("y", y), ("W_end", We), ("S_end", Se)):
        got = got.double().cpu().numpy().reshape(-1)
        want = as_f64(g[name], (-1,))
        assert np.linalg.norm(got - want) / np.linalg.norm(want) < 1e-5, name
