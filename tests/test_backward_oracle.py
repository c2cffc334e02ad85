"""Pins of the gradient oracle (oracle/backward.py), on the CPU: its forward
equals the C oracle's, and its gradients equal central finite differences of
J = sum <dy, y> + <dW_end, W_end> + <dS_end, S_end> evaluated with the C
oracle (an independent implementation of the recurrence)."""
import numpy as np
import pytest
import torch

import oracle
from oracle import backward as BW

CASES = [  # dims, T, C
    ([3, 3], 5, 2),          # linear memory, partial last chunk
    ([2, 3, 2], 4, 2),       # depth 2
    ([2, 2, 2, 2], 3, 3),    # depth 3, one chunk
    ([2, 3, 2, 3, 2], 5, 2),  # depth 4, two full chunks and a shorter last one
]


def _draw(dims, T, seed):
    rng = np.random.default_rng(seed)
    d, do = dims[0], dims[-1]
    P = sum(dims[l] * dims[l - 1] for l in range(1, len(dims)))
    k = rng.standard_normal((T, d))
    k /= np.linalg.norm(k, axis=1, keepdims=True)
    q = rng.standard_normal((T, d))
    v = rng.standard_normal((T, do))
    theta = rng.uniform(0.05, 0.2, T)
    eta = rng.uniform(0.5, 0.95, T)
    alpha = rng.uniform(0.0, 0.2, T)
    W0 = 0.5 * rng.standard_normal(P)
    S0 = 0.1 * rng.standard_normal(P)
    dy = rng.standard_normal((T, do))
    dW = rng.standard_normal(P)
    dS = rng.standard_normal(P)
    return dict(k=k, v=v, q=q, theta=theta, eta=eta, alpha=alpha, W0=W0, S0=S0), (dy, dW, dS)


def _J(dims, C, inp, up):
    out = oracle.run(dims, C, inp["k"][None], inp["v"][None], inp["q"][None], inp["theta"][None],
                     inp["eta"][None], inp["alpha"][None], inp["W0"][None], inp["S0"][None], threads=1)
    dy, dW, dS = up
    return float((out["y"][0] * dy).sum() + (out["W_end"][0] * dW).sum() + (out["S_end"][0] * dS).sum())


@pytest.mark.parametrize("case", CASES, ids=lambda c: "dims%s-T%d-C%d" % (c[0], c[1], c[2]))
def test_forward_restatement_equals_c_oracle(case):
    dims, T, C = case
    inp, _ = _draw(dims, T, 11)
    ref = oracle.run(dims, C, *(inp[n][None] for n in ("k", "v", "q", "theta", "eta", "alpha", "W0", "S0")),
                     threads=1)
    with torch.no_grad():
        y, We, Se = BW.recurrence(dims, C, *(torch.tensor(inp[n]) for n in
                                             ("k", "v", "q", "theta", "eta", "alpha", "W0", "S0")))
    np.testing.assert_allclose(y.numpy(), ref["y"][0], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(We.numpy(), ref["W_end"][0], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(Se.numpy(), ref["S_end"][0], rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("case", CASES, ids=lambda c: "dims%s-T%d-C%d" % (c[0], c[1], c[2]))
def test_gradients_equal_finite_differences_of_c_oracle(case):
    dims, T, C = case
    inp, up = _draw(dims, T, 12)
    g = BW.backward(dims, C, *(inp[n] for n in ("k", "v", "q", "theta", "eta", "alpha", "W0", "S0")), *up)
    h = 1e-6
    for name in ("k", "v", "q", "theta", "eta", "alpha", "W0", "S0"):
        a = inp[name]
        fd = np.zeros_like(a)
        for idx in np.ndindex(a.shape):
            old = a[idx]
            a[idx] = old + h
            jp = _J(dims, C, inp, up)
            a[idx] = old - h
            jm = _J(dims, C, inp, up)
            a[idx] = old
            fd[idx] = (jp - jm) / (2 * h)
        got = g["d" + name]
        err = np.linalg.norm(got - fd) / max(np.linalg.norm(fd), 1e-12)
        assert err < 1e-6, (name, err)
