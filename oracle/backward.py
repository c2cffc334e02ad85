"""Float64 oracle of the memory layer's gradients (test infrastructure only).

The write-and-read of "Titans, explained" steps 2-6 ("Attack of the Titans",
"Parallel training": gradients at the chunk-start weights) restated token by
token in plain PyTorch float64 CPU ops, with the surprise gradient written
out (forward, residual 2(M(k) - v), backward through SiLU), so that
torch.autograd can differentiate the whole recurrence, including through the
surprise itself. Given upstream gradients dy (of the reads y), dW_end, dS_end,
it returns the gradients of the objective
    J = sum_t <dy_t, y_t> + <dW_end, W_end> + <dS_end, S_end>
with respect to k, v, q, the gates theta, eta, alpha, and W0, S0.
Small inputs only (a Python loop over tokens). Only tests/ use it; it is
pinned against the C oracle's forward and against finite differences of J
evaluated with the C oracle.
"""
from __future__ import annotations

import numpy as np
import torch


def _silu(z):
    return z * torch.sigmoid(z)


def _silu_prime(z):
    s = torch.sigmoid(z)
    return s * (1 + z * (1 - s))


def _layers(flat, dims):
    out, o = [], 0
    for l in range(1, len(dims)):
        n = dims[l] * dims[l - 1]
        out.append(flat[o:o + n].reshape(dims[l], dims[l - 1]))
        o += n
    return out


def _forward(Ws, x):
    """Returns pre-activations z_l and activations x_l (x_0 = x)."""
    xs, zs = [x], []
    for l, W in enumerate(Ws):
        z = W @ xs[-1]
        zs.append(z)
        xs.append(z if l == len(Ws) - 1 else _silu(z))
    return zs, xs


def _surprise(Ws, k, v):
    """u_l = d||M(k) - v||^2 / dW_l, written out (no autograd inside)."""
    zs, xs = _forward(Ws, k)
    g = 2 * (xs[-1] - v)
    us = [None] * len(Ws)
    for l in range(len(Ws) - 1, -1, -1):
        us[l] = torch.outer(g, xs[l])
        if l > 0:
            g = (Ws[l].T @ g) * _silu_prime(zs[l - 1])
    return us


def recurrence(dims, C, k, v, q, theta, eta, alpha, W0, S0):
    """One stream, float64 torch tensors: k, q [T, d], v [T, d_out], gates [T],
    W0, S0 [P]. Returns y [T, d_out], W_end, S_end [P]."""
    T = k.shape[0]
    W = _layers(W0, dims)
    S = _layers(S0, dims)
    ys = []
    for t in range(T):
        if t % C == 0:
            Wf = [w for w in W]            # chunk-start weights (reads and surprise)
        u = _surprise(Wf, k[t], v[t])
        S = [eta[t] * s - theta[t] * ul for s, ul in zip(S, u)]
        W = [(1 - alpha[t]) * w + s for w, s in zip(W, S)]
        ys.append(_forward(Wf, q[t])[1][-1])
    flat = lambda ms: torch.cat([m.reshape(-1) for m in ms])
    return torch.stack(ys), flat(W), flat(S)


def backward(dims, C, k, v, q, theta, eta, alpha, W0, S0, dy, dW_end, dS_end):
    """One stream, numpy float64 in and out. Returns the gradients of J."""
    names = ["k", "v", "q", "theta", "eta", "alpha", "W0", "S0"]
    vals = [k, v, q, theta, eta, alpha, W0, S0]
    ts = {n: torch.tensor(np.asarray(a, dtype=np.float64), requires_grad=True) for n, a in zip(names, vals)}
    y, We, Se = recurrence(dims, C, *(ts[n] for n in names))
    J = (y * torch.as_tensor(dy, dtype=torch.float64)).sum() + \
        (We * torch.as_tensor(dW_end, dtype=torch.float64)).sum() + \
        (Se * torch.as_tensor(dS_end, dtype=torch.float64)).sum()
    grads = torch.autograd.grad(J, [ts[n] for n in names])
    return {"d" + n: g.detach().numpy() for n, g in zip(names, grads)}
