"""Pins for the float64 oracle: each check ties it to something other than itself.

Sources of truth used here:
  * torch autograd (a library gradient, independent of the oracle's hand-written
    backward) for the surprise u_t = grad ||M(k) - v||^2;
  * central finite differences of the loss;
  * closed forms the pages state ("Titans, explained": the "At the extremes"
    paragraph and "Where it sits among test-time learners": alpha = 1 wipes,
    theta = 0 writes nothing, eta = alpha = 0 with a linear memory is the
    DeltaNet delta rule with gradient 2 (M k - v) k^T);
  * exact rational arithmetic on tiny inputs;
  * invariants (state carry, stream independence, alpha = 0 sums momenta).
"""
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle


def rand_problem(rng, dims, n, T, theta=(0.01, 0.3), eta=(0.5, 0.99), alpha=(0.0, 0.2), s0=True):
    L = len(dims) - 1
    P = sum(dims[i] * dims[i + 1] for i in range(L))
    k = rng.standard_normal((n, T, dims[0]))
    q = rng.standard_normal((n, T, dims[0]))
    v = rng.standard_normal((n, T, dims[-1]))
    th = rng.uniform(*theta, (n, T))
    et = rng.uniform(*eta, (n, T))
    al = rng.uniform(*alpha, (n, T))
    W0 = 0.5 * rng.standard_normal((n, P))
    S0 = 0.1 * rng.standard_normal((n, P)) if s0 else np.zeros((n, P))
    return dict(k=k, v=v, q=q, theta=th, eta=et, alpha=al, W0=W0, S0=S0)


def orun(dims, C, p, **kw):
    return oracle.run(dims, C, p["k"], p["v"], p["q"], p["theta"], p["eta"], p["alpha"],
                      p["W0"], p["S0"], **kw)


def split_layers(flat, dims):
    out, off = [], 0
    for i in range(len(dims) - 1):
        n = dims[i + 1] * dims[i]
        out.append(flat[off:off + n].reshape(dims[i + 1], dims[i]))
        off += n
    return out


def torch_forward(Ws, x):
    for i, W in enumerate(Ws):
        x = W @ x
        if i < len(Ws) - 1:
            x = torch.nn.functional.silu(x)
    return x


def torch_grad(Ws_np, k, v):
    """Library gradient of ||M(k) - v||^2 (sum of squares) at Ws."""
    Ws = [torch.tensor(W, dtype=torch.float64, requires_grad=True) for W in Ws_np]
    out = torch_forward(Ws, torch.tensor(k, dtype=torch.float64))
    loss = ((out - torch.tensor(v, dtype=torch.float64)) ** 2).sum()
    loss.backward()
    return [W.grad.numpy() for W in Ws]


def autograd_recurrence(dims, C, p, s):
    """Independent restatement of the chunked write-and-read with torch autograd:
    gradients of all tokens of a chunk at the chunk-start weights, then the
    momentum and forget-then-write steps token by token, reads through the
    chunk-start weights."""
    W = split_layers(p["W0"][s].copy(), dims)
    S = split_layers(p["S0"][s].copy(), dims)
    T = p["k"].shape[1]
    ys = []
    for t in range(T):
        if t % C == 0:
            Wf = [w.copy() for w in W]
        u = torch_grad(Wf, p["k"][s, t], p["v"][s, t])
        for l in range(len(W)):
            S[l] = p["eta"][s, t] * S[l] - p["theta"][s, t] * u[l]
            W[l] = (1.0 - p["alpha"][s, t]) * W[l] + S[l]
        with torch.no_grad():
            ys.append(torch_forward([torch.tensor(w) for w in Wf],
                                    torch.tensor(p["q"][s, t])).numpy())
    flat = lambda ms: np.concatenate([m.ravel() for m in ms])
    return np.stack(ys), flat(W), flat(S)


# ---------------------------------------------------------------- gradient pins

@pytest.mark.parametrize("dims", [[4, 4], [5, 7, 4], [3, 6, 5, 4], [3, 5, 6, 4, 3], [6, 9, 2]])
def test_surprise_matches_autograd(dims):
    rng = np.random.default_rng(len(dims) * 10 + dims[0])
    P = sum(dims[i] * dims[i + 1] for i in range(len(dims) - 1))
    W = rng.standard_normal(P)
    k, v = rng.standard_normal(dims[0]), rng.standard_normal(dims[-1])
    u = oracle.surprise(dims, W, k, v)
    ref = np.concatenate([g.ravel() for g in torch_grad(split_layers(W, dims), k, v)])
    np.testing.assert_allclose(u, ref, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("dims", [[3, 3], [3, 5, 2], [2, 4, 3, 2], [3, 4, 5, 4, 3]])
def test_surprise_matches_finite_differences(dims):
    """P5: central differences of the loss, h = 1e-6."""
    rng = np.random.default_rng(7 + len(dims))
    P = sum(dims[i] * dims[i + 1] for i in range(len(dims) - 1))
    W = rng.standard_normal(P)
    k, v = rng.standard_normal(dims[0]), rng.standard_normal(dims[-1])

    def loss(Wflat):
        x = k
        Ws = split_layers(Wflat, dims)
        for i, M in enumerate(Ws):
            x = M @ x
            if i < len(Ws) - 1:
                x = x / (1.0 + np.exp(-x))
        return float(((x - v) ** 2).sum())

    u = oracle.surprise(dims, W, k, v)
    h = 1e-6
    fd = np.empty(P)
    for i in range(P):
        e = np.zeros(P)
        e[i] = h
        fd[i] = (loss(W + e) - loss(W - e)) / (2 * h)
    err = np.linalg.norm(u - fd) / np.linalg.norm(fd)
    assert err < 1e-7, err


def test_linear_gradient_closed_form():
    """'At the extremes': for a linear memory the gradient is 2 (M k - v) k^T."""
    rng = np.random.default_rng(3)
    d = 6
    W = rng.standard_normal((d, d))
    k, v = rng.standard_normal(d), rng.standard_normal(d)
    u = oracle.surprise([d, d], W.ravel(), k, v).reshape(d, d)
    np.testing.assert_allclose(u, 2.0 * np.outer(W @ k - v, k), rtol=1e-13, atol=1e-13)


# ------------------------------------------------------------- recurrence pins

def test_single_token_linear_no_momentum():
    """P1: linear memory, eta = 0, one token: W' = (1-alpha) W - 2 theta (W k - v) k^T,
    S' = -2 theta (W k - v) k^T, and the read uses the old W."""
    rng = np.random.default_rng(11)
    d = 5
    p = rand_problem(rng, [d, d], 1, 1)
    p["eta"][:] = 0.0
    r = orun([d, d], 4, p)
    W0 = p["W0"][0].reshape(d, d)
    k, v, q = p["k"][0, 0], p["v"][0, 0], p["q"][0, 0]
    th, al = p["theta"][0, 0], p["alpha"][0, 0]
    g = 2.0 * np.outer(W0 @ k - v, k)
    np.testing.assert_allclose(r["W_end"][0].reshape(d, d), (1 - al) * W0 - th * g, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(r["S_end"][0].reshape(d, d), -th * g, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(r["y"][0, 0], W0 @ q, rtol=1e-13, atol=1e-14)


@pytest.mark.parametrize("dims", [[4, 4], [3, 5, 3], [3, 4, 5, 3], [2, 3, 4, 3, 2]])
def test_chunk_size_one_is_online_descent_with_momentum(dims):
    """P2: with C = 1 every token is a plain online gradient step with momentum.
    The reference loop below takes gradients with torch autograd at the current
    weights (no chunk-start copy at all)."""
    rng = np.random.default_rng(sum(dims))
    p = rand_problem(rng, dims, 1, 9)
    r = orun(dims, 1, p)
    W = split_layers(p["W0"][0].copy(), dims)
    S = split_layers(p["S0"][0].copy(), dims)
    for t in range(9):
        with torch.no_grad():
            y = torch_forward([torch.tensor(w) for w in W], torch.tensor(p["q"][0, t])).numpy()
        np.testing.assert_allclose(r["y"][0, t], y, rtol=1e-11, atol=1e-12)
        u = torch_grad(W, p["k"][0, t], p["v"][0, t])
        for l in range(len(W)):
            S[l] = p["eta"][0, t] * S[l] - p["theta"][0, t] * u[l]
            W[l] = (1 - p["alpha"][0, t]) * W[l] + S[l]
    np.testing.assert_allclose(r["W_end"][0], np.concatenate([w.ravel() for w in W]), rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(r["S_end"][0], np.concatenate([s.ravel() for s in S]), rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("dims,C,T", [([4, 4], 3, 10), ([3, 6, 3], 4, 12), ([3, 5, 4, 3], 5, 13),
                                      ([2, 4, 4, 4, 2], 2, 7), ([3, 7, 3], 16, 9)])
def test_chunked_recurrence_matches_autograd_restatement(dims, C, T):
    """Gradients at the chunk-start weights; a partial last chunk when C does not
    divide T ('Attack of the Titans', 'Parallel training': t' = t - (t mod b))."""
    rng = np.random.default_rng(C * 100 + T)
    p = rand_problem(rng, dims, 2, T)
    r = orun(dims, C, p)
    for s in range(2):
        y, We, Se = autograd_recurrence(dims, C, p, s)
        np.testing.assert_allclose(r["y"][s], y, rtol=1e-11, atol=1e-12)
        np.testing.assert_allclose(r["W_end"][s], We, rtol=1e-11, atol=1e-12)
        np.testing.assert_allclose(r["S_end"][s], Se, rtol=1e-11, atol=1e-12)


def test_reads_see_no_write_of_their_own_chunk():
    """Reads inside chunk c use the weights at the end of chunk c-1: changing the
    keys/values of chunk c leaves chunk c's reads untouched."""
    rng = np.random.default_rng(5)
    dims, C = [3, 5, 3], 4
    p = rand_problem(rng, dims, 1, 12)
    a = orun(dims, C, p)
    p2 = {k: v.copy() for k, v in p.items()}
    p2["k"][0, 4:8] += 1.0
    p2["v"][0, 4:8] -= 2.0
    b = orun(dims, C, p2)
    np.testing.assert_array_equal(a["y"][0, :8], b["y"][0, :8])
    assert np.abs(a["y"][0, 8:] - b["y"][0, 8:]).max() > 1e-6


def test_theta_zero_writes_nothing():
    """P3: theta = 0 turns writing off. S_T = prod(eta) S_0 and
    W_T = prod(1-alpha) W_0 + sum_tau prod_{j>tau}(1-alpha_j) prod_{j<=tau} eta_j S_0,
    whatever the keys and values."""
    rng = np.random.default_rng(21)
    dims, C, T = [3, 5, 3], 4, 11
    p = rand_problem(rng, dims, 1, T)
    p["theta"][:] = 0.0
    r = orun(dims, C, p)
    et, al = p["eta"][0], p["alpha"][0]
    A = np.prod(et)
    coefS = sum(np.prod(1 - al[tau + 1:]) * np.prod(et[:tau + 1]) for tau in range(T))
    np.testing.assert_allclose(r["S_end"][0], A * p["S0"][0], rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(r["W_end"][0], np.prod(1 - al) * p["W0"][0] + coefS * p["S0"][0],
                               rtol=1e-12, atol=1e-15)
    p2 = {k: v.copy() for k, v in p.items()}
    p2["k"] = rng.standard_normal(p["k"].shape)
    p2["v"] = rng.standard_normal(p["v"].shape)
    r2 = orun(dims, C, p2)
    np.testing.assert_array_equal(r["W_end"], r2["W_end"])
    np.testing.assert_array_equal(r["S_end"], r2["S_end"])


def test_alpha_one_wipes_memory():
    """P4: alpha = 1 wipes the memory: W_t = S_t exactly; with theta = 0 and
    S_0 = 0 nothing is left at all."""
    rng = np.random.default_rng(23)
    dims = [3, 4, 3]
    p = rand_problem(rng, dims, 2, 10)
    p["alpha"][:] = 1.0
    r = orun(dims, 4, p)
    np.testing.assert_array_equal(r["W_end"], r["S_end"])
    p["theta"][:] = 0.0
    p["S0"][:] = 0.0
    r = orun(dims, 4, p)
    assert not r["W_end"].any() and not r["S_end"].any()


def test_eta_alpha_zero_linear_is_delta_rule():
    """P6: linear memory with eta = alpha = 0 is the DeltaNet delta rule.
    Token by token (C = 1): W <- W - 2 theta (W k - v) k^T.  One chunk of C
    tokens: W_C = W_0 - 2 (W_0 K^T - V^T) diag(theta) K (numpy matmuls)."""
    rng = np.random.default_rng(29)
    d, T = 4, 6
    p = rand_problem(rng, [d, d], 1, T)
    p["eta"][:] = 0.0
    p["alpha"][:] = 0.0
    r = orun([d, d], 1, p)
    W = p["W0"][0].reshape(d, d).copy()
    for t in range(T):
        k, v, th = p["k"][0, t], p["v"][0, t], p["theta"][0, t]
        W = W - 2 * th * np.outer(W @ k - v, k)
    np.testing.assert_allclose(r["W_end"][0].reshape(d, d), W, rtol=1e-12, atol=1e-13)
    r = orun([d, d], T, p)
    K, V, W0 = p["k"][0], p["v"][0], p["W0"][0].reshape(d, d)
    ref = W0 - 2.0 * (W0 @ K.T - V.T) @ np.diag(p["theta"][0]) @ K
    np.testing.assert_allclose(r["W_end"][0].reshape(d, d), ref, rtol=1e-12, atol=1e-13)


def test_alpha_zero_never_forgets():
    """P7: alpha = 0: W_T - W_0 = sum_t S_t."""
    rng = np.random.default_rng(31)
    dims = [3, 4, 3]
    p = rand_problem(rng, dims, 1, 9)
    p["alpha"][:] = 0.0
    r = orun(dims, 4, p, trace=True)
    np.testing.assert_allclose(r["W_end"][0] - p["W0"][0], r["S"][0].sum(axis=0), rtol=1e-12, atol=1e-13)


def test_chunk_closed_form_coefficients():
    """P8: inside one chunk the two recurrences unroll to
       W_C = B W_0 + c_S S_0 - sum_i c_i u_i,   S_C = A S_0 - sum_i e_i u_i
    with B = prod(1-alpha), A = prod(eta), e_i = theta_i prod_{j>i} eta_j,
    c_i = theta_i r_i, r_C = 1, r_i = prod_{j>i}(1-alpha_j) + eta_{i+1} r_{i+1},
    c_S = eta_1 r_1. This is the division-free form the CUDA path uses; here it
    is applied to the oracle's own materialised u_i at every chunk end."""
    rng = np.random.default_rng(37)
    dims, C, T = [3, 5, 3], 5, 15
    p = rand_problem(rng, dims, 1, T, alpha=(0.0, 0.5))
    p["alpha"][0, 3] = 1.0       # a wipe inside the first chunk
    p["eta"][0, 7] = 0.0          # a momentum reset inside the second
    r = orun(dims, C, p, trace=True)
    W, S = p["W0"][0].copy(), p["S0"][0].copy()
    for c0 in range(0, T, C):
        th, et, al = p["theta"][0, c0:c0 + C], p["eta"][0, c0:c0 + C], p["alpha"][0, c0:c0 + C]
        u = r["u"][0, c0:c0 + C]
        rr = np.zeros(C)
        rr[C - 1] = 1.0
        for i in range(C - 2, -1, -1):
            rr[i] = np.prod(1 - al[i + 1:]) + et[i + 1] * rr[i + 1]
        c = th * rr
        e = np.array([th[i] * np.prod(et[i + 1:]) for i in range(C)])
        Wn = np.prod(1 - al) * W + et[0] * rr[0] * S - np.einsum("i,ip->p", c, u)
        Sn = np.prod(et) * S - np.einsum("i,ip->p", e, u)
        np.testing.assert_allclose(Wn, r["W"][0, c0 + C - 1], rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(Sn, r["S"][0, c0 + C - 1], rtol=1e-12, atol=1e-13)
        W, S = Wn, Sn


def test_state_carry_equals_one_long_call():
    """P9: (W_end, S_end) carried into a second call equals one longer call, when
    the split falls on a chunk boundary ('titans-pytorch' review: mem_state is
    'state you can carry forward')."""
    rng = np.random.default_rng(41)
    dims, C, T, T1 = [3, 6, 3], 4, 20, 8
    p = rand_problem(rng, dims, 2, T)
    full = orun(dims, C, p)
    a = {k: (v[:, :T1] if v.ndim >= 2 and k not in ("W0", "S0") else v) for k, v in p.items()}
    ra = orun(dims, C, a)
    b = {k: (v[:, T1:] if k not in ("W0", "S0") else v) for k, v in p.items()}
    b["W0"], b["S0"] = ra["W_end"], ra["S_end"]
    rb = orun(dims, C, b)
    np.testing.assert_array_equal(np.concatenate([ra["y"], rb["y"]], axis=1), full["y"])
    np.testing.assert_array_equal(rb["W_end"], full["W_end"])
    np.testing.assert_array_equal(rb["S_end"], full["S_end"])


def test_streams_are_independent():
    """P10: a batched call equals per-stream calls; permuting streams permutes
    the outputs (one memory per batch entry and head)."""
    rng = np.random.default_rng(43)
    dims, C = [3, 4, 3], 3
    p = rand_problem(rng, dims, 4, 9)
    full = orun(dims, C, p, threads=3)
    perm = np.array([2, 0, 3, 1])
    pp = {k: v[perm] for k, v in p.items()}
    rp = orun(dims, C, pp, threads=1)
    for key in ("y", "W_end", "S_end"):
        np.testing.assert_array_equal(rp[key], full[key][perm])
    one = orun(dims, C, {k: v[2:3] for k, v in p.items()})
    np.testing.assert_array_equal(one["W_end"][0], full["W_end"][2])


def test_brute_force_rational_tiny():
    """P11: d = 2, T = 4, C = 2, linear memory, dyadic inputs. The recurrence is
    expanded by hand in exact rational arithmetic; float64 must agree to
    rounding."""
    F = Fraction
    k = [[F(1, 2), F(-1, 4)], [F(3, 4), F(1, 2)], [F(-1, 2), F(1, 8)], [F(1, 4), F(1, 4)]]
    v = [[F(1), F(-1, 2)], [F(0), F(1, 4)], [F(1, 2), F(1, 2)], [F(-1, 4), F(3, 4)]]
    q = [[F(1, 8), F(1, 2)], [F(-1, 4), F(1)], [F(1, 2), F(0)], [F(3, 8), F(-1, 8)]]
    th = [F(1, 4), F(1, 8), F(1, 2), F(1, 16)]
    et = [F(1, 2), F(3, 4), F(1, 4), F(7, 8)]
    al = [F(1, 8), F(0), F(1, 4), F(1, 2)]
    W = [[F(1, 2), F(1, 4)], [F(-1, 8), F(3, 4)]]
    S = [[F(1, 16), F(0)], [F(0), F(-1, 16)]]
    ys = []
    for t in range(4):
        if t % 2 == 0:
            Wf = [row[:] for row in W]
        mk = [Wf[i][0] * k[t][0] + Wf[i][1] * k[t][1] for i in range(2)]
        u = [[2 * (mk[i] - v[t][i]) * k[t][j] for j in range(2)] for i in range(2)]
        S = [[et[t] * S[i][j] - th[t] * u[i][j] for j in range(2)] for i in range(2)]
        W = [[(1 - al[t]) * W[i][j] + S[i][j] for j in range(2)] for i in range(2)]
        ys.append([Wf[i][0] * q[t][0] + Wf[i][1] * q[t][1] for i in range(2)])
    f = lambda a: np.array(a, dtype=np.float64)
    p = dict(k=f(k)[None], v=f(v)[None], q=f(q)[None], theta=f(th)[None], eta=f(et)[None],
             alpha=f(al)[None], W0=f(sum(([F(1, 2), F(1, 4)], [F(-1, 8), F(3, 4)]), []))[None],
             S0=f([F(1, 16), F(0), F(0), F(-1, 16)])[None])
    r = orun([2, 2], 2, p)
    np.testing.assert_allclose(r["y"][0], f(ys), rtol=1e-14, atol=1e-15)
    np.testing.assert_allclose(r["W_end"][0], f(sum(W, [])), rtol=1e-14, atol=1e-15)
    np.testing.assert_allclose(r["S_end"][0], f(sum(S, [])), rtol=1e-14, atol=1e-15)


def test_input_dtypes_upcast_exactly():
    """float32 and bfloat16-bit inputs are read as the exact float64 value of the
    stored number (bf16 path: the oracle consumes the rounded inputs)."""
    from gen import workloads as W
    rng = np.random.default_rng(47)
    dims, C = [4, 6, 4], 2
    p = rand_problem(rng, dims, 1, 6)
    p32 = {k: v.astype(np.float32) for k, v in p.items()}
    pbf = dict(p32)
    for key in ("k", "v", "q"):
        pbf[key] = W.f32_to_bf16_bits(p32[key])
    r32 = orun(dims, C, p32)
    r64 = orun(dims, C, {k: v.astype(np.float64) for k, v in p32.items()})
    np.testing.assert_array_equal(r32["W_end"], r64["W_end"])
    rbf = orun(dims, C, pbf)
    pbf64 = dict({k: v.astype(np.float64) for k, v in p32.items()})
    for key in ("k", "v", "q"):
        pbf64[key] = W.bf16_bits_to_f64(pbf[key])
    np.testing.assert_array_equal(rbf["y"], orun(dims, C, pbf64)["y"])
