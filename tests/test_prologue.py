"""The step before the memory: depthwise causal convolution of k, v, q and
L2 normalisation of keys and queries ("Titans, explained", step 1)."""
import numpy as np
import pytest
import torch

from gen import workloads as W
from oracle import prologue as P


def test_conv_matches_numpy_convolve():
    rng = np.random.default_rng(1)
    T, d, w = 37, 5, 4
    x, f = rng.standard_normal((T, d)), rng.standard_normal((d, w))
    out = P.conv_causal(x, f)
    for c in range(d):
        np.testing.assert_allclose(out[:, c], np.convolve(x[:, c], f[c])[:T], rtol=1e-13, atol=1e-13)


def test_delta_and_shift_filters():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((9, 3))
    f = np.zeros((3, 4))
    f[:, 0] = 1.0
    np.testing.assert_array_equal(P.conv_causal(x, f), x)
    f = np.zeros((3, 4))
    f[:, 1] = 1.0
    out = P.conv_causal(x, f)
    np.testing.assert_array_equal(out[1:], x[:-1])
    assert not out[0].any()


def test_history_equals_one_long_sequence():
    rng = np.random.default_rng(3)
    x, f = rng.standard_normal((20, 4)), rng.standard_normal((4, 3))
    full = P.conv_causal(x, f)
    tail = P.conv_causal(x[12:], f, history=x[12 - 2:12])
    np.testing.assert_allclose(tail, full[12:], rtol=1e-13, atol=1e-13)


def test_normalisation():
    rng = np.random.default_rng(4)
    x = rng.standard_normal((6, 8))
    x[2] = 0.0
    n = P.l2_normalise_rows(x)
    assert not n[2].any()
    np.testing.assert_allclose(np.linalg.norm(np.delete(n, 2, axis=0), axis=1), 1.0, rtol=1e-14)


def test_prologue_normalises_keys_and_queries_only():
    """With identity filters (tap 0 = 1) the step reduces to row normalisation
    of k and q (checked with numpy's norm) and leaves v exactly as it was."""
    rng = np.random.default_rng(6)
    k, v, q = (rng.standard_normal((7, 5)) for _ in range(3))
    f = np.zeros((5, 3))
    f[:, 0] = 1.0
    kk, vv, qq = P.prologue(k, v, q, f, f, f)
    np.testing.assert_allclose(kk, k / np.linalg.norm(k, axis=1, keepdims=True), rtol=1e-14)
    np.testing.assert_allclose(qq, q / np.linalg.norm(q, axis=1, keepdims=True), rtol=1e-14)
    np.testing.assert_array_equal(vv, v)


def _rand(shape, rng, dtype):
    x = rng.standard_normal(shape).astype(np.float32)
    if dtype == "bf16":
        return W.f32_to_bf16_bits(x)
    return x


def _to_t(a, dtype):
    a = np.ascontiguousarray(a)
    if dtype == "bf16":
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(a).cuda()


def _f64(a, dtype):
    return W.tokens_as_f64(a, dtype)


@pytest.mark.gpu
@pytest.mark.parametrize("B,H,T,d,width,dtype,hist", [
    (1, 2, 100, 64, 4, "bf16", False),      # ragged last tile
    (2, 1, 64, 128, 4, "bf16", True),
    (1, 1, 130, 384, 3, "bf16", True),
    (1, 3, 65, 32, 1, "f32", False),        # width 1: normalisation only
    (2, 2, 200, 256, 8, "f32", True),       # norm reduced across two warps
    (1, 1, 70, 768, 5, "bf16", True),       # widest row: six warps per row
    (3, 1, 9, 128, 2, "f32", True),         # sequence shorter than one tile
    (1, 2, 100, 128, 6, "bf16", True),      # filter wider than 4 taps, rows inside one warp
    (2, 8, 65600, 128, 4, "bf16", True),    # >= 2^20 rows: 16 output rows per row group, ragged end
    (1, 2, 524300, 32, 4, "bf16", False),   # the same form with 8-lane row groups
])
def test_prologue_matches_oracle(B, H, T, d, width, dtype, hist):
    from test_trained_neural_b200 import prologue
    rng = np.random.default_rng(B * 100 + T + d)
    xs = [_rand((B, H, T, d), rng, dtype) for _ in range(3)]
    fs = [rng.standard_normal((H, d, width)).astype(np.float32) * 0.5 for _ in range(3)]
    hs = [_rand((B, H, width - 1, d), rng, dtype) for _ in range(3)] if hist and width > 1 else None
    dev_x = [_to_t(x, dtype) for x in xs]
    dev_f = [torch.from_numpy(f).cuda() for f in fs]
    dev_h = [_to_t(h, dtype) for h in hs] if hs else None
    out = prologue(*dev_x, *dev_f, hist=dev_h)
    torch.cuda.synchronize()
    tol = 1e-2 if dtype == "bf16" else 1e-5
    for b in range(B):
        for h in range(H):
            hist_args = [None] * 3 if hs is None else [_f64(hs[i][b, h], dtype) for i in range(3)]
            ref = P.prologue(*[_f64(xs[i][b, h], dtype) for i in range(3)],
                             *[fs[i][h].astype(np.float64) for i in range(3)], *hist_args)
            for i in range(3):
                got = out[i][b, h].double().cpu().numpy()
                err = np.linalg.norm(got - ref[i]) / np.linalg.norm(ref[i])
                assert err < tol, (b, h, i, err)


@pytest.mark.gpu
def test_prologue_feeds_the_memory():
    """Raw projections -> prologue -> tensor-core write-and-read, end to end."""
    import oracle
    from test_trained_neural_b200 import NeuralMemory, prologue
    from gpu_util import gpu_to_np, parity_errors, run_lib
    w = W.make(2, 64, 2, 1, 2, 128, 64, index=700)
    inp = W.generate(w)
    rng = np.random.default_rng(7)
    fs = [rng.standard_normal((w.H, w.d, 4)).astype(np.float32) * 0.5 for _ in range(3)]
    dev = {key: _to_t(inp[key].reshape(w.B, w.H, w.T, w.d), "bf16") for key in ("k", "v", "q")}
    kp, vp, qp = prologue(dev["k"], dev["v"], dev["q"], *[torch.from_numpy(f).cuda() for f in fs])
    for key in ("theta", "eta", "alpha", "W0", "S0"):
        dev[key] = torch.from_numpy(np.ascontiguousarray(inp[key])).reshape(w.B, w.H, *inp[key].shape[1:]).cuda()
    dev["k"], dev["v"], dev["q"] = kp, vp, qp
    mem = NeuralMemory(w.L, w.d, w.expansion)
    y, We, Se = run_lib(mem, dev, w.C)
    # the oracle consumes the prologue's bf16 outputs exactly as stored
    sub = dict(inp)
    for key, t in (("k", kp), ("v", vp), ("q", qp)):
        sub[key] = t.view(torch.int16).cpu().numpy().view(np.uint16).reshape(w.streams, w.T, w.d)
    ref = oracle.run_workload(w, sub)
    errs = parity_errors(w.dims, inp["W0"], gpu_to_np(y, We, Se), ref)
    assert max(errs.values()) < 2e-2, errs
