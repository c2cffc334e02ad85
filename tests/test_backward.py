"""Gradients of the memory layer (tm_backward, depths 1 to 4) against the float64
gradient oracle (autograd through the restated recurrence, itself pinned
against finite differences of the C oracle).

Two arithmetic forms: fp32 FFMA throughout (fp32 inputs, or the SIMT path
for bf16 inputs), held to 1e-4; and, for bf16 inputs on the default path,
the chunk's products on tcgen05 with TF32 operands (10 explicit mantissa
bits, rounded to nearest) and fp32 accumulation, held to the 2e-2 bound of
the tensor-core forward."""
import ctypes

import numpy as np
import pytest
import torch

from gen import workloads as W
from oracle import backward as BW
from test_trained_neural_b200 import NeuralMemory
from test_trained_neural_b200 import _native as N

from gpu_util import rel, to_dev

TOL = 1e-4      # fp32 arithmetic against float64
TOL_TC = 2e-2   # TF32 operands on the tensor cores

BACKWARD = [  # L, d, expansion, B, H, T, C, dtype
    (1, 64, 1, 1, 1, 256, 16, "f32"),    # the linear workload's shape
    (1, 32, 1, 2, 1, 40, 8, "bf16"),
    (1, 16, 1, 1, 3, 50, 16, "f32"),     # a shorter last chunk (50 = 3 x 16 + 2)
    (1, 128, 1, 1, 1, 64, 32, "bf16"),
    (2, 16, 4, 1, 2, 48, 16, "f32"),     # depth 2, hidden 64
    (2, 32, 2, 2, 1, 50, 16, "bf16"),    # depth 2, a shorter last chunk
    (2, 64, 4, 1, 1, 64, 64, "bf16"),    # depth 2, the d = 64 workload's memory
    (3, 16, 2, 1, 2, 40, 16, "f32"),     # depth 3, a shorter last chunk (40 = 2 x 16 + 8)
    (4, 16, 2, 2, 1, 48, 16, "f32"),     # depth 4
    (4, 128, 2, 1, 1, 40, 32, "bf16"),   # the deep workload's memory 128-256-256-256-128
]


@pytest.mark.gpu
@pytest.mark.parametrize("path", ["auto", "simt"])
@pytest.mark.parametrize("cfg", BACKWARD, ids=lambda c: "L%d-d%d-e%d-B%dH%d-T%d-C%d-%s" % c)
def test_backward_matches_gradient_oracle(cfg, path):
    L, d, e, B, H, T, C, dt = cfg
    if dt == "f32" and path == "simt":
        pytest.skip("fp32 inputs take the fp32 form on every path")
    w = W.make(L, d, e, B, H, T, C, dtype=dt, index=700 + d + T)
    inp = W.generate(w)
    dev = to_dev(inp, B, H, dt)
    rng = np.random.default_rng(w.seed + 1)
    n = B * H
    dy = rng.standard_normal((n, T, d)).astype(np.float32)
    dWe = rng.standard_normal((n, w.P)).astype(np.float32)
    dSe = rng.standard_normal((n, w.P)).astype(np.float32)
    mem = NeuralMemory(L, d, e, path=path)
    t = lambda a, shape: torch.from_numpy(np.ascontiguousarray(a)).reshape(shape).cuda()
    out = mem.backward(dev["k"], dev["v"], dev["q"], dev["theta"], dev["eta"], dev["alpha"], dev["W0"], dev["S0"],
                       t(dy, (B, H, T, d)), t(dWe, (B, H, w.P)), t(dSe, (B, H, w.P)), C)
    torch.cuda.synchronize()
    kf, vf, qf = (W.tokens_as_f64(inp[x], dt) for x in ("k", "v", "q"))
    worst = {}
    for s in range(n):
        f32 = lambda x: np.asarray(inp[x][s], dtype=np.float32).astype(np.float64)   # as the GPU sees them
        ref = BW.backward(w.dims, C, kf[s], vf[s], qf[s], f32("theta"), f32("eta"), f32("alpha"),
                          f32("W0"), f32("S0"), dy[s], dWe[s], dSe[s])
        for name, g in ref.items():
            got = out[name].reshape(n, *g.shape).double().cpu().numpy()[s]
            worst[name] = max(worst.get(name, 0.0), rel(got, g))
    assert all(np.isfinite(v) for v in worst.values()), worst
    tc = dt == "bf16" and path == "auto"
    print(f"\n{'tcgen05 TF32' if tc else 'fp32 FFMA'} backward, worst relative error per gradient:",
          {k: f"{v:.1e}" for k, v in worst.items()})
    assert max(worst.values()) < (TOL_TC if tc else TOL), worst


@pytest.mark.gpu
def test_tensor_core_backward_is_bit_identical_across_runs():
    """The TF32 products sum over k in a fixed order: repeated calls agree bit for bit."""
    L, d, e, B, H, T, C = 4, 128, 2, 1, 2, 96, 32
    w = W.make(L, d, e, B, H, T, C, index=790)
    dev = to_dev(W.generate(w), B, H, "bf16")
    g = torch.Generator(device="cuda")
    g.manual_seed(7)
    dy = torch.randn((B, H, T, d), generator=g, device="cuda")
    dW = torch.randn(dev["W0"].shape, generator=g, device="cuda")
    dS = torch.randn(dev["S0"].shape, generator=g, device="cuda")
    mem = NeuralMemory(L, d, e)
    run = lambda: mem.backward(dev["k"], dev["v"], dev["q"], dev["theta"], dev["eta"], dev["alpha"], dev["W0"],
                               dev["S0"], dy, dW, dS, C)
    a = run()
    b = run()
    torch.cuda.synchronize()
    for k in a:
        assert torch.equal(a[k], b[k]), k


@pytest.mark.gpu
@pytest.mark.parametrize("idx", [2, 4], ids=["mlp2-d64-h8", "mlp4-d128-deep"])
def test_tensor_core_backward_matches_fp32_at_full_length(idx):
    """Over the whole stream (128 chunks of the eight-head workload, 256 of the
    deep one) the TF32 products do not drift: every gradient of every stream
    matches the fp32 form (itself held to 1e-4 of the float64 oracle above) within
    the TF32 bound. Measured: at most 9e-4 and 2.7e-3 (the alpha gradient)."""
    w = W.get(idx)
    dev = to_dev(W.generate(w), w.B, w.H, w.dtype)
    g = torch.Generator(device="cuda")
    g.manual_seed(5)
    dy = torch.randn((w.B, w.H, w.T, w.d), generator=g, device="cuda")
    dW = torch.randn(dev["W0"].shape, generator=g, device="cuda")
    dS = torch.randn(dev["S0"].shape, generator=g, device="cuda")
    out = {}
    for path in ("auto", "simt"):
        mem = NeuralMemory(w.L, w.d, w.expansion, path=path)
        out[path] = mem.backward(dev["k"], dev["v"], dev["q"], dev["theta"], dev["eta"], dev["alpha"], dev["W0"],
                                 dev["S0"], dy, dW, dS, w.C)
    torch.cuda.synchronize()
    n = w.streams
    worst = {}
    for k in out["auto"]:
        a = out["auto"][k].reshape(n, -1).double()
        b = out["simt"][k].reshape(n, -1).double()
        worst[k] = ((a - b).norm(dim=1) / b.norm(dim=1).clamp_min(1e-30)).max().item()
    print("\nTF32 vs fp32 backward at full length, worst per-stream relative error:",
          {k: f"{v:.1e}" for k, v in worst.items()})
    assert all(np.isfinite(v) for v in worst.values()), worst
    assert max(worst.values()) < TOL_TC, worst


@pytest.mark.gpu
def test_tensor_core_backward_timeout_is_reported_and_context_survives():
    """With the test hook on (tm_set_debug), each CTA's first tensor-core
    product first waits on a barrier that nothing completes: the wait runs out
    after 1 ms, TM_ERR_TIMEOUT is recorded in the call's workspace and reported
    by tm_sync, and nothing hangs. The next call on the same context (hook off)
    matches the fp32 form."""
    from test_trained_neural_b200._native import TitansMemError
    lib = N.load()
    L, d, e, B, H, T, C = 2, 64, 4, 1, 2, 128, 64
    w = W.make(L, d, e, B, H, T, C, index=795)
    dev = to_dev(W.generate(w), B, H, "bf16")
    g = torch.Generator(device="cuda")
    g.manual_seed(3)
    dy = torch.randn((B, H, T, d), generator=g, device="cuda")
    dW = torch.randn(dev["W0"].shape, generator=g, device="cuda")
    dS = torch.randn(dev["S0"].shape, generator=g, device="cuda")
    mem = NeuralMemory(L, d, e)
    args = (dev["k"], dev["v"], dev["q"], dev["theta"], dev["eta"], dev["alpha"], dev["W0"], dev["S0"], dy, dW, dS, C)
    ws = torch.empty(mem.backward_workspace_size(B, H, T, C, torch.bfloat16), dtype=torch.uint8, device="cuda")
    assert lib.tm_set_debug(1, 1_000_000) == N.TM_OK
    try:
        mem.backward(*args, workspace=ws)
        with pytest.raises(TitansMemError) as ei:
            mem.sync(ws)
        assert ei.value.code == N.TM_ERR_TIMEOUT
    finally:
        lib.tm_set_debug(0, 0)
    got = mem.backward(*args, workspace=ws)
    mem.sync(ws)
    ref = NeuralMemory(L, d, e, path="simt").backward(*args)
    torch.cuda.synchronize()
    for k in got:
        assert rel(got[k].double().cpu().numpy(), ref[k].double().cpu().numpy()) < TOL_TC, k


def test_backward_refuses_before_any_launch():
    lib = N.load()
    h = ctypes.c_void_p()
    n = ctypes.c_size_t()
    assert lib.tm_create(4, 64, 2, N.TM_ACT_SILU, ctypes.byref(h)) == N.TM_OK
    assert lib.tm_backward_workspace_size(h, 1, 1, 64, 16, N.TM_F32, ctypes.byref(n)) == N.TM_OK
    assert lib.tm_backward_workspace_size(h, 1, 1, 64, 512, N.TM_F32, ctypes.byref(n)) != N.TM_OK
    lib.tm_destroy(h)
    assert lib.tm_create(1, 64, 1, N.TM_ACT_SILU, ctypes.byref(h)) == N.TM_OK
    assert lib.tm_backward_workspace_size(h, 1, 1, 64, 16, N.TM_F32, ctypes.byref(n)) == N.TM_OK
    assert n.value > 256
    p = [ctypes.c_void_p((i + 1) << 32) for i in range(20)]
    assert lib.tm_backward(h, 1, 1, 64, 16, N.TM_F32, *p, ctypes.c_size_t(0), None) == N.TM_ERR_OOM
    assert lib.tm_backward(h, 1, 1, 64, 16, N.TM_F32, *([None] + p[1:]), ctypes.c_size_t(1 << 30), None) == \
        N.TM_ERR_INVALID_ARG
    lib.tm_destroy(h)
