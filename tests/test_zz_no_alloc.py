"""tm_run_noalloc: the write-and-read for callers that cannot allocate device
memory where they run it (a serving loop with a latency budget, in which
cudaMalloc/cudaFree may synchronize the device; code inside a framework whose
memory manager owns all device memory). Instead of a caller workspace it uses
a fixed array in the library's own device memory.

The test calls it through the C ABI twice in a row (the second call finds the
first call's leftovers in the shared array) and checks both results against
tm_run on the same inputs, within the fp32 tolerance of the other tests. It
also checks that a problem too large for the array is refused before any
launch. This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

from gen import workloads as W
from test_trained_neural_b200 import NeuralMemory
from test_trained_neural_b200 import _native as N

from gpu_util import gpu_to_np, parity_errors, to_dev

pytestmark = pytest.mark.gpu

TOL_F32 = 1e-4


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def run_noalloc(mem, dev, C):
    lib = N.load()
    B, H, T, d = dev["k"].shape
    dt = N.TM_BF16 if dev["k"].dtype == torch.bfloat16 else N.TM_F32
    y = torch.full((B, H, T, d), float("nan"), dtype=torch.float32, device="cuda")
    We = torch.full_like(dev["W0"], float("nan"))
    Se = torch.full_like(dev["S0"], float("nan"))
    stream = torch.cuda.current_stream()
    rc = lib.tm_run_noalloc(mem._h, B, H, T, C, dt, _p(dev["k"]), _p(dev["v"]), _p(dev["q"]),
                            _p(dev["theta"]), _p(dev["eta"]), _p(dev["alpha"]), _p(dev["W0"]),
                            _p(dev["S0"]), _p(y), _p(We), _p(Se), ctypes.c_void_p(stream.cuda_stream))
    torch.cuda.synchronize()
    return rc, y, We, Se


@pytest.mark.parametrize("w", [W.get(0), W.make(2, 64, 4, 1, 4, 256, 64, index=950),
                               W.make(4, 32, 2, 2, 1, 128, 32, dtype="f32", index=951)],
                         ids=["linear-f32", "mlp2-bf16", "mlp4-f32"])
def test_noalloc_matches_tm_run_on_two_calls(w):
    inp = W.generate(w)
    dev = to_dev(inp, w.B, w.H, w.dtype)
    mem = NeuralMemory(w.L, w.d, w.expansion, path="simt")
    ref = mem.run(dev["k"], dev["v"], dev["q"], dev["theta"], dev["eta"], dev["alpha"],
                  dev["W0"], dev["S0"], w.C, sync=True)
    torch.cuda.synchronize()
    ref_np = gpu_to_np(*ref)
    for call in range(2):
        rc, y, We, Se = run_noalloc(mem, dev, w.C)
        assert rc == N.TM_OK, N.status_string(rc)
        errs = parity_errors(w.dims, inp["W0"], gpu_to_np(y, We, Se), ref_np)
        assert all(np.isfinite(v) for v in errs.values()), (call, errs)
        assert max(errs.values()) < TOL_F32, (call, errs)


def test_noalloc_refuses_problems_larger_than_its_array():
    w = W.get(4)   # 64 streams of a depth-4 memory: far more than 16 MiB of activations
    mem = NeuralMemory(w.L, w.d, w.expansion)
    lib = N.load()
    small = torch.zeros(16, device="cuda")
    p = _p(small)
    rc = lib.tm_run_noalloc(mem._h, w.B, w.H, w.T, w.C, N.TM_BF16, *([p] * 11), None)
    assert rc == N.TM_ERR_OOM
