"""tm_run_noalloc: the write-and-read for callers that cannot allocate device
memory where they run it (a serving loop with a latency budget, in which
cudaMalloc/cudaFree may synchronize the device; code inside a framework whose
memory manager owns all device memory). Instead of a caller workspace it uses
a fixed array in the library's own device memory.

The test calls it through the C ABI several times in a row and checks each
result against tm_run on the same inputs (fp32 tolerance of the other tests)
and against the float64 oracle. A larger problem runs first, then a smaller
one with a different chunk size, so the second call finds the first call's
leftovers in the shared array. Around a warmed-up call, the device's free
memory does not move and torch's allocation count does not grow. It also checks that a
problem too large for the array, and a call whose y overlaps an input, are
refused before any launch. This file is collected last on purpose.
"""
import ctypes
import gc

import numpy as np
import pytest
import torch

import oracle
from gen import workloads as W
from test_trained_neural_b200 import NeuralMemory
from test_trained_neural_b200 import _native as N

from gpu_util import gpu_to_np, parity_errors, to_dev

pytestmark = pytest.mark.gpu

TOL_F32 = 1e-4


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def call_noalloc(mem, dev, C, y, We, Se):
    lib = N.load()
    B, H, T, d = dev["k"].shape
    dt = N.TM_BF16 if dev["k"].dtype == torch.bfloat16 else N.TM_F32
    stream = torch.cuda.current_stream()
    return lib.tm_run_noalloc(mem._h, B, H, T, C, dt, _p(dev["k"]), _p(dev["v"]), _p(dev["q"]),
                              _p(dev["theta"]), _p(dev["eta"]), _p(dev["alpha"]), _p(dev["W0"]),
                              _p(dev["S0"]), _p(y), _p(We), _p(Se), ctypes.c_void_p(stream.cuda_stream))


def run_noalloc(mem, dev, C):
    B, H, T, d = dev["k"].shape
    y = torch.full((B, H, T, d), float("nan"), dtype=torch.float32, device="cuda")
    We = torch.full_like(dev["W0"], float("nan"))
    Se = torch.full_like(dev["S0"], float("nan"))
    rc = call_noalloc(mem, dev, C, y, We, Se)
    torch.cuda.synchronize()
    return rc, y, We, Se


CASES = [  # (workload, chunk size used for the call)
    (W.make(2, 64, 4, 2, 2, 384, 64, index=952), 64),     # the larger problem first
    (W.get(0), None),
    (W.make(2, 64, 4, 1, 4, 256, 64, index=950), 32),     # smaller, another chunk size
    (W.make(4, 32, 2, 2, 1, 128, 32, dtype="f32", index=951), None),
]


def test_noalloc_matches_tm_run_and_oracle_on_calls_in_a_row():
    for w, C in CASES:
        C = C or w.C
        inp = W.generate(w)
        dev = to_dev(inp, w.B, w.H, w.dtype)
        mem = NeuralMemory(w.L, w.d, w.expansion, path="simt")
        ref = mem.run(dev["k"], dev["v"], dev["q"], dev["theta"], dev["eta"], dev["alpha"],
                      dev["W0"], dev["S0"], C, sync=True)
        torch.cuda.synchronize()
        ref_np = gpu_to_np(*ref)
        orc = oracle.run(w.dims, C, inp["k"], inp["v"], inp["q"], inp["theta"], inp["eta"], inp["alpha"],
                         inp["W0"], inp["S0"])
        for call in range(2):
            rc, y, We, Se = run_noalloc(mem, dev, C)
            assert rc == N.TM_OK, N.status_string(rc)
            got = gpu_to_np(y, We, Se)
            errs = parity_errors(w.dims, inp["W0"], got, ref_np)
            assert all(np.isfinite(v) for v in errs.values()), (w.name, call, errs)
            assert max(errs.values()) < TOL_F32, (w.name, call, errs)
            errs = parity_errors(w.dims, inp["W0"], got, orc)
            assert max(errs.values()) < TOL_F32, (w.name, call, "oracle", errs)


def test_noalloc_allocates_nothing():
    w = W.make(2, 64, 4, 1, 2, 256, 64, index=953)
    dev = to_dev(W.generate(w), w.B, w.H, w.dtype)
    mem = NeuralMemory(w.L, w.d, w.expansion)
    y = torch.empty((w.B, w.H, w.T, w.d), dtype=torch.float32, device="cuda")
    We, Se = torch.empty_like(dev["W0"]), torch.empty_like(dev["S0"])
    assert call_noalloc(mem, dev, w.C, y, We, Se) == N.TM_OK    # set-up on this device
    torch.cuda.synchronize()
    gc.collect()                 # tensors of earlier tests are released now, not during the calls
    free0, alloc0 = torch.cuda.mem_get_info()[0], torch.cuda.memory_allocated()
    for _ in range(3):
        assert call_noalloc(mem, dev, w.C, y, We, Se) == N.TM_OK
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0          # the device's free memory did not move
    assert torch.cuda.memory_allocated() <= alloc0


def test_noalloc_refuses_problems_larger_than_its_array():
    w = W.get(4)   # 64 streams of a depth-4 memory: far more than 16 MiB of activations
    mem = NeuralMemory(w.L, w.d, w.expansion)
    lib = N.load()
    small = torch.zeros(16, device="cuda")
    p = _p(small)
    rc = lib.tm_run_noalloc(mem._h, w.B, w.H, w.T, w.C, N.TM_BF16, *([p] * 11), None)
    assert rc == N.TM_ERR_OOM


def test_noalloc_refuses_y_overlapping_an_input():
    w = W.make(1, 64, 1, 1, 1, 64, 16, dtype="f32", index=954, xavier_w0=False)
    dev = to_dev(W.generate(w), w.B, w.H, w.dtype)
    mem = NeuralMemory(w.L, w.d, w.expansion)
    We, Se = torch.empty_like(dev["W0"]), torch.empty_like(dev["S0"])
    # y the same shape and dtype as k, and at k's address: tm_run refuses it, so must this
    assert call_noalloc(mem, dev, w.C, dev["k"], We, Se) == N.TM_ERR_INVALID_ARG
    # the state outputs partially overlapping the initial state
    y = torch.empty((w.B, w.H, w.T, w.d), dtype=torch.float32, device="cuda")
    both = torch.zeros(2 * w.P + 4, device="cuda")
    assert call_noalloc(mem, {**dev, "W0": both[:w.P]}, w.C, y, both[4:4 + w.P], Se) == N.TM_ERR_INVALID_ARG
