"""tm_run_host: the write-and-read with every input and output in host memory,
the copies made by the library in segments of T and overlapped with the
kernels. Its results equal one tm_run on device buffers bit for bit (the
state is carried on the device between segments, and carrying the state
equals one longer call: "titans-pytorch" review, "NeuralMemory as a
standalone module"), and match the oracle.
"""
import numpy as np
import pytest
import torch

import oracle
from gen import workloads as W
from test_trained_neural_b200 import NeuralMemory
from test_trained_neural_b200 import _native as N
from test_trained_neural_b200._native import TitansMemError

from gpu_util import gpu_to_np, parity_errors, run_lib, to_dev

TOL_F32 = 1e-4
TOL_BF16_TC = 2e-2


def _host(dev: dict, pin: bool) -> dict:
    return {k: (v.cpu().pin_memory() if pin else v.cpu()) for k, v in dev.items()}


CASES = [  # workload, path, segment lengths to try
    (W.make(1, 64, 1, 1, 2, 200, 16, dtype="f32", index=960, xavier_w0=False), "simt", [0, 32, 48, 200]),
    (W.make(2, 128, 4, 1, 3, 640, 64, index=961), "tc", [0, 128, 192, 1024]),
    (W.make(4, 64, 2, 2, 2, 768, 128, index=962), "tcl", [0, 256, 384]),
    (W.make(2, 64, 4, 1, 2, 300, 64, index=963), "tc", [128]),   # last segment ends with a short chunk
]


@pytest.mark.gpu
@pytest.mark.parametrize("case", CASES, ids=lambda c: f"{c[1]}-T{c[0].T}-C{c[0].C}")
def test_run_host_equals_device_run_and_oracle(case):
    w, path, segs = case
    inp = W.generate(w)
    dev = to_dev(inp, w.B, w.H, w.dtype)
    mem = NeuralMemory(w.L, w.d, w.expansion, path=path)
    ref_dev = run_lib(mem, dev, w.C)
    tol = TOL_F32 if w.dtype == "f32" else TOL_BF16_TC
    orc = oracle.run_workload(w, inp)
    for i, seg in enumerate(segs):
        host = _host(dev, pin=(i % 2 == 0))
        y, We, Se = mem.run_host(host["k"], host["v"], host["q"], host["theta"], host["eta"], host["alpha"],
                                 host["W0"], host["S0"], w.C, segment_tokens=seg)
        assert not y.is_cuda
        for a, b in zip((y, We, Se), ref_dev):
            assert torch.equal(a, b.cpu()), (path, seg)
        errs = parity_errors(w.dims, inp["W0"], gpu_to_np(y, We, Se), orc)
        assert max(errs.values()) < tol, (path, seg, errs)


@pytest.mark.gpu
def test_run_host_in_place_state_and_repeated_calls():
    """W_end = W0 and S_end = S0 on the host (in place), and a second call
    continuing from the state the first left (state carry across calls)."""
    w = W.make(2, 64, 4, 1, 2, 256, 64, index=964)
    inp = W.generate(w)
    dev = to_dev(inp, w.B, w.H, w.dtype)
    mem = NeuralMemory(w.L, w.d, w.expansion)
    host = _host(dev, pin=True)
    W0, S0 = host["W0"].clone(), host["S0"].clone()
    y1, _, _ = mem.run_host(host["k"], host["v"], host["q"], host["theta"], host["eta"], host["alpha"],
                            W0, S0, w.C, W_end=W0, S_end=S0, segment_tokens=64)
    y2, W2, S2 = mem.run_host(host["k"], host["v"], host["q"], host["theta"], host["eta"], host["alpha"],
                              W0, S0, w.C, segment_tokens=128)
    both = {k: torch.cat([v, v], dim=2) if k in ("k", "v", "q", "theta", "eta", "alpha") else v
            for k, v in dev.items()}
    yr, Wr, Sr = run_lib(mem, {k: v.contiguous() for k, v in both.items()}, w.C)
    assert torch.equal(torch.cat([y1, y2], dim=2), yr.cpu())
    assert torch.equal(W2, Wr.cpu()) and torch.equal(S2, Sr.cpu())


@pytest.mark.gpu
def test_run_host_argument_errors():
    w = W.make(2, 64, 4, 1, 2, 256, 64, index=965)
    mem = NeuralMemory(w.L, w.d, w.expansion)
    dev = to_dev(W.generate(w), w.B, w.H, w.dtype)
    host = _host(dev, pin=False)
    with pytest.raises(TitansMemError) as ei:       # segment not a multiple of C
        mem.run_host(host["k"], host["v"], host["q"], host["theta"], host["eta"], host["alpha"],
                     host["W0"], host["S0"], w.C, segment_tokens=100)
    assert ei.value.code == N.TM_ERR_INVALID_ARG
    with pytest.raises(TitansMemError) as ei:       # workspace too small
        mem.run_host(host["k"], host["v"], host["q"], host["theta"], host["eta"], host["alpha"],
                     host["W0"], host["S0"], w.C, workspace=torch.empty(1024, dtype=torch.uint8, device="cuda"))
    assert ei.value.code == N.TM_ERR_OOM


def test_host_workspace_size_without_a_gpu():
    """Sizes are host arithmetic: they grow with the segment, and a segment
    that is not a multiple of C (and shorter than T) is refused."""
    mem = NeuralMemory(1, 64, 1, path="simt")
    a = mem.host_workspace_size(1, 2, 1024, 16, torch.float32, segment_tokens=64)
    b = mem.host_workspace_size(1, 2, 1024, 16, torch.float32, segment_tokens=256)
    assert 0 < a < b
    assert mem.host_workspace_size(1, 2, 1024, 16, torch.float32, segment_tokens=5000) > b
    with pytest.raises(TitansMemError) as ei:
        mem.host_workspace_size(1, 2, 1024, 16, torch.float32, segment_tokens=40)
    assert ei.value.code == N.TM_ERR_INVALID_ARG
