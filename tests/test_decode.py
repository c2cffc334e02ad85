"""One-token decode step (the write-and-read with C = 1, state in place)
against the float64 oracle run with chunk size 1 over the same tokens."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from gen import workloads as W
from test_trained_neural_b200 import NeuralMemory
from test_trained_neural_b200 import _native as N

from gpu_util import parity_errors, to_dev

TOL = 1e-4   # fp32 arithmetic throughout (bf16 inputs are consumed exactly by the oracle)

DECODE = [  # L, d, expansion, B, H, T (steps), dtype
    (2, 128, 4, 1, 3, 6, "bf16"),    # cluster of 8 CTAs per stream
    (2, 64, 4, 2, 2, 5, "f32"),      # cluster of 4
    (2, 128, 1, 1, 2, 4, "bf16"),    # cluster of 2
    (1, 64, 1, 1, 2, 7, "f32"),      # linear memory
    (1, 96, 1, 2, 1, 3, "bf16"),
]


@pytest.mark.gpu
@pytest.mark.parametrize("cfg", DECODE, ids=lambda c: "L%d-d%d-e%d-B%dH%d-T%d-%s" % c)
def test_decode_steps_match_oracle(cfg):
    L, d, e, B, H, T, dt = cfg
    w = W.make(L, d, e, B, H, T, 1, dtype=dt, index=660 + T + d)
    inp = W.generate(w)
    dev = to_dev(inp, B, H, dt)
    mem = NeuralMemory(L, d, e)
    Wst, Sst = dev["W0"].clone(), dev["S0"].clone()
    ys = []
    for t in range(T):
        tok = {key: dev[key][:, :, t].contiguous() for key in ("k", "v", "q", "theta", "eta", "alpha")}
        ys.append(mem.decode_step(tok["k"], tok["v"], tok["q"], tok["theta"], tok["eta"], tok["alpha"], Wst, Sst))
    torch.cuda.synchronize()
    y = torch.stack(ys, dim=2)
    n = B * H
    got = {"y": y.reshape(n, T, d).double().cpu().numpy(),
           "W_end": Wst.reshape(n, -1).double().cpu().numpy(),
           "S_end": Sst.reshape(n, -1).double().cpu().numpy()}
    ref = oracle.run_workload(w, inp)
    errs = parity_errors(w.dims, inp["W0"], got, ref)
    assert all(np.isfinite(v) for v in errs.values()), errs
    assert max(errs.values()) < TOL, errs


def test_decode_refuses_before_any_launch():
    lib = N.load()
    h = ctypes.c_void_p()
    assert lib.tm_create(2, 384, 4, N.TM_ACT_SILU, ctypes.byref(h)) == N.TM_OK
    p = [ctypes.c_void_p((i + 1) << 32) for i in range(9)]   # never dereferenced: refused on the host
    assert lib.tm_decode_step(h, 1, 1, N.TM_BF16, *p, None) == N.TM_ERR_UNSUPPORTED
    assert lib.tm_decode_step(h, 1, 1, N.TM_BF16, *([None] + p[1:]), None) == N.TM_ERR_INVALID_ARG
    assert lib.tm_decode_step(h, 0, 1, N.TM_BF16, *p, None) == N.TM_ERR_INVALID_ARG
    lib.tm_destroy(h)
