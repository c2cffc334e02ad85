"""Full-length parity of the two long workloads: every stream's reads y, and
its final state W_end and S_end, against the float64 oracle.

The library runs each workload once, at full length and in the launch
configuration the benchmark times (automatic path choice). The oracle then
walks the same streams in segments of whole chunks, carrying its float64
state from one segment into the next; carrying (W_end, S_end) into the next
call equals one longer call ("titans-pytorch" review, "NeuralMemory as a
standalone module"), which the CPU pins check on the oracle itself. This keeps
host memory bounded while every token of every stream is compared.

Error measure: normwise relative error per stream and per output (y over the
whole stream; each layer of W_end and S_end; each layer of the written part
W_end - W0), max over streams. Tolerance 2e-2, that of the bf16 tensor-core
path. The worst error per tensor is printed (pytest -s shows it) together
with its growth over the stream (y error of the first and last segment).
"""
import numpy as np
import pytest
import torch

import oracle
from gen import workloads as W
from test_trained_neural_b200 import NeuralMemory

from gpu_util import to_dev

pytestmark = pytest.mark.gpu

TOL_BF16_TC = 2e-2


def _segment_inputs(inp, t0, t1):
    return {k: np.ascontiguousarray(inp[k][:, t0:t1]) for k in ("k", "v", "q", "theta", "eta", "alpha")}


@pytest.mark.parametrize("idx,seg", [(3, 16384), (4, 8192)], ids=["mlp2-d128-long", "mlp4-d128-deep"])
def test_full_length_state_and_reads(idx, seg):
    w = W.get(idx)
    assert w.T % seg == 0 and seg % w.C == 0
    inp = W.generate(w)
    n = w.streams
    dev = to_dev(inp, w.B, w.H, w.dtype)
    mem = NeuralMemory(w.L, w.d, w.expansion, path="auto")
    path = mem.query_path(w.B, w.H, w.T, w.C)
    assert path in ("tc", "tcl"), path
    y, We, Se = mem.run(dev["k"], dev["v"], dev["q"], dev["theta"], dev["eta"], dev["alpha"],
                        dev["W0"], dev["S0"], w.C, sync=True)
    torch.cuda.synchronize()
    del dev
    assert torch.isfinite(We).all() and torch.isfinite(Se).all()
    yf = y.reshape(n, w.T, w.d)

    # oracle in segments, float64 state carried across them
    Wc = inp["W0"].astype(np.float64)
    Sc = inp["S0"].astype(np.float64)
    dy2 = np.zeros(n)
    ny2 = np.zeros(n)
    seg_err = []
    for t0 in range(0, w.T, seg):
        part = _segment_inputs(inp, t0, t0 + seg)
        ref = oracle.run(w.dims, w.C, part["k"], part["v"], part["q"], part["theta"], part["eta"],
                         part["alpha"], Wc, Sc)
        Wc, Sc = ref["W_end"], ref["S_end"]
        got = yf[:, t0:t0 + seg].double().cpu().numpy()
        d2 = ((got - ref["y"]) ** 2).sum(axis=(1, 2))
        r2 = (ref["y"] ** 2).sum(axis=(1, 2))
        dy2 += d2
        ny2 += r2
        seg_err.append(float(np.max(np.sqrt(d2 / r2))))
        del got, ref, part
    errs = {"y": float(np.max(np.sqrt(dy2 / ny2)))}
    gW = We.reshape(n, -1).double().cpu().numpy()
    gS = Se.reshape(n, -1).double().cpu().numpy()
    W0 = inp["W0"].astype(np.float64)
    offs = W.layer_offsets(w.dims) + [w.P]
    rel = lambda a, b: float(np.linalg.norm(a - b) / np.linalg.norm(b))
    for key in ("W", "S", "dW"):
        errs[key] = 0.0
    for s in range(n):
        for l in range(w.L):
            sl = slice(offs[l], offs[l + 1])
            errs["W"] = max(errs["W"], rel(gW[s, sl], Wc[s, sl]))
            errs["S"] = max(errs["S"], rel(gS[s, sl], Sc[s, sl]))
            errs["dW"] = max(errs["dW"], rel(gW[s, sl] - W0[s, sl], Wc[s, sl] - W0[s, sl]))
    print(f"\nfull-length parity {w.name} path={path} T={w.T} streams={n}: "
          + " ".join(f"{k}={v:.3e}" for k, v in errs.items())
          + f" | y err first segment {seg_err[0]:.3e}, last segment {seg_err[-1]:.3e}")
    assert all(np.isfinite(v) for v in errs.values()), errs
    assert max(errs.values()) < TOL_BF16_TC, errs
