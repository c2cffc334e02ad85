"""Helpers shared by the GPU tests: move generator arrays to the device, run the
library, and compare with the float64 oracle."""
from __future__ import annotations

import numpy as np
import torch

from gen import workloads as W


def to_dev(inp: dict, B: int, H: int, dtype: str, device="cuda") -> dict:
    """Generator arrays [n, ...] -> contiguous CUDA tensors [B, H, ...]."""
    out = {}
    for key in ("k", "v", "q"):
        a = np.ascontiguousarray(inp[key])
        if dtype == "bf16":
            t = torch.from_numpy(a.view(np.int16)).view(torch.bfloat16)
        else:
            t = torch.from_numpy(a)
        out[key] = t.reshape(B, H, *a.shape[1:]).to(device)
    for key in ("theta", "eta", "alpha", "W0", "S0"):
        a = np.ascontiguousarray(inp[key], dtype=np.float32)
        out[key] = torch.from_numpy(a).reshape(B, H, *a.shape[1:]).to(device)
    return out


def run_lib(mem, dev: dict, C: int, **kw):
    y, We, Se = mem.run(dev["k"], dev["v"], dev["q"], dev["theta"], dev["eta"], dev["alpha"],
                        dev["W0"], dev["S0"], C, sync=True, **kw)
    torch.cuda.synchronize()
    return y, We, Se


def rel(a: np.ndarray, b: np.ndarray) -> float:
    """Normwise relative error ||a - b|| / ||b|| (absolute when ||b|| = 0)."""
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    nb = np.linalg.norm(b)
    d = np.linalg.norm(a - b)
    return float(d / nb) if nb > 0 else float(d)


def parity_errors(dims, W0, gpu: dict, ref: dict) -> dict:
    """Max over streams of the normwise relative error of y, of each layer of
    W_end and S_end, and of each layer's written part W_end - W0."""
    offs = W.layer_offsets(dims) + [W.param_count(dims)]
    n = ref["y"].shape[0]
    errs = {"y": 0.0, "W": 0.0, "S": 0.0, "dW": 0.0}
    for s in range(n):
        errs["y"] = max(errs["y"], rel(gpu["y"][s], ref["y"][s]))
        for l in range(len(dims) - 1):
            sl = slice(offs[l], offs[l + 1])
            errs["W"] = max(errs["W"], rel(gpu["W_end"][s, sl], ref["W_end"][s, sl]))
            errs["S"] = max(errs["S"], rel(gpu["S_end"][s, sl], ref["S_end"][s, sl]))
            w0 = np.asarray(W0[s, sl], dtype=np.float64)
            errs["dW"] = max(errs["dW"], rel(gpu["W_end"][s, sl] - w0, ref["W_end"][s, sl] - w0))
    return errs


def gpu_to_np(y, We, Se) -> dict:
    n = y.shape[0] * y.shape[1]
    return {"y": y.reshape(n, *y.shape[2:]).double().cpu().numpy(),
            "W_end": We.reshape(n, -1).double().cpu().numpy(),
            "S_end": Se.reshape(n, -1).double().cpu().numpy()}
