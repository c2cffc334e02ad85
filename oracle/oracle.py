"""ctypes front end of the float64 oracle (test infrastructure).

Only tests/, the smoke check and bench.py's CPU-baseline leg may use it. The
arithmetic lives in titans_oracle.c; this file only marshals arrays.
"""
from __future__ import annotations

import contextlib
import ctypes
import os

import numpy as np

from . import build as _build

DT_F64, DT_F32, DT_BF16 = 0, 1, 2
_lib = None


def _open(path):
    lib = ctypes.CDLL(path)
    P = ctypes.c_void_p
    I = ctypes.c_int
    lib.titans_oracle_run.argtypes = [I, P, I, I, I, I, P, P, P, I, P, P, P, I, P, P,
                                      P, P, P, P, P, P, I]
    lib.titans_oracle_run.restype = I
    lib.titans_oracle_surprise.argtypes = [I, P, P, P, P, P]
    lib.titans_oracle_surprise.restype = I
    return lib


def _load():
    global _lib
    if _lib is None:
        _lib = _open(_build.build())
    return _lib


@contextlib.contextmanager
def use_library(path):
    """Within the block, run() and surprise() call the oracle compiled at
    `path` (the tests use this to show that the pins reject an oracle with a
    planted mistake)."""
    global _lib
    prev = _load()
    _lib = _open(path)
    try:
        yield
    finally:
        _lib = prev


def _dtype_code(a: np.ndarray) -> int:
    if a.dtype == np.float64:
        return DT_F64
    if a.dtype == np.float32:
        return DT_F32
    if a.dtype == np.uint16:
        return DT_BF16
    raise TypeError(f"unsupported dtype {a.dtype}")


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def run(dims, C, k, v, q, theta, eta, alpha, W0, S0, threads=None, trace=False):
    """Run the recurrence. Shapes: k, q [n, T, dims[0]], v [n, T, dims[-1]],
    gates [n, T], W0/S0 [n, P]. bf16 tokens are passed as uint16 bit patterns.
    Returns dict y [n, T, d_out], W_end, S_end [n, P] (float64), plus u/S/W
    traces [n, T, P] when trace=True."""
    lib = _load()
    dims = [int(x) for x in dims]
    L = len(dims) - 1
    k, v, q = (np.ascontiguousarray(a) for a in (k, v, q))
    theta, eta, alpha = (np.ascontiguousarray(a) for a in (theta, eta, alpha))
    W0, S0 = np.ascontiguousarray(W0), np.ascontiguousarray(S0)
    n, T = k.shape[0], k.shape[1]
    P = sum(dims[i] * dims[i + 1] for i in range(L))
    assert k.shape == (n, T, dims[0]) and q.shape == (n, T, dims[0]), (k.shape, dims)
    assert v.shape == (n, T, dims[-1])
    assert theta.shape == (n, T) and eta.shape == (n, T) and alpha.shape == (n, T)
    assert W0.shape == (n, P) and S0.shape == (n, P)
    tdt = _dtype_code(k)
    assert _dtype_code(v) == tdt and _dtype_code(q) == tdt
    gdt = _dtype_code(theta)
    assert _dtype_code(eta) == gdt and _dtype_code(alpha) == gdt and gdt != DT_BF16
    sdt = _dtype_code(W0)
    assert _dtype_code(S0) == sdt and sdt != DT_BF16
    y = np.zeros((n, T, dims[-1]), dtype=np.float64)
    We = np.zeros((n, P), dtype=np.float64)
    Se = np.zeros((n, P), dtype=np.float64)
    tr = [np.zeros((n, T, P), dtype=np.float64) for _ in range(3)] if trace else [None] * 3
    dims_c = (ctypes.c_int * len(dims))(*dims)
    threads = threads or min(n, os.cpu_count() or 1) or 1
    rc = lib.titans_oracle_run(L, ctypes.cast(dims_c, ctypes.c_void_p), n, T, int(C),
                               tdt, _ptr(k), _ptr(v), _ptr(q),
                               gdt, _ptr(theta), _ptr(eta), _ptr(alpha),
                               sdt, _ptr(W0), _ptr(S0),
                               _ptr(y), _ptr(We), _ptr(Se),
                               _ptr(tr[0]), _ptr(tr[1]), _ptr(tr[2]), int(threads))
    if rc != 0:
        raise RuntimeError(f"titans_oracle_run failed with code {rc}")
    out = {"y": y, "W_end": We, "S_end": Se}
    if trace:
        out["u"], out["S"], out["W"] = tr
    return out


def run_workload(w, inputs, threads=None):
    """Run the oracle on inputs drawn by gen.workloads.generate for workload w."""
    return run(w.dims, w.C, inputs["k"], inputs["v"], inputs["q"], inputs["theta"],
               inputs["eta"], inputs["alpha"], inputs["W0"], inputs["S0"], threads=threads)


def surprise(dims, W, k, v):
    """u = grad_W ||M(k) - v||^2 at weights W (float64 [P]); returns [P]."""
    lib = _load()
    dims = [int(x) for x in dims]
    L = len(dims) - 1
    W = np.ascontiguousarray(W, dtype=np.float64)
    k = np.ascontiguousarray(k, dtype=np.float64)
    v = np.ascontiguousarray(v, dtype=np.float64)
    u = np.zeros_like(W)
    dims_c = (ctypes.c_int * len(dims))(*dims)
    rc = lib.titans_oracle_surprise(L, ctypes.cast(dims_c, ctypes.c_void_p), _ptr(W), _ptr(k),
                                    _ptr(v), _ptr(u))
    if rc != 0:
        raise RuntimeError(f"titans_oracle_surprise failed with code {rc}")
    return u
