"""Seeded synthetic inputs for the neural long-term memory write-and-read.

This module only draws random numbers and fixes shapes. It holds none of the
memory's arithmetic (no forward pass, gradient, momentum or forgetting), so both
the float64 oracle and the CUDA path can consume the same bytes from it.

Workloads
---------
The five workloads are synthetic stand-ins for the shapes the Titans pages talk
about ("titans-pytorch" review, section "NeuralMemory as a standalone module":
dim=384, chunk_size=64, input (2, 1024, 384)); no dataset is involved.

Draw recipe (fixed; changing it changes every stored expectation)
----------------------------------------------------------------
* Stream s = b*H + h has its own generator
  ``PCG64(SeedSequence(entropy=seed, spawn_key=(s,)))`` with seed = 1000 + index.
* Tokens are drawn in blocks of ``BLOCK`` (1024) tokens. Per block, in order:
  k (BLOCK x d normal), v (BLOCK x d normal), q (BLOCK x d normal),
  theta, eta, alpha (BLOCK uniform each), then for spiking workloads a
  Bernoulli(p) mask (BLOCK uniform < p) and, for the masked rows only,
  a fresh N(0, sigma^2) draw that replaces v.  A prefix of T' tokens therefore
  equals the first T' tokens of the full draw, whatever T is.
* k and q rows are L2-normalised in float64, then cast to the workload dtype.
  float32: numpy round-to-nearest-even.  bfloat16: float64 -> float32 (RNE),
  then float32 -> bfloat16 by round-to-nearest-even on the top 16 bits; stored
  as raw uint16.
* Gates are cast to float32.
* W0 is Xavier-normal per layer, std = sqrt(2 / (fan_in + fan_out)), drawn per
  head from ``PCG64(SeedSequence(entropy=seed, spawn_key=(1_000_000 + h,)))``
  and shared by every batch entry of that head; W0 = 0 for the linear workload.
  S0 = 0 everywhere.  Both are float32.
"""
from __future__ import annotations

import concurrent.futures
import dataclasses
import os
from typing import Sequence

import numpy as np

BLOCK = 1024


@dataclasses.dataclass(frozen=True)
class Workload:
    index: int
    name: str
    L: int            # memory depth (number of weight matrices)
    d: int            # head dimension d_h
    expansion: int    # hidden width = expansion * d (unused for L == 1)
    B: int
    H: int
    T: int
    C: int            # chunk size
    dtype: str        # "f32" or "bf16" for k, v, q
    theta: tuple      # U[lo, hi]
    eta: tuple
    alpha: tuple
    xavier_w0: bool
    spike_p: float = 0.0
    spike_sigma: float = 0.0
    theta_damping: float = 1.0  # multiplies the theta draws
    alpha_damping: float = 1.0  # multiplies the alpha draws (eta is never damped)

    @property
    def dims(self) -> list:
        return layer_dims(self.L, self.d, self.expansion)

    @property
    def P(self) -> int:
        return param_count(self.dims)

    @property
    def streams(self) -> int:
        return self.B * self.H

    @property
    def seed(self) -> int:
        return 1000 + self.index


def layer_dims(L: int, d: int, expansion: int) -> list:
    """n_0..n_L: d, then L-1 hidden widths of expansion*d, then d."""
    if L == 1:
        return [d, d]
    return [d] + [expansion * d] * (L - 1) + [d]


def param_count(dims: Sequence[int]) -> int:
    return int(sum(dims[i + 1] * dims[i] for i in range(len(dims) - 1)))


def layer_offsets(dims: Sequence[int]) -> list:
    """Offset of layer l (0-based) inside a flat [P] parameter vector; layer l is
    a row-major [dims[l+1] x dims[l]] block."""
    off, out = 0, []
    for i in range(len(dims) - 1):
        out.append(off)
        off += dims[i + 1] * dims[i]
    return out


_G_SMALL = (0.001, 0.1)
WORKLOADS = [
    Workload(0, "linear-d64", 1, 64, 1, 1, 1, 256, 16, "f32",
             _G_SMALL, (0.8, 0.99), (0.0, 0.01), xavier_w0=False),
    Workload(1, "mlp2-d384-readme", 2, 384, 4, 2, 1, 1024, 64, "bf16",
             _G_SMALL, (0.8, 0.99), (0.0, 0.01), xavier_w0=True),
    Workload(2, "mlp2-d64-h8", 2, 64, 4, 4, 8, 8192, 64, "bf16",
             _G_SMALL, (0.8, 0.99), (0.0, 0.01), xavier_w0=True),
    Workload(3, "mlp2-d128-long", 2, 128, 4, 1, 16, 262144, 64, "bf16",
             _G_SMALL, (0.8, 0.99), (0.0, 0.01), xavier_w0=True,
             spike_p=0.01, spike_sigma=2.0),
    Workload(4, "mlp4-d128-deep", 4, 128, 2, 8, 8, 32768, 128, "bf16",
             (0.001, 0.05), (0.9, 0.99), (0.0, 0.005), xavier_w0=True),
]


# Gate damping of the MLP workloads. Drawn literally, theta ~ U[.001, .1] (or
# U[.001, .05]) and alpha ~ U[0, .01] (or U[0, .005]) make a depth >= 2 memory
# fed i.i.d. keys and values overflow within a few chunks; lowering theta alone
# makes it collapse to zero under the forgetting, and the band in between is a
# knife edge that gives way over a long stream (the float64 oracle shows all
# three). Scaling the theta draws by 0.03 and the alpha draws by 0.01 keeps
# every MLP workload finite, non-zero and insensitive to small perturbations
# over its full length. The linear workload is stable as drawn.
MLP_THETA_DAMPING = 0.03
MLP_ALPHA_DAMPING = 0.01


def get(index: int) -> Workload:
    """Workload `index` as used for parity and benchmarking (damped gates for
    the MLP memories)."""
    w = WORKLOADS[index]
    if w.L >= 2:
        return dataclasses.replace(w, theta_damping=MLP_THETA_DAMPING,
                                   alpha_damping=MLP_ALPHA_DAMPING)
    return w


def get_literal(index: int) -> Workload:
    """Workload `index` with the gate ranges exactly as specified."""
    return WORKLOADS[index]


def make(L: int, d: int, expansion: int, B: int, H: int, T: int, C: int, dtype: str = "bf16",
         theta=(0.001, 0.1), eta=(0.8, 0.99), alpha=(0.0, 0.01), theta_damping=None,
         alpha_damping=None, index: int = 100, xavier_w0: bool = True,
         spike_p: float = 0.0, spike_sigma: float = 0.0) -> Workload:
    """A custom workload (tests use small ones); seed = 1000 + index. The gate
    damping defaults to that of the MLP workloads for L >= 2, none for L = 1."""
    if theta_damping is None:
        theta_damping = MLP_THETA_DAMPING if L >= 2 else 1.0
    if alpha_damping is None:
        alpha_damping = MLP_ALPHA_DAMPING if L >= 2 else 1.0
    return Workload(index, f"custom-{index}", L, d, expansion, B, H, T, C, dtype, tuple(theta),
                    tuple(eta), tuple(alpha), xavier_w0, spike_p, spike_sigma, theta_damping,
                    alpha_damping)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bfloat16 bit patterns (uint16), round to nearest even."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    rounding = ((u >> 16) & 1) + 0x7FFF
    out = ((u + rounding) >> 16).astype(np.uint16)
    nan = np.isnan(x)
    if nan.any():
        out[nan] = 0x7FC0
    return out


def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _stream_rng(seed: int, s: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence(entropy=seed, spawn_key=(s,))))


def _head_rng(seed: int, h: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence(entropy=seed, spawn_key=(1_000_000 + h,))))


def _cast_tokens(x: np.ndarray, dtype: str) -> np.ndarray:
    if dtype == "f32":
        return x.astype(np.float32)
    return f32_to_bf16_bits(x.astype(np.float32))


def draw_stream(w: Workload, s: int, T: int | None = None, seed: int | None = None) -> dict:
    """Tokens and gates of stream s, first T tokens (default: all)."""
    T = w.T if T is None else T
    seed = w.seed if seed is None else seed
    rng = _stream_rng(seed, s)
    d = w.d
    tdt = np.float32 if w.dtype == "f32" else np.uint16
    out = {k: np.empty((T, d), dtype=tdt) for k in ("k", "v", "q")}
    for g in ("theta", "eta", "alpha"):
        out[g] = np.empty((T,), dtype=np.float32)
    for t0 in range(0, T, BLOCK):
        n = min(BLOCK, T - t0)
        k = rng.standard_normal((BLOCK, d))
        v = rng.standard_normal((BLOCK, d))
        q = rng.standard_normal((BLOCK, d))
        th = rng.uniform(w.theta[0], w.theta[1], BLOCK) * w.theta_damping
        et = rng.uniform(w.eta[0], w.eta[1], BLOCK)
        al = rng.uniform(w.alpha[0], w.alpha[1], BLOCK) * w.alpha_damping
        if w.spike_p > 0.0:
            mask = rng.uniform(0.0, 1.0, BLOCK) < w.spike_p
            nsp = int(mask.sum())
            v[mask] = w.spike_sigma * rng.standard_normal((nsp, d))
        k /= np.linalg.norm(k, axis=1, keepdims=True)
        q /= np.linalg.norm(q, axis=1, keepdims=True)
        out["k"][t0:t0 + n] = _cast_tokens(k[:n], w.dtype)
        out["v"][t0:t0 + n] = _cast_tokens(v[:n], w.dtype)
        out["q"][t0:t0 + n] = _cast_tokens(q[:n], w.dtype)
        out["theta"][t0:t0 + n] = th[:n]
        out["eta"][t0:t0 + n] = et[:n]
        out["alpha"][t0:t0 + n] = al[:n]
    return out


def draw_w0_head(w: Workload, h: int, seed: int | None = None) -> np.ndarray:
    """float32 [P] initial weights for head h (shared over the batch)."""
    seed = w.seed if seed is None else seed
    dims = w.dims
    if not w.xavier_w0:
        return np.zeros((w.P,), dtype=np.float32)
    rng = _head_rng(seed, h)
    parts = []
    for i in range(len(dims) - 1):
        fan_in, fan_out = dims[i], dims[i + 1]
        std = np.sqrt(2.0 / (fan_in + fan_out))
        parts.append((std * rng.standard_normal((fan_out, fan_in))).ravel())
    return np.concatenate(parts).astype(np.float32)


def generate(w: Workload, streams: Sequence[int] | None = None, T: int | None = None,
             seed: int | None = None) -> dict:
    """Inputs for the listed streams (default: all B*H), first T tokens.

    Returns k, v, q [n, T, d] (float32 or uint16 bf16 bits), theta/eta/alpha
    [n, T] float32, W0/S0 [n, P] float32, plus 'streams' (the indices).
    """
    streams = list(range(w.streams)) if streams is None else list(streams)
    T = w.T if T is None else T
    n = len(streams)
    tdt = np.float32 if w.dtype == "f32" else np.uint16
    out = {k: np.empty((n, T, w.d), dtype=tdt) for k in ("k", "v", "q")}
    for g in ("theta", "eta", "alpha"):
        out[g] = np.empty((n, T), dtype=np.float32)
    out["W0"] = np.empty((n, w.P), dtype=np.float32)
    out["S0"] = np.zeros((n, w.P), dtype=np.float32)

    def fill(i_s):
        i, s = i_s
        st = draw_stream(w, s, T, seed)
        for key in ("k", "v", "q", "theta", "eta", "alpha"):
            out[key][i] = st[key]

    # Each stream has its own generator, so streams can be drawn concurrently
    # (numpy releases the GIL inside its fill loops); the bytes do not depend
    # on the thread count.
    workers = min(n, os.cpu_count() or 1, 32)
    if workers > 1:
        with concurrent.futures.ThreadPoolExecutor(workers) as ex:
            list(ex.map(fill, enumerate(streams)))
    else:
        for i_s in enumerate(streams):
            fill(i_s)
    heads = {}
    for i, s in enumerate(streams):
        h = s % w.H
        if h not in heads:
            heads[h] = draw_w0_head(w, h, seed)
        out["W0"][i] = heads[h]
    out["streams"] = np.asarray(streams, dtype=np.int64)
    return out


def tokens_as_f64(x: np.ndarray, dtype: str) -> np.ndarray:
    """Exact float64 view of stored token values (bf16 bits or float32)."""
    if dtype == "f32":
        return np.asarray(x, dtype=np.float64)
    return bf16_bits_to_f64(x)
