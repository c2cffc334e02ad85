"""Float64 oracle of the step before the memory (test infrastructure only).

"Titans, explained", step 1 ("Project each token to a key and a value"): the
projections are followed by a short depthwise convolution, and keys and
queries are L2-normalised. Here, per stream (batch entry, head) and channel c:

    out[t, c] = sum_{j=0}^{w-1} f[h, c, j] * x[t - j, c]      (causal; x[t] for
                t < 0 comes from `history`, the last w-1 tokens of the previous
                call, or is zero)
    then, for keys and queries only, out[t] /= ||out[t]||_2   (whole row; a zero
                row stays zero)

Plain loops over the definition; only tests and the benchmark's CPU leg use it.
"""
from __future__ import annotations

import numpy as np


def conv_causal(x: np.ndarray, filt: np.ndarray, history: np.ndarray | None = None) -> np.ndarray:
    """x [T, d], filt [d, w], history [w-1, d] or None -> [T, d] (float64)."""
    x = np.asarray(x, dtype=np.float64)
    filt = np.asarray(filt, dtype=np.float64)
    T, d = x.shape
    w = filt.shape[1]
    hist = np.zeros((w - 1, d)) if history is None else np.asarray(history, dtype=np.float64)
    full = np.concatenate([hist, x], axis=0)          # row w-1+t is x[t]
    out = np.zeros((T, d))
    for t in range(T):
        for j in range(w):
            out[t] += filt[:, j] * full[w - 1 + t - j]
    return out


def l2_normalise_rows(x: np.ndarray) -> np.ndarray:
    x = np.asarray(x, dtype=np.float64)
    n = np.sqrt((x * x).sum(axis=-1, keepdims=True))
    return np.where(n > 0, x / np.where(n > 0, n, 1.0), 0.0)


def prologue(k, v, q, filt_k, filt_v, filt_q, hist_k=None, hist_v=None, hist_q=None):
    """One stream: returns (k', v', q') float64 [T, d]."""
    kk = l2_normalise_rows(conv_causal(k, filt_k, hist_k))
    vv = conv_causal(v, filt_v, hist_v)
    qq = l2_normalise_rows(conv_causal(q, filt_q, hist_q))
    return kk, vv, qq
