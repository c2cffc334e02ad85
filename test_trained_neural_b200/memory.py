"""Python front end of libtitansmem: the neural long-term memory write-and-read.

``NeuralMemory(L, d_h, expansion).run(...)`` hands torch CUDA tensors to the C
ABI ``tm_run``; torch only supplies device memory and the stream.
"""
from __future__ import annotations

import ctypes

import torch

from . import _native as N


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr())


class NeuralMemory:
    """A context for memories of depth L, head dim d_h, hidden = expansion * d_h."""

    def __init__(self, L: int, d_h: int, expansion: int = 4, path: str = "auto"):
        self._lib = N.load()
        h = ctypes.c_void_p()
        N.check(self._lib.tm_create(L, d_h, expansion, N.TM_ACT_SILU, ctypes.byref(h)), "tm_create")
        self._h = h
        self.L, self.d_h, self.expansion = L, d_h, expansion
        self.P = int(self._lib.tm_param_count(h))
        self.set_path(path)

    def close(self):
        if getattr(self, "_h", None) is not None and self._h.value:
            self._lib.tm_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def set_path(self, path: str) -> None:
        code = {"auto": N.TM_PATH_AUTO, "simt": N.TM_PATH_SIMT, "tc": N.TM_PATH_TC,
                "tcl": N.TM_PATH_TC_LAYERED, "tcl-phased": N.TM_PATH_TC_PHASED,
                "tc-global": N.TM_PATH_TC_GLOBAL}[path]
        N.check(self._lib.tm_set_path(self._h, code), "tm_set_path")
        self.path = path

    @staticmethod
    def _dtype_code(t: torch.Tensor) -> int:
        if t.dtype == torch.bfloat16:
            return N.TM_BF16
        if t.dtype == torch.float32:
            return N.TM_F32
        raise TypeError(f"k/v/q must be float32 or bfloat16, got {t.dtype}")

    def query_path(self, B, H, T, C, dtype=torch.bfloat16) -> str:
        out = ctypes.c_int()
        code = N.TM_BF16 if dtype == torch.bfloat16 else N.TM_F32
        N.check(self._lib.tm_query_path(self._h, B, H, T, C, code, ctypes.byref(out)), "tm_query_path")
        return {N.TM_PATH_SIMT: "simt", N.TM_PATH_TC: "tc", N.TM_PATH_TC_LAYERED: "tcl",
                N.TM_PATH_TC_PHASED: "tcl-phased", N.TM_PATH_TC_GLOBAL: "tc-global"}[out.value]

    def launch_count(self, B, H, T, C, dtype=torch.bfloat16) -> int:
        """Kernel launches one run() of this problem makes."""
        out = ctypes.c_longlong()
        code = N.TM_BF16 if dtype == torch.bfloat16 else N.TM_F32
        N.check(self._lib.tm_launch_count(self._h, B, H, T, C, code, ctypes.byref(out)), "tm_launch_count")
        return int(out.value)

    def workspace_size(self, B, H, T, C, dtype=torch.bfloat16) -> int:
        out = ctypes.c_size_t()
        code = N.TM_BF16 if dtype == torch.bfloat16 else N.TM_F32
        N.check(self._lib.tm_workspace_size(self._h, B, H, T, C, code, ctypes.byref(out)),
                "tm_workspace_size")
        return int(out.value)

    def alloc_workspace(self, B, H, T, C, dtype=torch.bfloat16, device="cuda") -> torch.Tensor:
        n = self.workspace_size(B, H, T, C, dtype)
        return torch.empty(n, dtype=torch.uint8, device=device)

    def run(self, k, v, q, theta, eta, alpha, W0, S0, C, y=None, W_end=None, S_end=None,
            workspace=None, stream=None, sync=False):
        """Write-and-read over T tokens for B*H streams.

        k, v, q: [B, H, T, d_h] float32 or bfloat16 CUDA tensors; gates [B, H, T]
        float32; W0, S0 [B, H, P] float32. Returns (y, W_end, S_end); pass
        W_end=W0 / S_end=S0 to update in place.
        """
        B, H, T, d = k.shape
        dt = self._dtype_code(k)
        for t in (k, v, q, theta, eta, alpha, W0, S0):
            if not t.is_cuda or not t.is_contiguous():
                raise ValueError("all tensors must be contiguous CUDA tensors")
        if y is None:
            y = torch.empty((B, H, T, d), dtype=torch.float32, device=k.device)
        if W_end is None:
            W_end = torch.empty_like(W0)
        if S_end is None:
            S_end = torch.empty_like(S0)
        if workspace is None:
            workspace = self.alloc_workspace(B, H, T, C, k.dtype, k.device)
        if stream is None:
            stream = torch.cuda.current_stream(k.device)
        code = self._lib.tm_run(self._h, B, H, T, C, dt, _ptr(k), _ptr(v), _ptr(q), _ptr(theta),
                                _ptr(eta), _ptr(alpha), _ptr(W0), _ptr(S0), _ptr(y), _ptr(W_end),
                                _ptr(S_end), _ptr(workspace), workspace.numel(),
                                ctypes.c_void_p(stream.cuda_stream))
        N.check(code, "tm_run")
        if sync:
            self.sync(workspace, stream)
        return y, W_end, S_end

    def host_workspace_size(self, B, H, T, C, dtype=torch.bfloat16, segment_tokens=0) -> int:
        out = ctypes.c_size_t()
        code = N.TM_BF16 if dtype == torch.bfloat16 else N.TM_F32
        N.check(self._lib.tm_host_workspace_size(self._h, B, H, T, C, code, int(segment_tokens),
                                                 ctypes.byref(out)), "tm_host_workspace_size")
        return int(out.value)

    def run_host(self, k, v, q, theta, eta, alpha, W0, S0, C, y=None, W_end=None, S_end=None,
                 workspace=None, segment_tokens=0, stream=None, sync=True):
        """run() with every input and output in host memory (CPU tensors,
        pinned for the copies to overlap the kernels): the library copies the
        segments in and out itself, overlapped with the kernels. Returns
        (y, W_end, S_end) as CPU tensors; with sync=False they are complete
        once `stream` reaches this point."""
        B, H, T, d = k.shape
        dt = self._dtype_code(k)
        for t in (k, v, q, theta, eta, alpha, W0, S0):
            if t.is_cuda or not t.is_contiguous():
                raise ValueError("run_host takes contiguous CPU tensors")
        pin = k.is_pinned()
        if y is None:
            y = torch.empty((B, H, T, d), dtype=torch.float32, pin_memory=pin)
        if W_end is None:
            W_end = torch.empty_like(W0, pin_memory=pin)
        if S_end is None:
            S_end = torch.empty_like(S0, pin_memory=pin)
        dev = torch.device("cuda", torch.cuda.current_device())
        if workspace is None:
            n = self.host_workspace_size(B, H, T, C, k.dtype, segment_tokens)
            workspace = torch.empty(n, dtype=torch.uint8, device=dev)
        if stream is None:
            stream = torch.cuda.current_stream(dev)
        code = self._lib.tm_run_host(self._h, B, H, T, C, dt, _ptr(k), _ptr(v), _ptr(q), _ptr(theta),
                                     _ptr(eta), _ptr(alpha), _ptr(W0), _ptr(S0), _ptr(y), _ptr(W_end),
                                     _ptr(S_end), int(segment_tokens), _ptr(workspace), workspace.numel(),
                                     ctypes.c_void_p(stream.cuda_stream))
        N.check(code, "tm_run_host")
        if sync:
            self.sync(workspace, stream)
        return y, W_end, S_end

    def decode_step(self, k, v, q, theta, eta, alpha, W, S, y=None, stream=None):
        """One token per stream (k, v, q [B, H, d_h]; gates [B, H]): returns
        y = M_W(q) and updates W, S ([B, H, P] float32) in place."""
        B, H, d = k.shape
        if y is None:
            y = torch.empty((B, H, d), dtype=torch.float32, device=k.device)
        if stream is None:
            stream = torch.cuda.current_stream(k.device)
        code = self._lib.tm_decode_step(self._h, B, H, self._dtype_code(k), _ptr(k), _ptr(v), _ptr(q),
                                        _ptr(theta), _ptr(eta), _ptr(alpha), _ptr(W), _ptr(S), _ptr(y),
                                        ctypes.c_void_p(stream.cuda_stream))
        N.check(code, "tm_decode_step")
        return y

    def backward(self, k, v, q, theta, eta, alpha, W0, S0, dy, dW_end, dS_end, C, stream=None, workspace=None):
        """Gradients of sum <dy, y> + <dW_end, W_end> + <dS_end, S_end> for the
        run with these inputs (any depth). Returns a dict of float32 tensors dk,
        dv, dq, dtheta, deta, dalpha, dW0, dS0. With a caller's workspace (uint8,
        at least backward_workspace_size bytes), sync(workspace) then reports
        the call's device-side status."""
        B, H, T, d = k.shape
        dt = self._dtype_code(k)
        if workspace is None:
            workspace = torch.empty(self.backward_workspace_size(B, H, T, C, k.dtype), dtype=torch.uint8,
                                    device=k.device)
        ws = workspace
        f32 = dict(dtype=torch.float32, device=k.device)
        out = {"dk": torch.empty((B, H, T, d), **f32), "dv": torch.empty((B, H, T, d), **f32),
               "dq": torch.empty((B, H, T, d), **f32), "dtheta": torch.empty((B, H, T), **f32),
               "deta": torch.empty((B, H, T), **f32), "dalpha": torch.empty((B, H, T), **f32),
               "dW0": torch.empty_like(W0), "dS0": torch.empty_like(S0)}
        if stream is None:
            stream = torch.cuda.current_stream(k.device)
        code = self._lib.tm_backward(
            self._h, B, H, T, C, dt, _ptr(k), _ptr(v), _ptr(q), _ptr(theta), _ptr(eta), _ptr(alpha), _ptr(W0),
            _ptr(S0), _ptr(dy), _ptr(dW_end), _ptr(dS_end), _ptr(out["dk"]), _ptr(out["dv"]), _ptr(out["dq"]),
            _ptr(out["dtheta"]), _ptr(out["deta"]), _ptr(out["dalpha"]), _ptr(out["dW0"]), _ptr(out["dS0"]),
            _ptr(ws), ws.numel(), ctypes.c_void_p(stream.cuda_stream))
        N.check(code, "tm_backward")
        return out

    def backward_workspace_size(self, B, H, T, C, dtype) -> int:
        n = ctypes.c_size_t()
        dt = N.TM_BF16 if dtype == torch.bfloat16 else N.TM_F32
        N.check(self._lib.tm_backward_workspace_size(self._h, B, H, T, C, dt, ctypes.byref(n)),
                "tm_backward_workspace_size")
        return int(n.value)

    def sync(self, workspace, stream=None):
        if stream is None:
            stream = torch.cuda.current_stream(workspace.device)
        N.check(self._lib.tm_sync(self._h, _ptr(workspace), ctypes.c_void_p(stream.cuda_stream)),
                "tm_sync")


def prologue(k, v, q, filt_k, filt_v, filt_q, hist=None, out=None, stream=None):
    """Depthwise causal convolution of k, v, q ([B, H, T, d], float32 or
    bfloat16, CUDA) with per-head filters [H, d, width] (float32), then L2
    normalisation of the key and query rows. hist: optional (hk, hv, hq)
    [B, H, width-1, d] tails of the previous call. Returns (k', v', q')."""
    lib = N.load()
    B, H, T, d = k.shape
    width = filt_k.shape[-1]
    dt = N.TM_BF16 if k.dtype == torch.bfloat16 else N.TM_F32
    if out is None:
        out = (torch.empty_like(k), torch.empty_like(v), torch.empty_like(q))
    hk, hv, hq = hist if hist is not None else (None, None, None)
    hp = lambda t: None if t is None else _ptr(t)
    if stream is None:
        stream = torch.cuda.current_stream(k.device)
    code = lib.tm_prologue(B, H, T, d, width, dt, _ptr(k), _ptr(v), _ptr(q), _ptr(filt_k),
                           _ptr(filt_v), _ptr(filt_q), hp(hk), hp(hv), hp(hq), _ptr(out[0]),
                           _ptr(out[1]), _ptr(out[2]), ctypes.c_void_p(stream.cuda_stream))
    N.check(code, "tm_prologue")
    return out
