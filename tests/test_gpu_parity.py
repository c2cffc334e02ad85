"""GPU parity: libtitansmem against the float64 oracle on the same seeded inputs.

Tolerances (max normwise relative error per stream and per output tensor, each
layer of W and S separately): 1e-4 for fp32 arithmetic, 2e-2 for the bf16
tensor-core path.
"""
import numpy as np
import pytest
import torch

import oracle
from gen import workloads as W
from test_trained_neural_b200 import NeuralMemory

from gpu_util import gpu_to_np, parity_errors, run_lib, to_dev

pytestmark = pytest.mark.gpu

TOL_F32 = 1e-4
TOL_BF16_TC = 2e-2


def check(w: W.Workload, path: str, tol: float, streams=None, T=None):
    inp = W.generate(w, streams=streams, T=T)
    n = len(inp["streams"])
    B, H = (w.B, w.H) if n == w.streams else (1, n)
    Tn = inp["k"].shape[1]
    mem = NeuralMemory(w.L, w.d, w.expansion, path=path)
    dev = to_dev(inp, B, H, w.dtype)
    y, We, Se = run_lib(mem, dev, w.C)
    ref = oracle.run_workload(w, inp)
    errs = parity_errors(w.dims, inp["W0"], gpu_to_np(y, We, Se), ref)
    assert all(np.isfinite(v) for v in errs.values()), errs
    assert max(errs.values()) < tol, (w.name, path, Tn, errs)
    return errs


def test_linear_fp32_workload():
    """The linear fp32 workload in full (B=H=1, d=64, T=256, C=16)."""
    check(W.get(0), "auto", TOL_F32)


SMALL = [  # L, d, expansion, B, H, T, C
    (1, 16, 1, 1, 3, 48, 16),
    (1, 64, 1, 2, 1, 40, 8),
    (2, 16, 4, 1, 2, 64, 16),
    (2, 32, 4, 2, 2, 96, 32),
    (2, 64, 4, 1, 2, 128, 64),
    (2, 24, 3, 1, 1, 30, 10),      # ragged widths (72 hidden), odd chunk count
    (3, 16, 2, 1, 2, 48, 16),
    (4, 32, 2, 1, 2, 128, 64),
    (4, 16, 2, 2, 1, 40, 5),
    (2, 32, 4, 1, 2, 32, 1),       # C = 1: token-by-token descent
    (2, 32, 4, 1, 1, 128, 128),    # one chunk covers the whole stream
]


@pytest.mark.parametrize("cfg", SMALL, ids=lambda c: "L%d-d%d-e%d-B%dH%d-T%d-C%d" % c)
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("damped", [True, False], ids=["damped", "literal"])
def test_simt_small_shapes(cfg, dtype, damped):
    """Literal gates give large writes; the short streams here stay finite."""
    L, d, e, B, H, T, C = cfg
    extra = {} if damped else {"theta_damping": 1.0, "alpha_damping": 1.0}
    w = W.make(L, d, e, B, H, T, C, dtype=dtype, index=200 + sum(cfg), **extra)
    check(w, "simt", TOL_F32)


def test_simt_literal_gates_short_horizon():
    """The gates exactly as specified, over the horizon where the memory is
    still finite (a few chunks), on the README-shaped workload."""
    w = W.get_literal(1)
    check(w, "simt", TOL_F32, T=128)


def _dev_inputs(w, streams=None, T=None):
    inp = W.generate(w, streams=streams, T=T)
    n = len(inp["streams"])
    B, H = (w.B, w.H) if n == w.streams else (1, n)
    return inp, to_dev(inp, B, H, w.dtype)


@pytest.mark.parametrize("path", ["simt", "tc", "tcl"])
def test_in_place_state_equals_out_of_place(path):
    w = W.make(2, 64, 4, 1, 2, 256, 64, index=301)
    _, dev = _dev_inputs(w)
    mem = NeuralMemory(w.L, w.d, w.expansion, path=path)
    y1, We1, Se1 = run_lib(mem, dev, w.C)
    W0, S0 = dev["W0"].clone(), dev["S0"].clone()
    y2, We2, Se2 = mem.run(dev["k"], dev["v"], dev["q"], dev["theta"], dev["eta"], dev["alpha"],
                           W0, S0, w.C, W_end=W0, S_end=S0, sync=True)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2) and torch.equal(We1, W0) and torch.equal(Se1, S0)


@pytest.mark.parametrize("path", ["simt", "tc", "tcl"])
def test_state_carry_and_determinism(path):
    w = W.make(2, 64, 2, 2, 1, 384, 64, index=302)
    _, dev = _dev_inputs(w)
    mem = NeuralMemory(w.L, w.d, w.expansion, path=path)
    y, We, Se = run_lib(mem, dev, w.C)
    y_b, We_b, Se_b = run_lib(mem, dev, w.C)
    assert torch.equal(y, y_b) and torch.equal(We, We_b) and torch.equal(Se, Se_b)
    T1 = 128
    first = {k: (v[:, :, :T1].contiguous() if k in ("k", "v", "q", "theta", "eta", "alpha") else v)
             for k, v in dev.items()}
    ya, Wa, Sa = run_lib(mem, first, w.C)
    second = {k: (v[:, :, T1:].contiguous() if k in ("k", "v", "q", "theta", "eta", "alpha") else v)
              for k, v in dev.items()}
    second["W0"], second["S0"] = Wa, Sa
    yb, Wb, Sb = run_lib(mem, second, w.C)
    assert torch.equal(torch.cat([ya, yb], dim=2), y)
    assert torch.equal(Wb, We) and torch.equal(Sb, Se)


@pytest.mark.parametrize("shape", [(2, 128, 8, 2, 1, 256, 64), (4, 128, 2, 1, 2, 384, 128)],
                         ids=["split-K-hidden1024", "transposed-update-deep"])
def test_layered_runs_are_bit_identical(shape):
    """The split reduction adds its partial tiles in split order and the
    transposed update's chunks are fixed per warp: two runs (and a run split
    in two with the state carried) give the same bits."""
    L, d, e, B, H, T, C = shape
    w = W.make(L, d, e, B, H, T, C, index=330 + d + e)
    _, dev = _dev_inputs(w)
    mem = NeuralMemory(w.L, w.d, w.expansion, path="tcl")
    y, We, Se = run_lib(mem, dev, w.C)
    for _ in range(2):
        y_b, We_b, Se_b = run_lib(mem, dev, w.C)
        assert torch.equal(y, y_b) and torch.equal(We, We_b) and torch.equal(Se, Se_b)
    T1 = 2 * C
    first = {k: (v[:, :, :T1].contiguous() if k in ("k", "v", "q", "theta", "eta", "alpha") else v)
             for k, v in dev.items()}
    ya, Wa, Sa = run_lib(mem, first, w.C)
    second = {k: (v[:, :, T1:].contiguous() if k in ("k", "v", "q", "theta", "eta", "alpha") else v)
              for k, v in dev.items()}
    second["W0"], second["S0"] = Wa, Sa
    yb, Wb, Sb = run_lib(mem, second, w.C)
    assert torch.equal(torch.cat([ya, yb], dim=2), y)
    assert torch.equal(Wb, We) and torch.equal(Sb, Se)


@pytest.mark.parametrize("path", ["simt", "tc", "tcl"])
def test_streams_independent_and_permutable(path):
    w = W.make(2, 64, 1, 1, 4, 128, 64, index=303)
    inp, dev = _dev_inputs(w)
    mem = NeuralMemory(w.L, w.d, w.expansion, path=path)
    y, We, Se = run_lib(mem, dev, w.C)
    perm = torch.tensor([3, 1, 0, 2], device="cuda")
    pdev = {k: v[:, perm].contiguous() for k, v in dev.items()}
    yp, Wp, Sp = run_lib(mem, pdev, w.C)
    assert torch.equal(yp, y[:, perm]) and torch.equal(Wp, We[:, perm]) and torch.equal(Sp, Se[:, perm])


def test_gate_extremes_on_gpu():
    """alpha = 1 wipes (W_end = S_end up to rounding); theta = 0 writes nothing."""
    w = W.make(2, 32, 4, 1, 2, 64, 16, index=304)
    inp = W.generate(w)
    inp["alpha"][:] = 1.0
    dev = to_dev(inp, 1, 2, w.dtype)
    mem = NeuralMemory(w.L, w.d, w.expansion, path="simt")
    _, We, Se = run_lib(mem, dev, w.C)
    assert torch.allclose(We, Se, rtol=1e-6, atol=1e-7)
    inp = W.generate(w)
    inp["theta"][:] = 0.0
    dev = to_dev(inp, 1, 2, w.dtype)
    _, We, Se = run_lib(mem, dev, w.C)
    ref = oracle.run_workload(w, inp)
    errs = parity_errors(w.dims, inp["W0"], gpu_to_np(torch.zeros(1, 2, 64, 32, device="cuda"), We, Se),
                         {**ref, "y": np.zeros_like(ref["y"])})
    assert errs["W"] < TOL_F32 and errs["S"] < TOL_F32


# Full-size workloads, in the launch configuration the benchmark times, checked
# on outputs the oracle can afford: every output of the smaller workloads, and
# for the long ones the reads y of sampled streams over a prefix (the
# recurrence is causal, so a prefix run of the oracle gives the same y).
FULL = [(1, None, None), (2, None, None), (3, [0, 9], 2048), (4, [0, 37], 1024)]


@pytest.mark.parametrize("idx,sample_streams,prefix", FULL, ids=lambda x: str(x))
def test_full_size_workloads(idx, sample_streams, prefix):
    w = W.get(idx)
    inp = W.generate(w)
    dev = to_dev(inp, w.B, w.H, w.dtype)
    if sample_streams is not None:
        del inp
    mem = NeuralMemory(w.L, w.d, w.expansion, path="auto")
    tol = TOL_BF16_TC if mem.query_path(w.B, w.H, w.T, w.C) in ("tc", "tcl", "tcl-phased") else TOL_F32
    y, We, Se = run_lib(mem, dev, w.C)
    assert torch.isfinite(y).all() and torch.isfinite(We).all() and torch.isfinite(Se).all()
    if sample_streams is None:
        ref = oracle.run_workload(w, inp)
        errs = parity_errors(w.dims, inp["W0"], gpu_to_np(y, We, Se), ref)
        assert max(errs.values()) < tol, errs
    else:
        sub = W.generate(w, streams=sample_streams, T=prefix)
        ref = oracle.run_workload(w, sub)
        yf = y.reshape(w.streams, w.T, w.d)
        for i, s in enumerate(sample_streams):
            got = yf[s, :prefix].double().cpu().numpy()
            err = np.linalg.norm(got - ref["y"][i]) / np.linalg.norm(ref["y"][i])
            assert err < tol, (idx, s, err)


@pytest.mark.parametrize("idx,sample_streams,T", [(3, [0, 15], 1024), (4, [0, 63], 512)])
def test_all_streams_short_stream_state(idx, sample_streams, T):
    """Every stream of the long workloads over a shortened stream: the state
    (W_end, S_end) and reads of sampled streams against the oracle."""
    w = W.get(idx)
    inp = W.generate(w, T=T)
    dev = to_dev(inp, w.B, w.H, w.dtype)
    mem = NeuralMemory(w.L, w.d, w.expansion, path="auto")
    tol = TOL_BF16_TC if mem.query_path(w.B, w.H, T, w.C) in ("tc", "tcl", "tcl-phased") else TOL_F32
    y, We, Se = run_lib(mem, dev, w.C)
    gpu = gpu_to_np(y, We, Se)
    sub = {k: (v[sample_streams] if k != "streams" else v) for k, v in inp.items()}
    ref = oracle.run_workload(w, sub)
    gsub = {k: v[sample_streams] for k, v in gpu.items()}
    errs = parity_errors(w.dims, inp["W0"][sample_streams], gsub, ref)
    assert max(errs.values()) < tol, errs


# ---------------------------------------------------------------- tensor cores
TC_SHAPES = [  # d, expansion (hidden = 64 G), B, H, T
    (64, 1, 1, 1, 64),
    (64, 2, 1, 2, 192),
    (64, 4, 2, 2, 256),
    (128, 1, 1, 1, 128),
    (128, 2, 1, 1, 256),
    (128, 4, 1, 3, 320),
    (128, 4, 1, 1, 64),
]


@pytest.mark.parametrize("cfg", TC_SHAPES, ids=lambda c: "d%d-e%d-B%dH%d-T%d" % c)
def test_tc_small_shapes(cfg):
    d, e, B, H, T = cfg
    w = W.make(2, d, e, B, H, T, 64, index=400 + sum(cfg))
    mem = NeuralMemory(2, d, e)
    assert mem.query_path(B, H, T, 64) == "tc"
    check(w, "tc", TOL_BF16_TC)


@pytest.mark.parametrize("cfg", TC_SHAPES + [(128, 4, 1, 2, 256)], ids=lambda c: "d%d-e%d-B%dH%d-T%d" % c)
def test_tc_global_exchange_small_shapes(cfg):
    """The chunk walker with its CTAs exchanging through global memory (no
    cluster): against the oracle, and bit for bit against the cluster form
    (same bf16 partials, same fp32 summation order)."""
    d, e, B, H, T = cfg
    w = W.make(2, d, e, B, H, T, 64, index=420 + sum(cfg))
    check(w, "tc-global", TOL_BF16_TC)
    inp, dev = _dev_inputs(w)
    outs = {}
    for path in ("tc", "tc-global"):
        mem = NeuralMemory(2, d, e, path=path)
        outs[path] = gpu_to_np(*run_lib(mem, dev, w.C))
    for key in ("y", "W_end", "S_end"):
        np.testing.assert_array_equal(outs["tc"][key], outs["tc-global"][key], err_msg=key)


def test_tc_streams_beyond_resident_clusters():
    """16 streams of the long d=128 shape: 15 clusters of 8 fit at once, the
    16th stream runs beside them on the global-exchange walker. Every
    stream against the oracle, and the whole result bit for bit against the
    all-global form."""
    w = W.make(2, 128, 4, 1, 16, 256, 64, index=430)
    mem = NeuralMemory(2, 128, 4)
    assert mem.query_path(1, 16, 256, 64) == "tc"
    check(w, "tc", TOL_BF16_TC)
    inp, dev = _dev_inputs(w)
    outs = {}
    for path in ("tc", "tc-global"):
        m = NeuralMemory(2, 128, 4, path=path)
        outs[path] = gpu_to_np(*run_lib(m, dev, w.C))
    for key in ("y", "W_end", "S_end"):
        np.testing.assert_array_equal(outs["tc"][key], outs["tc-global"][key], err_msg=key)


def test_tc_cluster_of_eight_d128():
    """Hidden 512 split over a cluster of 8 CTAs (the long-stream shape)."""
    check(W.make(2, 128, 4, 1, 2, 256, 64, index=410), "tc", TOL_BF16_TC)


def test_tc_literal_gates_short_stream():
    """Gates exactly as specified over a finite horizon: large writes."""
    check(W.make(2, 64, 4, 1, 2, 128, 64, index=411, theta_damping=1.0, alpha_damping=1.0),
          "tc", TOL_BF16_TC)


def test_tc_matches_simt_path():
    w = W.make(2, 128, 4, 1, 2, 512, 64, index=412)
    inp, dev = _dev_inputs(w)
    out = {}
    for path in ("simt", "tc"):
        mem = NeuralMemory(2, 128, 4, path=path)
        out[path] = gpu_to_np(*run_lib(mem, dev, w.C))
    errs = parity_errors(w.dims, inp["W0"], out["tc"], out["simt"])
    assert max(errs.values()) < TOL_BF16_TC, errs


def test_tc_timeout_is_reported_and_context_survives():
    """A wait that nothing completes expires after 1 ms; the kernel records
    TM_ERR_TIMEOUT, cleans up and returns; the next call works."""
    from test_trained_neural_b200 import _native as N
    from test_trained_neural_b200._native import TitansMemError
    lib = N.load()
    w = W.make(2, 64, 2, 1, 2, 128, 64, index=413)
    inp, dev = _dev_inputs(w)
    mem = NeuralMemory(2, 64, 2, path="tc")
    assert lib.tm_set_debug(1, 1_000_000) == N.TM_OK
    try:
        with pytest.raises(TitansMemError) as ei:
            run_lib(mem, dev, w.C)
        assert ei.value.code == N.TM_ERR_TIMEOUT
    finally:
        lib.tm_set_debug(0, 0)
    y, We, Se = run_lib(mem, dev, w.C)
    ref = oracle.run_workload(w, inp)
    errs = parity_errors(w.dims, inp["W0"], gpu_to_np(y, We, Se), ref)
    assert max(errs.values()) < TOL_BF16_TC, errs


# ------------------------------------------------- layered tensor-core kernels
TCL_SHAPES = [  # L, d, expansion, B, H, T, C
    (1, 64, 1, 1, 2, 128, 64),      # linear memory
    (2, 64, 2, 1, 2, 256, 64),
    (2, 128, 3, 1, 1, 128, 64),     # hidden 384: 128-wide output tiles
    (2, 192, 2, 1, 1, 128, 64),     # d = 192: 64-wide tiles, partial M tiles
    (3, 64, 2, 2, 1, 256, 128),     # C = 128: two row tiles of keys and queries
    (4, 64, 2, 1, 2, 256, 128),
    (4, 128, 2, 1, 1, 256, 128),    # the deep workload's layer shapes
    (2, 64, 2, 1, 2, 384, 192),     # C = 192: a partial row tile in the backward
    (2, 128, 2, 1, 1, 512, 256),    # C = 256: four key/query row tiles, pipelined K loop
    (2, 64, 2, 3, 3, 256, 64),      # 9 streams: two concurrent groups of 4 and 5
    (4, 64, 2, 2, 4, 256, 128),     # 8 streams in two groups, depth 4
    (2, 128, 8, 1, 1, 128, 64),     # hidden 1024: the last forward's K = 1024 split over 4 CTAs per tile
]


@pytest.mark.parametrize("path", ["tcl", "tcl-phased"])
@pytest.mark.parametrize("cfg", TCL_SHAPES, ids=lambda c: "L%d-d%d-e%d-B%dH%d-T%d-C%d" % c)
def test_tcl_small_shapes(cfg, path):
    """Layered path; "tcl" runs the fused forward + backward kernel wherever
    every width is at most 256, "tcl-phased" one launch per phase."""
    L, d, e, B, H, T, C = cfg
    w = W.make(L, d, e, B, H, T, C, index=600 + sum(cfg))
    check(w, path, TOL_BF16_TC)


def test_tcl_fused_matches_phased():
    """The fused forward + backward kernel against the per-phase launches on
    the deep workload's layer shapes. Both round G to bf16 for the next MMA;
    the fused kernel forms -c G and -e G from that bf16 G (one more rounding,
    at most half a bf16 ulp per element) where the per-phase one scales the
    fp32 G, hence a bound a little above bf16 resolution."""
    w = W.make(4, 128, 2, 2, 2, 512, 128, index=630)
    inp, dev = _dev_inputs(w)
    out = {}
    for path in ("tcl", "tcl-phased"):
        mem = NeuralMemory(w.L, w.d, w.expansion, path=path)
        out[path] = gpu_to_np(*run_lib(mem, dev, w.C))
    errs = parity_errors(w.dims, inp["W0"], out["tcl"], out["tcl-phased"])
    assert max(errs.values()) < 5e-3, errs


def test_tcl_graph_replay_matches_direct_launches():
    """The layered path captures its launch sequence into a CUDA graph when a
    call repeats the previous one exactly, and replays it from then on: the
    replays give the direct launches' results bit for bit, and read the
    inputs' current contents (new data behind the same pointers)."""
    w = W.make(4, 64, 2, 4, 4, 384, 128, index=640)     # 16 streams: two concurrent groups
    _, dev = _dev_inputs(w)
    mem = NeuralMemory(w.L, w.d, w.expansion, path="tcl")
    y = torch.empty((w.B, w.H, w.T, w.d), dtype=torch.float32, device="cuda")
    We, Se = torch.empty_like(dev["W0"]), torch.empty_like(dev["S0"])
    ws = mem.alloc_workspace(w.B, w.H, w.T, w.C, dev["k"].dtype)
    call = lambda: mem.run(dev["k"], dev["v"], dev["q"], dev["theta"], dev["eta"], dev["alpha"], dev["W0"],
                           dev["S0"], w.C, y=y, W_end=We, S_end=Se, workspace=ws, sync=True)
    outs = []
    for _ in range(3):                                   # direct, capture + replay, replay
        y.fill_(float("nan"))
        call()
        torch.cuda.synchronize()
        outs.append((y.clone(), We.clone(), Se.clone()))
    for o in outs[1:]:
        assert all(torch.equal(a, b) for a, b in zip(o, outs[0]))
    dev["k"].copy_(torch.flip(dev["k"], dims=[2]))
    dev["alpha"].mul_(0.5)
    call()
    torch.cuda.synchronize()
    fresh = NeuralMemory(w.L, w.d, w.expansion, path="tcl")
    ref = run_lib(fresh, dev, w.C)
    assert all(torch.equal(a, b) for a, b in zip((y, We, Se), ref))
    assert not torch.equal(y, outs[0][0])


RAGGED = [  # L, d, expansion, B, H, T, C, dtype, path
    (1, 64, 1, 1, 1, 100, 16, "f32", "simt"),     # linear memory, 6 whole chunks + 4 tokens
    (2, 32, 4, 2, 1, 75, 32, "bf16", "simt"),
    (2, 64, 4, 1, 2, 209, 64, "bf16", "tc"),       # 3 whole chunks on the cluster kernel + 17
    (2, 64, 4, 1, 2, 40, 64, "bf16", "tc"),        # T < C: only the short chunk
    (4, 64, 2, 1, 2, 296, 128, "bf16", "tcl"),     # 2 whole chunks, fused layered kernels + 40
    (2, 128, 3, 1, 1, 150, 64, "bf16", "tcl"),     # per-phase layered kernels + 22
]


@pytest.mark.parametrize("cfg", RAGGED, ids=lambda c: "L%d-d%d-e%d-B%dH%d-T%d-C%d-%s-%s" % c)
def test_shorter_last_chunk(cfg):
    """C does not divide T: chunks start at multiples of C and the last one is
    shorter (the oracle's partial last chunk). The tensor-core paths run the
    whole chunks, then the short one on the CUDA-core kernel."""
    L, d, e, B, H, T, C, dt, path = cfg
    w = W.make(L, d, e, B, H, T, C, dtype=dt, index=640 + T)
    mem = NeuralMemory(L, d, e)
    assert mem.query_path(B, H, T, C, torch.bfloat16 if dt == "bf16" else torch.float32) == path
    check(w, path, TOL_F32 if dt == "f32" else TOL_BF16_TC)


def test_tcl_literal_gates_short_stream():
    check(W.make(2, 64, 2, 1, 2, 128, 64, index=620, theta_damping=1.0, alpha_damping=1.0),
          "tcl", TOL_BF16_TC)


def test_tcl_matches_cluster_kernel():
    """The two tensor-core designs on a shape both support."""
    w = W.make(2, 64, 4, 1, 2, 512, 64, index=621)
    inp, dev = _dev_inputs(w)
    out = {}
    for path in ("tc", "tcl"):
        mem = NeuralMemory(2, 64, 4, path=path)
        out[path] = gpu_to_np(*run_lib(mem, dev, w.C))
    errs = parity_errors(w.dims, inp["W0"], out["tcl"], out["tc"])
    assert max(errs.values()) < TOL_BF16_TC, errs




@pytest.mark.parametrize("path", ["tcl", "tcl-phased", "tcl-phased-split"])
def test_tcl_timeout_is_reported_and_context_survives(path):
    """The layered kernels' failure handling: with the test hook on, every CTA
    of the forward/backward (fused or per phase) and update kernels first
    waits on a barrier that nothing completes; the wait runs out after 1 ms,
    the kernel records TM_ERR_TIMEOUT, issues nothing further and returns.
    The next call on the same context (hook off) matches the oracle."""
    from test_trained_neural_b200 import _native as N
    from test_trained_neural_b200._native import TitansMemError
    lib = N.load()
    # "tcl": fused kernel and the update for 64-wide inputs; "tcl-phased": the
    # per-phase GEMMs and the transposed update; "-split": hidden 1024, whose
    # last forward splits K = 1024 over 4 CTAs per tile
    w = {"tcl": W.make(4, 64, 2, 1, 2, 256, 128, index=650),
         "tcl-phased": W.make(2, 128, 3, 1, 1, 128, 64, index=651),
         "tcl-phased-split": W.make(2, 128, 8, 1, 1, 128, 64, index=652)}[path]
    inp, dev = _dev_inputs(w)
    mem = NeuralMemory(w.L, w.d, w.expansion, path=path.replace("-split", ""))
    assert lib.tm_set_debug(1, 1_000_000) == N.TM_OK
    try:
        for _ in range(2):          # a repeated call goes through graph capture and replay
            with pytest.raises(TitansMemError) as ei:
                run_lib(mem, dev, w.C)
            assert ei.value.code == N.TM_ERR_TIMEOUT
    finally:
        lib.tm_set_debug(0, 0)
    y, We, Se = run_lib(mem, dev, w.C)
    ref = oracle.run_workload(w, inp)
    errs = parity_errors(w.dims, inp["W0"], gpu_to_np(y, We, Se), ref)
    assert max(errs.values()) < TOL_BF16_TC, errs


@pytest.mark.parametrize("idx,T", [(1, 128), (2, 128), (3, 128), (4, 256)])
def test_literal_gates_on_the_benchmark_path(idx, T):
    """Each MLP workload with its gates drawn exactly as specified (no
    damping), on the path the benchmark times, over a stream short enough
    that the memory is still finite: every stream against the oracle."""
    w = W.get_literal(idx)
    inp = W.generate(w, T=T)
    dev = to_dev(inp, w.B, w.H, w.dtype)
    mem = NeuralMemory(w.L, w.d, w.expansion, path="auto")
    assert mem.query_path(w.B, w.H, T, w.C) in ("tc", "tcl", "tcl-phased")
    y, We, Se = run_lib(mem, dev, w.C)
    ref = oracle.run_workload(w, inp)
    assert np.isfinite(ref["W_end"]).all() and np.isfinite(ref["y"]).all()
    errs = parity_errors(w.dims, inp["W0"], gpu_to_np(y, We, Se), ref)
    assert max(errs.values()) < TOL_BF16_TC, (w.name, errs)
