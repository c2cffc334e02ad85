"""The seeded input generator, and the gate-range reading of the MLP workloads."""
import numpy as np
import pytest

import oracle
from gen import workloads as W


def test_prefix_draws_match_full_draws():
    w = W.get(3)
    full = W.draw_stream(w, 5, T=3000)
    pre = W.draw_stream(w, 5, T=1100)
    for key in ("k", "v", "q", "theta", "eta", "alpha"):
        np.testing.assert_array_equal(pre[key], full[key][:1100])


def test_streams_and_heads_are_seeded_independently():
    w = W.get(2)
    a = W.generate(w, streams=[3, 11], T=256)
    b = W.generate(w, streams=[11], T=256)
    np.testing.assert_array_equal(a["k"][1], b["k"][0])
    assert not np.array_equal(a["k"][0], a["k"][1])
    # W0 is one draw per head, shared over the batch: streams 3 and 11 are head 3
    np.testing.assert_array_equal(a["W0"][0], a["W0"][1])


def test_keys_queries_normalised_and_bf16_rounding():
    w = W.get(1)
    x = W.generate(w, T=64)
    k = W.tokens_as_f64(x["k"], "bf16")
    assert np.allclose(np.linalg.norm(k, axis=-1), 1.0, atol=1e-2)
    f = np.array([1.0, 1.00390625, 1.0078125, -2.5, 3.14159], dtype=np.float32)
    b = W.bf16_bits_to_f64(W.f32_to_bf16_bits(f))
    np.testing.assert_array_equal(b[:3], [1.0, 1.0, 1.0078125])   # ties to even
    assert abs(b[4] - 3.140625) < 1e-12


def test_gate_ranges_and_damping():
    for i in (1, 2, 3, 4):
        lit, used = W.get_literal(i), W.get(i)
        assert used.theta_damping == W.MLP_THETA_DAMPING and used.alpha_damping == W.MLP_ALPHA_DAMPING
        a = W.draw_stream(lit, 0, T=1024)
        b = W.draw_stream(used, 0, T=1024)
        np.testing.assert_allclose(b["theta"], a["theta"] * W.MLP_THETA_DAMPING, rtol=1e-6)
        np.testing.assert_allclose(b["alpha"], a["alpha"] * W.MLP_ALPHA_DAMPING, rtol=1e-6)
        np.testing.assert_array_equal(b["eta"], a["eta"])
        assert lit.theta[0] <= a["theta"].min() and a["theta"].max() <= lit.theta[1]
    assert W.get(0).theta_damping == 1.0


@pytest.mark.parametrize("idx,T", [(2, 1024), (1, 1024)])
def test_literal_gates_make_mlp_memory_overflow(idx, T):
    """The reading behind the damped gates: with the gate ranges as specified,
    the float64 recurrence of a depth-2 memory leaves any finite range within
    a few hundred tokens, while the damped gates keep it finite and non-zero."""
    lit = W.get_literal(idx)
    r = oracle.run_workload(lit, W.generate(lit, streams=[0], T=T))
    assert not np.isfinite(r["W_end"]).all() or np.abs(r["W_end"]).max() > 1e30
    used = W.get(idx)
    r = oracle.run_workload(used, W.generate(used, streams=[0], T=T))
    assert np.isfinite(r["W_end"]).all() and np.isfinite(r["y"]).all()
    assert 1.0 < np.linalg.norm(r["W_end"]) < 1e3 and np.abs(r["y"]).max() > 1e-3


def test_linear_workload_stable_as_specified():
    w = W.get(0)
    r = oracle.run_workload(w, W.generate(w))
    assert np.isfinite(r["W_end"]).all() and np.abs(r["y"]).max() < 100
