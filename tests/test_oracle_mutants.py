"""The oracles' pins reject an oracle with a plausible mistake in it.

Each case plants one mistake in a copy of oracle/titans_oracle.c (a wrong
sign, a dropped factor, a transposed operand, an off-by-one chunk start, the
wrong weights for a read or a surprise, a wrong derivative), compiles it with
the oracle's own flags and runs a battery of the pins against it: at least one
pin must fail. The unmodified source, compiled the same way, must pass them
all, so the failures come from the planted mistakes. The second part does the
same for the prologue's oracle (oracle/prologue.py): taps, causality, history
order, the norm and which of k, v, q are normalised; the third for the
gradient oracle (oracle/backward.py), whose pins compare it with the C oracle
and with finite differences of the C oracle."""
import importlib.util
import os

import pytest

import oracle
from oracle import build as obuild

import test_backward_oracle as backward_pins
import test_golden as golden
import test_oracle_pins as pins
import test_prologue as prologue_pins

SRC = os.path.join(os.path.dirname(obuild.__file__), "titans_oracle.c")

MUTANTS = {  # name: (text in the oracle, text that replaces it)
    "momentum sign": ("S[i] = et * S[i] - th * u[i];", "S[i] = et * S[i] + th * u[i];"),
    "momentum decays the new surprise": ("S[i] = et * S[i] - th * u[i];", "S[i] = et * (S[i] - th * u[i]);"),
    "forget factor": ("W[i] = (1.0 - al) * W[i] + S[i];", "W[i] = (1.0 + al) * W[i] + S[i];"),
    "write subtracts the momentum": ("W[i] = (1.0 - al) * W[i] + S[i];", "W[i] = (1.0 - al) * W[i] - S[i];"),
    "write before the momentum update": (
        "for (size_t i = 0; i < P; ++i) S[i] = et * S[i] - th * u[i];\n"
        "    for (size_t i = 0; i < P; ++i) W[i] = (1.0 - al) * W[i] + S[i];",
        "for (size_t i = 0; i < P; ++i) W[i] = (1.0 - al) * W[i] + S[i];\n"
        "    for (size_t i = 0; i < P; ++i) S[i] = et * S[i] - th * u[i];"),
    "loss without the factor 2": ("g[i] = 2.0 * (xs[L][i] - v[i]);", "g[i] = (xs[L][i] - v[i]);"),
    "residual sign": ("g[i] = 2.0 * (xs[L][i] - v[i]);", "g[i] = 2.0 * (v[i] - xs[L][i]);"),
    "sigmoid' for silu'": ("return s * (1.0 + z * (1.0 - s));", "return s * (1.0 - s);"),
    "transposed weights in the backward": ("acc += Wl[(size_t)r * cols + c] * g[r];",
                                           "acc += Wl[(size_t)c * rows + r] * g[r];"),
    "silu after the last layer": ("xs[l][r] = (l < n->L) ? silu(acc) : acc;", "xs[l][r] = silu(acc);"),
    "chunk start one token late": ("if (t % C == 0) memcpy(Wf, W, sizeof(double) * P);",
                                   "if (t % C == 0 || t % C == 1) memcpy(Wf, W, sizeof(double) * P);"),
    "surprise at the current weights": ("forward(n, Wf, xs, zs);\n    surprise(n, Wf, xs, zs, vt, u, g, gn);",
                                        "forward(n, W, xs, zs);\n    surprise(n, W, xs, zs, vt, u, g, gn);"),
    "read at the current weights": ("forward(n, Wf, xs, zs);\n    memcpy(jb->y", "forward(n, W, xs, zs);\n    memcpy(jb->y"),
}


def battery():
    """Pins that between them exercise every line the mutants touch."""
    return [
        ("surprise vs autograd", lambda: pins.test_surprise_matches_autograd([3, 6, 5, 4])),
        ("C = 1 online descent", lambda: pins.test_chunk_size_one_is_online_descent_with_momentum([3, 4, 5, 3])),
        ("chunked recurrence", lambda: pins.test_chunked_recurrence_matches_autograd_restatement([3, 5, 4, 3], 5, 13)),
        ("reads see no write", pins.test_reads_see_no_write_of_their_own_chunk),
        ("exact rational tiny", pins.test_brute_force_rational_tiny),
        ("exact worked example", golden.test_oracle_matches_exact_example),
    ]


def failures_with(lib_path):
    failed = []
    with oracle.use_library(lib_path):
        for name, pin in battery():
            try:
                pin()
            except AssertionError:
                failed.append(name)
    return failed


def build_variant(tmp_path, old=None, new=None):
    src = open(SRC).read()
    if old is not None:
        assert src.count(old) == 1, old
        src = src.replace(old, new)
    path = tmp_path / "variant.c"
    path.write_text(src)
    return obuild.compile_source(str(path), str(tmp_path / "libvariant.so"))


def test_unmodified_oracle_passes_the_battery(tmp_path):
    assert failures_with(build_variant(tmp_path)) == []


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_fails_a_pin(tmp_path, name):
    old, new = MUTANTS[name]
    assert failures_with(build_variant(tmp_path, old, new)), name


# ---------------------------------------------------------------- prologue oracle

PRO_SRC = os.path.join(os.path.dirname(obuild.__file__), "prologue.py")

PRO_MUTANTS = {
    "taps reversed": ("out[t] += filt[:, j] * full[w - 1 + t - j]", "out[t] += filt[:, w - 1 - j] * full[w - 1 + t - j]"),
    "looks ahead": ("out[t] += filt[:, j] * full[w - 1 + t - j]", "out[t] += filt[:, j] * full[min(w - 1 + t + j, T + w - 2)]"),
    "history after the tokens": ("full = np.concatenate([hist, x], axis=0)", "full = np.concatenate([x, hist], axis=0)"),
    "norm without the square root": ("n = np.sqrt((x * x).sum(axis=-1, keepdims=True))", "n = (x * x).sum(axis=-1, keepdims=True)"),
    "norm over tokens": ("n = np.sqrt((x * x).sum(axis=-1, keepdims=True))", "n = np.sqrt((x * x).sum(axis=0, keepdims=True))"),
    "values normalised": ("vv = conv_causal(v, filt_v, hist_v)", "vv = l2_normalise_rows(conv_causal(v, filt_v, hist_v))"),
    "keys not normalised": ("kk = l2_normalise_rows(conv_causal(k, filt_k, hist_k))", "kk = conv_causal(k, filt_k, hist_k)"),
}


def prologue_battery():
    return [
        ("numpy convolve", prologue_pins.test_conv_matches_numpy_convolve),
        ("delta and shift", prologue_pins.test_delta_and_shift_filters),
        ("history", prologue_pins.test_history_equals_one_long_sequence),
        ("normalisation", prologue_pins.test_normalisation),
        ("keys and queries only", prologue_pins.test_prologue_normalises_keys_and_queries_only),
    ]


def prologue_failures(tmp_path, old=None, new=None, monkeypatch=None):
    src = open(PRO_SRC).read()
    if old is not None:
        assert src.count(old) == 1, old
        src = src.replace(old, new)
    path = tmp_path / "prologue_variant.py"
    path.write_text(src)
    spec = importlib.util.spec_from_file_location("prologue_variant", str(path))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    monkeypatch.setattr(prologue_pins, "P", mod)
    failed = []
    for name, pin in prologue_battery():
        try:
            pin()
        except (AssertionError, IndexError, ValueError):
            failed.append(name)
    return failed


def test_unmodified_prologue_oracle_passes_the_battery(tmp_path, monkeypatch):
    assert prologue_failures(tmp_path, monkeypatch=monkeypatch) == []


@pytest.mark.parametrize("name", sorted(PRO_MUTANTS))
def test_planted_prologue_mistake_fails_a_pin(tmp_path, monkeypatch, name):
    old, new = PRO_MUTANTS[name]
    assert prologue_failures(tmp_path, old, new, monkeypatch=monkeypatch), name


# ---------------------------------------------------------------- gradient oracle

BW_SRC = os.path.join(os.path.dirname(obuild.__file__), "backward.py")

BW_MUTANTS = {
    "silu' sign": ("return s * (1 + z * (1 - s))", "return s * (1 - z * (1 - s))"),
    "surprise without the factor 2": ("g = 2 * (xs[-1] - v)", "g = xs[-1] - v"),
    "outer product transposed": ("us[l] = torch.outer(g, xs[l])", "us[l] = torch.outer(g, xs[l]).T.reshape(g.shape[0], -1)"),
    "momentum without eta": ("S = [eta[t] * s - theta[t] * ul for s, ul in zip(S, u)]",
                             "S = [s - theta[t] * ul for s, ul in zip(S, u)]"),
    "reads at the current weights": ("ys.append(_forward(Wf, q[t])[1][-1])", "ys.append(_forward(W, q[t])[1][-1])"),
    "dS_end dropped from J": ("(Se * torch.as_tensor(dS_end, dtype=torch.float64)).sum()", "0.0 * Se.sum()"),
}


def backward_battery():
    c2, c4 = backward_pins.CASES[1], backward_pins.CASES[3]
    return [
        ("forward = C oracle (depth 2)", lambda: backward_pins.test_forward_restatement_equals_c_oracle(c2)),
        ("forward = C oracle (depth 4)", lambda: backward_pins.test_forward_restatement_equals_c_oracle(c4)),
        ("finite differences (depth 2)", lambda: backward_pins.test_gradients_equal_finite_differences_of_c_oracle(c2)),
    ]


def backward_failures(tmp_path, monkeypatch, old=None, new=None):
    src = open(BW_SRC).read()
    if old is not None:
        assert src.count(old) == 1, old
        src = src.replace(old, new)
    path = tmp_path / "backward_variant.py"
    path.write_text(src)
    spec = importlib.util.spec_from_file_location("backward_variant", str(path))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    monkeypatch.setattr(backward_pins, "BW", mod)
    failed = []
    for name, pin in backward_battery():
        try:
            pin()
        except (AssertionError, RuntimeError, ValueError):
            failed.append(name)
    return failed


def test_unmodified_gradient_oracle_passes_the_battery(tmp_path, monkeypatch):
    assert backward_failures(tmp_path, monkeypatch) == []


@pytest.mark.parametrize("name", sorted(BW_MUTANTS))
def test_planted_gradient_oracle_mistake_fails_a_pin(tmp_path, monkeypatch, name):
    old, new = BW_MUTANTS[name]
    assert backward_failures(tmp_path, monkeypatch, old, new), name
