"""The oracle's pins reject an oracle with a plausible mistake in it.

Each case plants one mistake in a copy of oracle/titans_oracle.c (a wrong
sign, a dropped factor, a transposed operand, an off-by-one chunk start, the
wrong weights for a read or a surprise, a wrong derivative), compiles it with
the oracle's own flags and runs a battery of the pins against it: at least one
pin must fail. The unmodified source, compiled the same way, must pass them
all, so the failures come from the planted mistakes."""
import os

import pytest

import oracle
from oracle import build as obuild

import test_golden as golden
import test_oracle_pins as pins

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
