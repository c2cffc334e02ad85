"""Writes linear_d4_T5_C2.txt: a worked example of the linear memory in exact
rational arithmetic.

The pages print no numeric example, so this one is computed here, exactly,
from the update rules as the pages state them, with no floating point and
without the oracle or the library:
  surprise   u_t = 2 (W_frz k_t - v_t) k_t^T      ("Titans, explained", step 2
             "Measure surprise": the gradient of ||M(k) - v||^2 for M(x) = W x)
  momentum   S_t = eta_t S_{t-1} - theta_t u_t    (step 3 "Accumulate surprise
             with momentum")
  forget     W_t = (1 - alpha_t) W_{t-1} + S_t    (step 4 "Forget, then write")
  read       y_t = W_frz q_t                      (step 5 "Read without writing")
where W_frz is the state after the last token of the previous chunk ("Attack
of the Titans", section "Parallel training": gradients at the chunk-start
weights). d = 4, T = 5, C = 2: two whole chunks and a last chunk of one token.
Every input is a dyadic rational with a small denominator, so float32 holds it
exactly.

Run from the repository root: python tests/golden/make_linear_exact.py
"""
from __future__ import annotations

import os
from fractions import Fraction as F

D, T, C = 4, 5, 2
HERE = os.path.dirname(os.path.abspath(__file__))
OUT = os.path.join(HERE, "linear_d4_T5_C2.txt")


def inputs():
    k = [[F((3 * t + 5 * j) % 7 - 3, 8) for j in range(D)] for t in range(T)]
    v = [[F((2 * t + 3 * j) % 5 - 2, 4) for j in range(D)] for t in range(T)]
    q = [[F((5 * t + j) % 6 - 2, 8) for j in range(D)] for t in range(T)]
    theta = [F(1, 16), F(1, 8), F(3, 32), F(1, 4), F(1, 32)]
    eta = [F(1, 2), F(3, 4), F(7, 8), F(1, 4), F(5, 8)]
    alpha = [F(0), F(1, 8), F(1, 16), F(1, 4), F(3, 16)]
    W0 = [[F((i * 3 + j) % 5 - 2, 8) for j in range(D)] for i in range(D)]
    S0 = [[F(1, 16) if i == j else F(0) for j in range(D)] for i in range(D)]
    return dict(k=k, v=v, q=q, theta=theta, eta=eta, alpha=alpha, W0=W0, S0=S0)


def run(x):
    W = [row[:] for row in x["W0"]]
    S = [row[:] for row in x["S0"]]
    ys = []
    for t in range(T):
        if t % C == 0:
            Wf = [row[:] for row in W]
        k, v, q = x["k"][t], x["v"][t], x["q"][t]
        r = [sum(Wf[i][j] * k[j] for j in range(D)) - v[i] for i in range(D)]
        S = [[x["eta"][t] * S[i][j] - x["theta"][t] * 2 * r[i] * k[j] for j in range(D)] for i in range(D)]
        W = [[(1 - x["alpha"][t]) * W[i][j] + S[i][j] for j in range(D)] for i in range(D)]
        ys.append([sum(Wf[i][j] * q[j] for j in range(D)) for i in range(D)])
    return ys, W, S


def flat(a):
    out = []
    for e in a:
        out.extend(flat(e) if isinstance(e, list) else [e])
    return out


def main():
    x = inputs()
    y, W, S = run(x)
    lines = ["# Linear memory, d = 4, T = 5, C = 2, exact rationals (written by make_linear_exact.py).",
             "# Matrices row-major: k, v, q, y [T x d]; W0, S0, W_end, S_end [d x d]; gates [T]."]
    for name in ("k", "v", "q", "theta", "eta", "alpha", "W0", "S0"):
        lines.append(name + " " + " ".join(str(e) for e in flat(x[name])))
    for name, val in (("y", y), ("W_end", W), ("S_end", S)):
        lines.append(name + " " + " ".join(str(e) for e in flat(val)))
    with open(OUT, "w") as f:
        f.write("\n".join(lines) + "\n")


if __name__ == "__main__":
    main()
