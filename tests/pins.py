"""Independent references used to pin the oracle: brute-force matrix form and input builders.

Written from the definition of the scan (see the oracle's header), not from the
oracle's code: the matrix form sums every (t, s) pair with its decay exponent
taken term by term.
"""
import math

import numpy as np


def rand_params(rng, b, L, H, P, N, G, A_zero=False):
    x = rng.standard_normal((b, L, H, P))
    dt = np.log1p(np.exp(rng.standard_normal((b, L, H)) - 1.0))
    A = np.zeros(H) if A_zero else -np.exp(rng.uniform(0, math.log(16.0), H))
    B = rng.standard_normal((b, L, G, N)) / math.sqrt(N)
    C = rng.standard_normal((b, L, G, N)) / math.sqrt(N)
    D = rng.uniform(0, 1, H)
    return dict(x=x, dt=dt, A=A, B=B, C=C, D=D)


def matrix_form(p, direction):
    """Brute force: y_t = sum_s (C_t . B_s) exp(A * sum of dt strictly after s up to t) dt_s x_s + D x_t.

    Forward sums over s <= t with the decay exponent A * (dt_{s+1} + ... + dt_t);
    reverse sums over s >= t with A * (dt_t + ... + dt_{s-1}).  Each decay sum is
    taken term by term, no prefix sums.
    """
    x, dt, A, B, C, D = p["x"], p["dt"], p["A"], p["B"], p["C"], p.get("D")
    b, L, H, P = x.shape
    G = B.shape[2]
    y = np.zeros_like(x)
    for bi in range(b):
        for h in range(H):
            g = h // (H // G)
            for t in range(L):
                acc = np.zeros(P)
                srange = range(0, t + 1) if direction > 0 else range(t, L)
                for s in srange:
                    if direction > 0:
                        expo = sum(dt[bi, r, h] for r in range(s + 1, t + 1))
                    else:
                        expo = sum(dt[bi, r, h] for r in range(t, s))
                    coef = float(np.dot(C[bi, t, g], B[bi, s, g])) * math.exp(A[h] * expo) * dt[bi, s, h]
                    acc += coef * x[bi, s, h]
                if D is not None:
                    acc += D[h] * x[bi, t, h]
                y[bi, t, h] = acc
    return y
