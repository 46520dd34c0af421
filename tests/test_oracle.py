"""Pins for the float64 oracle (CPU only).

Every check here ties the oracle to something other than itself: a value
worked by hand, the explicit semiseparable-matrix sum computed by brute
force, a closed form (cumulative sum, geometric series, impulse response),
or an identity of the recurrence (reverse = flip . forward . flip,
linearity in x, chunk-size invariance of the chunked form).
"""
import json
import math
import os

import numpy as np
import pytest

import oracle
import ssd_inputs as si
from pins import matrix_form as _matrix_form, rand_params as _rand_params

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _scan(p, direction, **kw):
    return oracle.ssd_scan_f64(p["x"], p["dt"], p["A"], p["B"], p["C"], p.get("D"), direction, **kw)


# ----------------------------------------------------------------- golden

def test_golden_handworked():
    g = json.load(open(os.path.join(GOLDEN, "ssd_handworked_L3.json")))
    p = dict(x=np.array(g["x"])[None, :, None, :], dt=np.array(g["dt"])[None, :, None],
             A=np.array(g["A"]), B=np.array(g["B"])[None, :, None, :],
             C=np.array(g["C"])[None, :, None, :], D=np.array(g["D"]))
    tol = g["tolerance"]
    yf = _scan(p, 1)[0, :, 0, :]
    yr = _scan(p, -1)[0, :, 0, :]
    np.testing.assert_allclose(yf, g["y_forward"], rtol=0, atol=tol)
    np.testing.assert_allclose(yr, g["y_reverse"], rtol=0, atol=tol)
    yb = oracle.bidir_f64(p, p)[0, :, 0, :]
    np.testing.assert_allclose(yb, g["y_bidirectional"], rtol=0, atol=tol)
    res = np.array(g["residual"])[None]
    out = oracle.r2l_block_f64(p, g["gate_s"], res)[0]
    np.testing.assert_allclose(out, g["r2l_out"], rtol=0, atol=tol)


# ------------------------------------------------------------ matrix form

@pytest.mark.parametrize("direction", [1, -1])
def test_matrix_form_tiny_workload(direction):
    """The tiny fp32 workload (b1 L64 H2 P16 N16), exact stored inputs, both directions."""
    shape = si.WORKLOADS["tiny_f32"]["shape"]
    pf, pr = si.make_bidir(shape, seed=0)
    p = oracle.params_f64(pf if direction > 0 else pr)
    y = _scan(p, direction)
    ref = _matrix_form(p, direction)
    assert oracle.rel_err(y, ref) <= 1e-12


@pytest.mark.parametrize("direction", [1, -1])
def test_matrix_form_groups_ragged(direction):
    """Two groups over four heads (head h uses group h // 2), odd length, no D."""
    rng = np.random.default_rng(7)
    p = _rand_params(rng, 2, 13, 4, 3, 5, 2)
    p["D"] = None
    assert oracle.rel_err(_scan(p, direction), _matrix_form(p, direction)) <= 1e-12


# ----------------------------------------------------------- closed forms

def test_A_zero_is_cumulative_sum():
    """A = 0: the state is the running sum of dt x (outer) B, so y_t = C_t . cumsum + D x_t."""
    rng = np.random.default_rng(1)
    p = _rand_params(rng, 2, 40, 3, 4, 6, 1, A_zero=True)
    outer = p["dt"][..., None, None] * p["x"][..., :, None] * p["B"][:, :, 0][:, :, None, None, :]
    Sc = np.cumsum(outer, axis=1)                                    # [b, L, H, P, N]
    ref = np.einsum("blhpn,bln->blhp", Sc, p["C"][:, :, 0]) + p["D"][None, None, :, None] * p["x"]
    assert oracle.rel_err(_scan(p, 1), ref) <= 1e-12
    Sr = np.cumsum(outer[:, ::-1], axis=1)[:, ::-1]
    ref_r = np.einsum("blhpn,bln->blhp", Sr, p["C"][:, :, 0]) + p["D"][None, None, :, None] * p["x"]
    assert oracle.rel_err(_scan(p, -1), ref_r) <= 1e-12


def test_scalar_state_is_plain_cumsum():
    """N = 1, B = C = 1, A = 0, D = 0: the scan is the textbook cumulative sum of dt * x."""
    rng = np.random.default_rng(2)
    L = 50
    x = rng.standard_normal((1, L, 1, 1)); dt = rng.uniform(0.1, 1.0, (1, L, 1))
    ones = np.ones((1, L, 1, 1))
    p = dict(x=x, dt=dt, A=np.zeros(1), B=ones, C=ones, D=None)
    np.testing.assert_allclose(_scan(p, 1)[0, :, 0, 0], np.cumsum(dt[0, :, 0] * x[0, :, 0, 0]),
                               rtol=1e-13, atol=1e-13)


def test_geometric_series():
    """Constant dt and x, B = C = e1, D = 0: y_t = dt x (1 - a^(t+1)) / (1 - a), a = exp(dt A)."""
    L, dtv, xv, Av = 60, 0.3, 1.7, -2.5
    e1 = np.zeros((1, L, 1, 4)); e1[..., 0] = 1.0
    p = dict(x=np.full((1, L, 1, 1), xv), dt=np.full((1, L, 1), dtv), A=np.array([Av]),
             B=e1, C=e1, D=None)
    a = math.exp(dtv * Av)
    ref = np.array([dtv * xv * (1 - a ** (t + 1)) / (1 - a) for t in range(L)])
    np.testing.assert_allclose(_scan(p, 1)[0, :, 0, 0], ref, rtol=1e-13)
    np.testing.assert_allclose(_scan(p, -1)[0, :, 0, 0], ref[::-1], rtol=1e-13)


def test_impulse_response():
    """x nonzero only at s0: y_t = dt_s0 (C_t . B_s0) exp(A sum_{s0<r<=t} dt_r) x_s0 for t >= s0, else 0."""
    rng = np.random.default_rng(3)
    p = _rand_params(rng, 1, 30, 1, 2, 8, 1)
    s0 = 11
    x = np.zeros_like(p["x"]); x[0, s0, 0] = [1.25, -0.5]; p["x"] = x
    y = _scan(p, 1)[0, :, 0]
    dt, A, B, C, D = p["dt"][0, :, 0], p["A"][0], p["B"][0, :, 0], p["C"][0, :, 0], p["D"][0]
    for t in range(30):
        if t < s0:
            ref = np.zeros(2)
        else:
            ref = dt[s0] * float(C[t] @ B[s0]) * math.exp(A * dt[s0 + 1:t + 1].sum()) * x[0, s0, 0]
            if t == s0:
                ref = ref + D * x[0, s0, 0]
        np.testing.assert_allclose(y[t], ref, rtol=1e-12, atol=1e-15)


def test_single_token():
    rng = np.random.default_rng(4)
    p = _rand_params(rng, 3, 1, 2, 4, 8, 1)
    ref = (p["dt"][..., None] * np.einsum("bgn,bgn->bg", p["C"][:, 0], p["B"][:, 0])[:, None, :, None]
           * p["x"] + p["D"][None, None, :, None] * p["x"])
    for d in (1, -1):
        assert oracle.rel_err(_scan(p, d), ref) <= 1e-14


def test_dt_zero_gives_skip_term_exactly():
    rng = np.random.default_rng(5)
    p = _rand_params(rng, 2, 9, 2, 4, 4, 1)
    p["dt"] = np.zeros_like(p["dt"])
    for d in (1, -1):
        assert np.array_equal(_scan(p, d), p["D"][None, None, :, None] * p["x"])


# ------------------------------------------------------------- identities

def test_reverse_is_flip_forward_flip():
    rng = np.random.default_rng(6)
    p = _rand_params(rng, 2, 33, 4, 8, 16, 2)
    flip = {k: (np.ascontiguousarray(v[:, ::-1]) if k in ("x", "dt", "B", "C") else v) for k, v in p.items()}
    yr = _scan(p, -1)
    yff = _scan(flip, 1)[:, ::-1]
    assert np.max(np.abs(yr - yff)) <= 1e-15 * max(1.0, np.max(np.abs(yr)))


def test_linear_in_x():
    rng = np.random.default_rng(8)
    p = _rand_params(rng, 1, 24, 2, 4, 8, 1)
    x2 = rng.standard_normal(p["x"].shape)
    al, be = 0.75, -1.5
    q = dict(p, x=al * p["x"] + be * x2)
    y = _scan(q, 1)
    ref = al * _scan(p, 1) + be * _scan(dict(p, x=x2), 1)
    assert oracle.rel_err(y, ref) <= 1e-12


def test_thread_count_does_not_change_result():
    rng = np.random.default_rng(9)
    p = _rand_params(rng, 3, 20, 5, 4, 8, 1)
    assert np.array_equal(_scan(p, 1, nthreads=1), _scan(p, 1, nthreads=7))


def test_empty_inputs():
    p = _rand_params(np.random.default_rng(0), 0, 8, 2, 4, 4, 1)
    assert _scan(p, 1).shape == (0, 8, 2, 4)
    p = _rand_params(np.random.default_rng(0), 2, 0, 2, 4, 4, 1)
    assert _scan(p, -1).shape == (2, 0, 2, 4)


# ------------------------------------------------------------ chunked form

@pytest.mark.parametrize("chunk", [1, 4, 16, 32, 64])
@pytest.mark.parametrize("direction", [1, -1])
def test_chunked_form_matches_recurrence(chunk, direction):
    rng = np.random.default_rng(10)
    p = _rand_params(rng, 2, 64, 4, 8, 16, 2)
    y = oracle.ssd_chunked_f64(p["x"], p["dt"], p["A"], p["B"], p["C"], p["D"], direction, chunk)
    assert oracle.rel_err(y, _scan(p, direction)) <= 1e-12


def test_chunked_form_tiny_workload_chunk16():
    shape = si.WORKLOADS["tiny_f32"]["shape"]
    pf, _ = si.make_bidir(shape, seed=0)
    p = oracle.params_f64(pf)
    y = oracle.ssd_chunked_f64(p["x"], p["dt"], p["A"], p["B"], p["C"], p["D"], 1, 16)
    assert oracle.rel_err(y, _matrix_form(p, 1)) <= 1e-12


# ------------------------------------------------------------------- gate

def test_gate_zero_returns_residual_bitwise():
    rng = np.random.default_rng(11)
    p = _rand_params(rng, 2, 8, 2, 4, 4, 1)
    res = rng.standard_normal((2, 8, 8))
    res[0, 0, 0] = -0.0
    out = oracle.r2l_block_f64(p, 0.0, res)
    assert np.array_equal(out.view(np.uint64), res.view(np.uint64))


def test_gate_nonzero():
    rng = np.random.default_rng(12)
    p = _rand_params(rng, 2, 8, 2, 4, 4, 1)
    res = rng.standard_normal((2, 8, 8))
    out = oracle.r2l_block_f64(p, 0.3, res)
    ref = res + 0.3 * _matrix_form(p, -1).reshape(res.shape)
    assert oracle.rel_err(out, ref) <= 1e-12


# ------------------------------------------------------------------ state carried across calls

def _scan_state(p, direction, s0=None):
    return oracle.ssd_scan_state_f64(p["x"], p["dt"], p["A"], p["B"], p["C"], p.get("D"), direction, s0)


def _piece(p, lo, hi):
    return {k: (v[:, lo:hi] if k in ("x", "dt", "B", "C") else v) for k, v in p.items()}


@pytest.mark.parametrize("split", [1, 17, 39])
def test_state_carry_splits_the_sequence(split):
    """Scanning in two pieces, the second starting from the first's final state, equals scanning
    whole: the recurrence sees only S and the current token (both directions; for the reverse
    the right-hand piece is scanned first)."""
    rng = np.random.default_rng(11)
    p = _rand_params(rng, 2, 40, 3, 4, 6, 1)
    L = 40
    y_all, s_all = _scan_state(p, 1)
    assert oracle.rel_err(y_all, _scan(p, 1)) == 0.0
    y1, s1 = _scan_state(_piece(p, 0, split), 1)
    y2, s2 = _scan_state(_piece(p, split, L), 1, s1)
    assert oracle.rel_err(np.concatenate([y1, y2], axis=1), y_all) <= 1e-13
    assert oracle.rel_err(s2, s_all) <= 1e-13
    yr_all, sr_all = _scan_state(p, -1)
    yr2, sr2 = _scan_state(_piece(p, split, L), -1)
    yr1, sr1 = _scan_state(_piece(p, 0, split), -1, sr2)
    assert oracle.rel_err(np.concatenate([yr1, yr2], axis=1), yr_all) <= 1e-13
    assert oracle.rel_err(sr1, sr_all) <= 1e-13


def test_state_in_decays_in_closed_form():
    """x = 0 and a nonzero starting state S0: the state only decays, S_t = exp(A sum_{r<=t} dt_r) S0,
    so y_t[p] = sum_n C_t[n] S_t[p, n]; the final state is exp(A sum dt) S0."""
    rng = np.random.default_rng(12)
    p = _rand_params(rng, 2, 30, 3, 4, 5, 1)
    p["x"] = np.zeros_like(p["x"])
    s0 = rng.standard_normal((2, 3, 4, 5))
    for direction in (1, -1):
        y, s = _scan_state(p, direction, s0)
        dts = p["dt"] if direction > 0 else p["dt"][:, ::-1]
        decay = np.exp(np.cumsum(dts, axis=1) * p["A"][None, None, :])      # [b, L, H] in scan order
        if direction < 0:
            decay = decay[:, ::-1]
        ref = np.einsum("blh,bhpn,bln->blhp", decay, s0, p["C"][:, :, 0])
        assert oracle.rel_err(y, ref) <= 1e-12
        total = np.exp(p["A"][None, :] * p["dt"].sum(axis=1))                  # [b, H]
        assert oracle.rel_err(s, total[:, :, None, None] * s0) <= 1e-12


def test_final_state_is_the_decayed_sum_of_inputs():
    """Final state = sum over tokens s of exp(A * sum of dt after s in scan order) dt_s x_s (outer) B_s,
    plus the decayed starting state; every decay sum taken term by term."""
    rng = np.random.default_rng(13)
    b, L, H, P, N = 1, 12, 2, 3, 4
    p = _rand_params(rng, b, L, H, P, N, 1)
    s0 = rng.standard_normal((b, H, P, N))
    for direction in (1, -1):
        _, s = _scan_state(p, direction, s0)
        ref = np.zeros((b, H, P, N))
        for h in range(H):
            for t in range(L):
                after = range(t + 1, L) if direction > 0 else range(0, t)
                e = math.exp(p["A"][h] * sum(p["dt"][0, r, h] for r in after))
                ref[0, h] += e * p["dt"][0, t, h] * np.outer(p["x"][0, t, h], p["B"][0, t, 0])
            ref[0, h] += math.exp(p["A"][h] * sum(p["dt"][0, r, h] for r in range(L))) * s0[0, h]
        assert oracle.rel_err(s, ref) <= 1e-12


def test_empty_sequence_passes_the_state_through():
    rng = np.random.default_rng(14)
    p = _rand_params(rng, 2, 5, 3, 4, 5, 1)
    s0 = rng.standard_normal((2, 3, 4, 5))
    _, s = _scan_state(_piece(p, 0, 0), 1, s0)
    assert np.array_equal(s, s0)


# ------------------------------------------------------------------ gradients

def _loss(p, direction, gy):
    return float(np.sum(gy * _scan(p, direction)))


def _grads(p, direction, gy):
    return oracle.ssd_scan_bwd_f64(p["x"], p["dt"], p["A"], p["B"], p["C"], p.get("D"), direction, gy)


@pytest.mark.parametrize("direction", [1, -1])
@pytest.mark.parametrize("G", [1, 2])
def test_gradients_match_central_differences(direction, G):
    """Every gradient entry against a central difference of L = sum(gy * y) computed with the forward
    recurrence, on a small problem (L = 11 crosses no checkpoint; the second case is grouped)."""
    rng = np.random.default_rng(21 + G)
    p = _rand_params(rng, 2, 11, 4, 3, 4, G)
    gy = rng.standard_normal(p["x"].shape)
    g = _grads(p, direction, gy)
    eps = 1e-6
    for name in ("x", "dt", "A", "B", "C", "D"):
        base = p[name]
        idx = list(np.ndindex(base.shape))
        pick = [idx[i] for i in rng.choice(len(idx), size=min(12, len(idx)), replace=False)]
        for ix in pick:
            q = {k: (v.copy() if v is not None else None) for k, v in p.items()}
            q[name][ix] += eps
            lp = _loss(q, direction, gy)
            q[name][ix] -= 2 * eps
            lm = _loss(q, direction, gy)
            fd = (lp - lm) / (2 * eps)
            assert abs(fd - g[name][ix]) <= 1e-6 * max(1.0, abs(fd)), (name, ix, fd, g[name][ix])


def test_gradients_are_exact_for_the_linear_inputs():
    """y is linear in x, and y - D x is linear in B and in C, so L = sum(gy * y) equals the gradient's
    inner product with the input exactly: <gx, x> = L, <gB, B> = <gC, C> = L - <gy, D x>, and
    gD = sum_t <gy_t, x_t>.  Long enough (L = 150) to cross the checkpoint segments."""
    rng = np.random.default_rng(31)
    p = _rand_params(rng, 2, 150, 3, 4, 5, 1)
    gy = rng.standard_normal(p["x"].shape)
    for direction in (1, -1):
        g = _grads(p, direction, gy)
        L_ = _loss(p, direction, gy)
        Ldx = float(np.sum(gy * p["D"][None, None, :, None] * p["x"]))
        assert abs(np.sum(g["x"] * p["x"]) - L_) <= 1e-10 * max(1.0, abs(L_))
        assert abs(np.sum(g["B"] * p["B"]) - (L_ - Ldx)) <= 1e-10 * max(1.0, abs(L_))
        assert abs(np.sum(g["C"] * p["C"]) - (L_ - Ldx)) <= 1e-10 * max(1.0, abs(L_))
        np.testing.assert_allclose(g["D"], np.einsum("blhp,blhp->h", gy, p["x"]), rtol=1e-12)


def test_gradients_reverse_is_flip_of_forward():
    rng = np.random.default_rng(41)
    p = _rand_params(rng, 1, 70, 2, 3, 4, 1)
    gy = rng.standard_normal(p["x"].shape)
    flip = {k: (v[:, ::-1].copy() if k in ("x", "dt", "B", "C") else v) for k, v in p.items()}
    gr = _grads(p, -1, gy)
    gf = _grads(flip, 1, gy[:, ::-1].copy())
    for name in ("x", "dt", "B", "C"):
        np.testing.assert_allclose(gr[name], gf[name][:, ::-1], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(gr["A"], gf["A"], rtol=1e-12)
