"""Planted mistakes in the oracle must be caught by its pins.

Each case rewrites one line of ``oracle/ssd_oracle.c`` into a plausible bug
(a dropped term, a wrong sign or index, a transposed operand), compiles the
mutant into a temporary directory and runs the pins against it.  A mutant
that passes every pin would mean the pins cannot tell that bug from the
correct recurrence.  CPU only; nothing here touches a GPU.
"""
import json
import math
import os
import subprocess

import numpy as np
import pytest

import oracle
from pins import matrix_form, rand_params

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "ssd_oracle.c")

MUTANTS = {
    "B_and_C_swapped_in_update": ("u * Bt[n]", "u * Ct[n]"),
    "C_replaced_by_B_in_output": ("acc += Ct[n] * Sp[n]", "acc += Bt[n] * Sp[n]"),
    "skip_term_dropped": ("yt[p] = acc + d_h * xt[p];", "yt[p] = acc;"),
    "decay_sign_flipped": ("exp(dt * a_h)", "exp(-dt * a_h)"),
    "decay_after_input": ("Sp[n] = decay * Sp[n] + u * Bt[n];", "Sp[n] = decay * (Sp[n] + u * Bt[n]);"),
    "dt_missing_on_input": ("const double u = dt * xt[p];", "const double u = xt[p];"),
    "reverse_runs_forward": ("j->direction > 0 ? k : L - 1 - k", "k"),
    "reverse_off_by_one": ("j->direction > 0 ? k : L - 1 - k", "j->direction > 0 ? k : (k == 0 ? 0 : L - k)"),
    "group_index_wrong": ("h / (H / j->ngroups)", "h % j->ngroups"),
    "dt_head_index_dropped": ("j->dt[((size_t)b * L + t) * H + h]", "j->dt[((size_t)b * L + t) * H]"),
    "output_before_update": ("Sp[n] = decay * Sp[n] + u * Bt[n];\n                acc += Ct[n] * Sp[n];",
                             "acc += Ct[n] * Sp[n];\n                Sp[n] = decay * Sp[n] + u * Bt[n];"),
    "state_in_ignored": ("if (j->s_in)\n        memcpy", "if (0)\n        memcpy"),
    "state_slot_head_dropped": ("const size_t soff = ((size_t)b * H + h)", "const size_t soff = ((size_t)b * H)"),
    "bwd_adjoint_not_decayed": ("G[i] *= a;", "G[i] *= 1.0;"),
    "bwd_dt_gradient_misses_decay_term": ("gxb + a_h * a * q", "gxb"),
    "bwd_B_gradient_without_dt": ("gBt[n] += dt * acc;", "gBt[n] += acc;"),
}


def _build_mutant(tmp_path, name, old, new):
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation site for {name} not found"
    mut = src.replace(old, new, 1)
    c = tmp_path / f"{name}.c"
    so = tmp_path / f"lib{name}.so"
    c.write_text(mut)
    subprocess.check_call(["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-pthread", "-o", str(so), str(c), "-lm"])
    return oracle.load_library(str(so))


def _pins_pass(lib) -> bool:
    """Runs a compact set of the oracle's pins against ``lib``; True only if all hold."""
    def scan(p, d):
        return oracle.ssd_scan_f64(p["x"], p["dt"], p["A"], p["B"], p["C"], p.get("D"), d, lib=lib)

    g = json.load(open(os.path.join(ROOT, "tests", "golden", "ssd_handworked_L3.json")))
    pg = dict(x=np.array(g["x"])[None, :, None, :], dt=np.array(g["dt"])[None, :, None],
              A=np.array(g["A"]), B=np.array(g["B"])[None, :, None, :],
              C=np.array(g["C"])[None, :, None, :], D=np.array(g["D"]))
    checks = [
        np.allclose(scan(pg, 1)[0, :, 0], g["y_forward"], rtol=0, atol=1e-12),
        np.allclose(scan(pg, -1)[0, :, 0], g["y_reverse"], rtol=0, atol=1e-12),
    ]
    rng = np.random.default_rng(7)
    p = rand_params(rng, 2, 13, 4, 3, 5, 2)
    for d in (1, -1):
        checks.append(oracle.rel_err(scan(p, d), matrix_form(p, d)) <= 1e-12)
    L, dtv, xv, Av = 40, 0.3, 1.7, -2.5
    e1 = np.zeros((1, L, 1, 4)); e1[..., 0] = 1.0
    pgeo = dict(x=np.full((1, L, 1, 1), xv), dt=np.full((1, L, 1), dtv), A=np.array([Av]),
                B=e1, C=e1, D=None)
    a = math.exp(dtv * Av)
    ref = np.array([dtv * xv * (1 - a ** (t + 1)) / (1 - a) for t in range(L)])
    checks.append(np.allclose(scan(pgeo, 1)[0, :, 0, 0], ref, rtol=1e-13))
    # state carried across a split of the sequence, from a nonzero starting state
    s0 = rng.standard_normal((2, 4, 3, 5))
    def scan_state(q, d, s_in):
        return oracle.ssd_scan_state_f64(q["x"], q["dt"], q["A"], q["B"], q["C"], q.get("D"), d, s_in, lib=lib)
    piece = lambda lo, hi: {k: (v[:, lo:hi] if k in ("x", "dt", "B", "C") else v) for k, v in p.items()}
    y_all, s_all = scan_state(p, 1, s0)
    y1, s1 = scan_state(piece(0, 5), 1, s0)
    y2, s2 = scan_state(piece(5, 13), 1, s1)
    checks.append(oracle.rel_err(np.concatenate([y1, y2], axis=1), y_all) <= 1e-12)
    checks.append(oracle.rel_err(s2, s_all) <= 1e-12)
    zero_x = dict(p, x=np.zeros_like(p["x"]))
    y0, _ = scan_state(zero_x, 1, s0)
    decay = np.exp(np.cumsum(p["dt"], axis=1) * p["A"][None, None, :])
    g = np.arange(4) // 2
    ref0 = np.einsum("blh,bhpn,blhn->blhp", decay, s0, p["C"][:, :, g])
    checks.append(oracle.rel_err(y0, ref0) <= 1e-12)
    # gradients: exact inner-product identities for x and B, a central difference for dt
    gy = rng.standard_normal(p["x"].shape)
    for d in (1, -1):
        g = oracle.ssd_scan_bwd_f64(p["x"], p["dt"], p["A"], p["B"], p["C"], p["D"], d, gy, lib=lib)
        L_ = float(np.sum(gy * scan(p, d)))
        Ldx = float(np.sum(gy * p["D"][None, None, :, None] * p["x"]))
        checks.append(abs(np.sum(g["x"] * p["x"]) - L_) <= 1e-10 * max(1.0, abs(L_)))
        checks.append(abs(np.sum(g["B"] * p["B"]) - (L_ - Ldx)) <= 1e-10 * max(1.0, abs(L_)))
        q = {k: (v.copy() if v is not None else None) for k, v in p.items()}
        q["dt"][0, 4, 1] += 1e-6
        lp = float(np.sum(gy * scan(q, d)))
        q["dt"][0, 4, 1] -= 2e-6
        lm = float(np.sum(gy * scan(q, d)))
        checks.append(abs((lp - lm) / 2e-6 - g["dt"][0, 4, 1]) <= 1e-6 * max(1.0, abs(lp - lm) / 2e-6))
    return all(bool(c) for c in checks)


def test_unmutated_oracle_passes_compact_pins():
    assert _pins_pass(oracle.load_library())


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(tmp_path, name):
    old, new = MUTANTS[name]
    lib = _build_mutant(tmp_path, name, old, new)
    assert not _pins_pass(lib), f"planted mistake '{name}' passed every pin"
