"""Pins of the Mamba-2 mixer oracle (oracle/mixer.py), CPU only.

The pages name the layer but print nothing of its inside, so nothing here is
a printed value.  The pins are what the reading fixes by itself:
  * the depthwise causal convolution's impulse response is its taps, and
    nothing before the impulse moves;
  * the forward layer is causal and the reverse layer anti-causal: a change
    of u at position t moves the forward layer's output only at >= t and the
    reverse layer's only at <= t;
  * with the same weights in both layers the mixer commutes with reversal;
  * the gated RMS norm is invariant to the scale of y and has unit RMS
    before its weight;
  * an independent scalar-loop evaluation of the whole layer (projections,
    convolution, activations, the recurrence itself, norm) on a tiny shape
    agrees to rounding;
and planted mistakes (a convolution one step off, a missing activation, the
norm over the wrong axis, a dropped dt bias, z and x swapped) each fail one.
"""
import math

import numpy as np
import pytest

import oracle
from oracle import mixer as om
import ssd_inputs as si

TINY = si.MixerShape(batch=2, seqlen=12, d_model=8, nheads=2, headdim=4, dstate=4, ngroups=1, d_conv=4)


def _inputs(shape, seed=0):
    u, f, r = si.make_mixer(shape, seed)
    return u.f64(), om.layer_to_f64(f), om.layer_to_f64(r)


def test_conv_impulse_response_is_the_taps():
    rng = np.random.default_rng(0)
    ch, K, L, t0 = 3, 4, 10, 4
    w, bias = rng.standard_normal((ch, K)), rng.standard_normal(ch)
    v = np.zeros((1, L, ch))
    v[0, t0, 1] = 1.0
    out = om.causal_conv_f64(v, w, bias)
    for t in range(L):
        want = bias.copy()
        s = t - t0
        if 0 <= s < K:
            want[1] += w[1, K - 1 - s]
        np.testing.assert_allclose(out[0, t], want, rtol=0, atol=1e-15)


def _layer_out(u, layer, shape, direction):
    if direction > 0:
        return om.layer_f64(u, layer, shape)
    return om.layer_f64(u[:, ::-1], layer, shape)[:, ::-1]


@pytest.mark.parametrize("direction", [1, -1])
def test_layer_causality(direction):
    u, f, _ = _inputs(TINY)
    base = _layer_out(u, f, TINY, direction)
    t = 5
    u2 = u.copy()
    u2[:, t] += 1.0
    moved = np.abs(_layer_out(u2, f, TINY, direction) - base).max(axis=(0, 2))
    if direction > 0:
        assert moved[:t].max() == 0.0 and moved[t:].min() > 0.0
    else:
        assert moved[t + 1:].max() == 0.0 and moved[:t + 1].min() > 0.0


def test_mixer_with_equal_layers_commutes_with_reversal():
    u, f, _ = _inputs(TINY)
    a = om.mixer_bidir_f64(u[:, ::-1], f, f, TINY)
    b = om.mixer_bidir_f64(u, f, f, TINY)[:, ::-1]
    np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-12)


def test_gated_norm_scale_invariance_and_unit_rms():
    rng = np.random.default_rng(1)
    y, z = rng.standard_normal((3, 5, 64)) * 3, rng.standard_normal((3, 5, 64))
    w = 1 + 0.1 * rng.standard_normal(64)
    a = om.gated_rmsnorm_f64(y, z, w)
    b = om.gated_rmsnorm_f64(7.0 * y, z, w)
    np.testing.assert_allclose(a, b, rtol=1e-5)
    rms = np.sqrt(np.mean((a / w) ** 2, axis=-1))
    g = y * z / (1 + np.exp(-z))
    ms = np.mean(g * g, axis=-1)
    np.testing.assert_allclose(rms, np.sqrt(ms / (ms + om.EPS)), rtol=1e-12)


def _loop_layer(u, L_, shape):
    """The forward layer with scalar loops: an evaluation independent of the oracle's
    vectorised one (and of the C recurrence)."""
    b, L, dm = u.shape
    H, P, N, G, K = shape.nheads, shape.headdim, shape.dstate, shape.ngroups, shape.d_conv
    di, cd = shape.d_inner, shape.conv_dim
    sig = lambda v: 1.0 / (1.0 + math.exp(-v))
    out = np.zeros((b, L, dm))
    for bb in range(b):
        proj = [[sum(u[bb, t, k] * L_["W_in"][o, k] for k in range(dm)) for o in range(shape.d_in_proj)]
                for t in range(L)]
        xbc = [[0.0] * cd for _ in range(L)]
        for t in range(L):
            for c in range(cd):
                acc = L_["conv_b"][c]
                for k in range(K):
                    tt = t + k - (K - 1)
                    if tt >= 0:
                        acc += L_["conv_w"][c, k] * proj[tt][di + c]
                xbc[t][c] = acc * sig(acc)
        S = np.zeros((H, P, N))
        for t in range(L):
            ys = [0.0] * di
            for h in range(H):
                raw = proj[t][di + cd + h] + L_["dt_bias"][h]
                dt = math.log1p(math.exp(raw))
                a = math.exp(dt * L_["A"][h])
                g = h // (H // G)
                for p in range(P):
                    xv = xbc[t][h * P + p]
                    acc = 0.0
                    for n in range(N):
                        Bv = xbc[t][di + g * N + n]
                        Cv = xbc[t][di + G * N + g * N + n]
                        S[h, p, n] = a * S[h, p, n] + dt * xv * Bv
                        acc += Cv * S[h, p, n]
                    ys[h * P + p] = acc + L_["D"][h] * xv
            gated = [ys[i] * proj[t][i] * sig(proj[t][i]) for i in range(di)]
            ms = sum(v * v for v in gated) / di
            yn = [gated[i] / math.sqrt(ms + om.EPS) * L_["norm_w"][i] for i in range(di)]
            for o in range(dm):
                out[bb, t, o] = sum(yn[i] * L_["W_out"][o, i] for i in range(di))
    return out


def test_layer_matches_scalar_loops():
    u, f, _ = _inputs(TINY, seed=3)
    np.testing.assert_allclose(om.layer_f64(u, f, TINY), _loop_layer(u, f, TINY), rtol=1e-10, atol=1e-12)


# planted mistakes: each must fail one of the pins above
def _mutant_parts(u, layer, shape, kind):
    b, L, _ = u.shape
    H, P, N, G = shape.nheads, shape.headdim, shape.dstate, shape.ngroups
    di, cd = shape.d_inner, shape.conv_dim
    zxbcdt = u @ layer["W_in"].T
    z, xbc_raw, dt_raw = zxbcdt[..., :di], zxbcdt[..., di:di + cd], zxbcdt[..., di + cd:]
    if kind == "z_x_swapped":
        z, xbc_raw = xbc_raw[..., :di], np.concatenate([z, xbc_raw[..., di:]], axis=-1)
    conv = om.causal_conv_f64(xbc_raw, layer["conv_w"], layer["conv_b"])
    if kind == "conv_one_step_late":
        conv = np.concatenate([np.broadcast_to(layer["conv_b"], (b, 1, cd)), conv[:, :-1]], axis=1)
    xbc = conv if kind == "no_silu" else om.silu(conv)
    x = xbc[..., :di].reshape(b, L, H, P)
    B = xbc[..., di:di + G * N].reshape(b, L, G, N)
    C = xbc[..., di + G * N:].reshape(b, L, G, N)
    dt = om.softplus(dt_raw + (0.0 if kind == "no_dt_bias" else layer["dt_bias"]))
    y = oracle.ssd_scan_f64(x, dt, layer["A"], B, C, layer["D"], 1).reshape(b, L, di)
    if kind == "norm_over_tokens":
        g = y * om.silu(z)
        yn = g / np.sqrt(np.mean(g * g, axis=1, keepdims=True) + om.EPS) * layer["norm_w"]
    else:
        yn = om.gated_rmsnorm_f64(y, z, layer["norm_w"])
    return yn @ layer["W_out"].T


@pytest.mark.parametrize("kind", ["conv_one_step_late", "no_silu", "norm_over_tokens", "no_dt_bias", "z_x_swapped"])
def test_planted_mistakes_are_caught(kind):
    u, f, _ = _inputs(TINY, seed=3)
    assert not np.allclose(_mutant_parts(u, f, TINY, kind), _loop_layer(u, f, TINY), rtol=1e-6, atol=1e-9)
    # and the unmutated restatement of the same code path agrees, so the difference is the mistake
    np.testing.assert_allclose(_mutant_parts(u, f, TINY, "none"), om.layer_f64(u, f, TINY), rtol=1e-12)
