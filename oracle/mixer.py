"""Float64 oracle of the Mamba-2 mixer around the scan (test infrastructure only).

The DiffuMamba page ("DiffuMamba: High-Throughput Diffusion LMs with Mamba
Backbone", technical summary, section 2) replaces attention with
bidirectional Mamba-2 layers: two independent layers, one run forward and
one run on the reversed sequence, combined by summation.  The page names
the layer, not its inside; this module takes the plainest reading, the
standard Mamba-2 block:

    zxbcdt = u W_in^T                                 (one projection, no bias)
    z, xBC, dt_raw = split(zxbcdt, [d_inner, d_inner + 2 G N, H])
    xBC = silu(causal depthwise conv1d(xBC, width d_conv) + conv_b)
    x, B, C = split(xBC, [d_inner, G N, G N])
    dt = softplus(dt_raw + dt_bias)
    y = scan(x, dt, A, B, C, D)                       (the plain recurrence, ssd_scan_f64)
    g = y * silu(z);  yn = g / sqrt(mean(g^2) + eps) * norm_w      (over d_inner, eps 1e-5)
    out = yn W_out^T

and the bidirectional mixer  out_fwd(u) + flip(out_rev(flip(u))), each layer with its own
weights.  Every step is written out with numpy primitives (matmul, elementwise), in the
order above; the reverse layer is literally the forward layer on the flipped sequence.
"""
from __future__ import annotations

import numpy as np

from . import ssd_scan_f64

EPS = 1e-5


def silu(v):
    return v / (1.0 + np.exp(-v))


def softplus(v):
    return np.logaddexp(0.0, v)


def causal_conv_f64(v, w, bias):
    """Depthwise causal convolution over the sequence axis: v [b, L, ch], w [ch, K], bias [ch];
    out[t] = bias + sum_k w[:, k] v[t + k - (K - 1)], zero before the first position."""
    b, L, ch = v.shape
    K = w.shape[1]
    out = np.broadcast_to(bias, (b, L, ch)).astype(np.float64).copy()
    for k in range(K):
        shift = K - 1 - k                      # v[t - shift]
        if shift == 0:
            out += w[:, k] * v
        else:
            out[:, shift:] += w[:, k] * v[:, :-shift]
    return out


def gated_rmsnorm_f64(y, z, weight, eps=EPS):
    """y * silu(z), normalised by its root mean square over the last axis, times weight."""
    g = y * silu(z)
    return g / np.sqrt(np.mean(g * g, axis=-1, keepdims=True) + eps) * weight


def layer_parts_f64(u, layer, shape):
    """The forward-run layer on u [b, L, d_model] (float64 arrays in `layer`): every
    intermediate, for tests that check a stage on its own."""
    b, L, _ = u.shape
    H, P, N, G = shape.nheads, shape.headdim, shape.dstate, shape.ngroups
    di, cd = shape.d_inner, shape.conv_dim
    zxbcdt = u @ layer["W_in"].T
    z = zxbcdt[..., :di]
    xbc_raw = zxbcdt[..., di:di + cd]
    dt_raw = zxbcdt[..., di + cd:]
    xbc = silu(causal_conv_f64(xbc_raw, layer["conv_w"], layer["conv_b"]))
    x = xbc[..., :di].reshape(b, L, H, P)
    B = xbc[..., di:di + G * N].reshape(b, L, G, N)
    C = xbc[..., di + G * N:].reshape(b, L, G, N)
    dt = softplus(dt_raw + layer["dt_bias"])
    y = ssd_scan_f64(x, dt, layer["A"], B, C, layer["D"], 1).reshape(b, L, di)
    yn = gated_rmsnorm_f64(y, z, layer["norm_w"])
    out = yn @ layer["W_out"].T
    return {"zxbcdt": zxbcdt, "z": z, "xbc": xbc, "x": x, "B": B, "C": C, "dt": dt, "y": y, "yn": yn, "out": out}


def layer_f64(u, layer, shape):
    return layer_parts_f64(u, layer, shape)["out"]


def mixer_bidir_f64(u, fwd, rev, shape):
    """out_fwd(u) + flip(out_rev(flip(u))) over the sequence axis."""
    return layer_f64(u, fwd, shape) + layer_f64(u[:, ::-1], rev, shape)[:, ::-1]


def layer_to_f64(layer: dict) -> dict:
    """Stored weights (ssd_inputs) to float64 arrays."""
    return {k: v.f64() for k, v in layer.items()}
