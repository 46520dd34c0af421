"""Float64 oracle of the DiffuMamba-H attention mixer (test infrastructure only).

The DiffuMamba page ("DiffuMamba: High-Throughput Diffusion LMs with Mamba
Backbone", technical summary, section 2) describes DiffuMamba-H as the same
stack with one Transformer block (an attention mixer) after every five Mamba
blocks.  The page does not spell the attention out; this module takes the
plainest reading for a diffusion language model, whose tokens all see the whole
sequence ("Bifocal Diffusion Language Models", section 1: bidirectional
attention): multi-head softmax attention with no mask,

    O[b, i, h, :] = sum_j softmax_j(scale * Q[b, i, h, :] . K[b, j, h, :]) V[b, j, h, :]

with scale = 1 / sqrt(headdim) unless given, and, for the whole block, the
projections around it:

    qkv = u W_qkv^T;  q, k, v = split(qkv, 3);  out = attention(q, k, v) W_o^T

(no bias, no positional encoding: the pages name none).  Each softmax is taken
with its row maximum subtracted (the mathematically identical, overflow-free
form); everything is numpy float64.
"""
from __future__ import annotations

import numpy as np


def attention_f64(q, k, v, scale=None):
    """q, k, v: [batch, L, H, D] (any float dtype); returns float64 [batch, L, H, D]."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    D = q.shape[-1]
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    # scores [batch, H, L_q, L_k]
    s = np.einsum("bihd,bjhd->bhij", q, k) * scale
    s = s - s.max(axis=-1, keepdims=True)
    w = np.exp(s)
    w = w / w.sum(axis=-1, keepdims=True)
    return np.einsum("bhij,bjhd->bihd", w, v)


def attention_rows_f64(q, k, v, rows, scale=None):
    """The output rows `rows` (a list of (b, i, h)) only, one at a time: for sampled checks of
    sizes whose full score matrix is too large.  Returns float64 [len(rows), D]."""
    q = np.asarray(q, dtype=np.float64)
    D = q.shape[-1]
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    out = np.empty((len(rows), D))
    for n, (b, i, h) in enumerate(rows):
        kk = np.asarray(k[b, :, h, :], dtype=np.float64)
        vv = np.asarray(v[b, :, h, :], dtype=np.float64)
        s = kk @ q[b, i, h, :] * scale
        s = s - s.max()
        w = np.exp(s)
        out[n] = (w / w.sum()) @ vv
    return out


def attention_layer_f64(u, w_qkv, w_o, nheads, scale=None):
    """The attention block: u [batch, L, d_model]; w_qkv [3 H D, d_model]; w_o [d_model, H D]."""
    u = np.asarray(u, dtype=np.float64)
    bsz, L, _ = u.shape
    qkv = u @ np.asarray(w_qkv, dtype=np.float64).T
    hd = qkv.shape[-1] // 3
    D = hd // nheads
    q, k, v = (qkv[..., i * hd:(i + 1) * hd].reshape(bsz, L, nheads, D) for i in range(3))
    o = attention_f64(q, k, v, scale).reshape(bsz, L, hd)
    return o @ np.asarray(w_o, dtype=np.float64).T


__all__ = ["attention_f64", "attention_rows_f64", "attention_layer_f64"]
