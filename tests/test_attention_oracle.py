"""Pins of the float64 attention oracle (oracle/attention.py) against closed forms and brute force.

Each pin is chosen so that a plausible slip in the oracle fails it: a missing or
wrong scale, a softmax over the query axis instead of the key axis, Q and K
transposed, the q/k/v split taken in the wrong order, a dropped normalisation.
"""
import math

import numpy as np
import pytest

from oracle import attention as oa


def _rand(rng, *shape):
    return rng.standard_normal(shape)


def test_two_keys_closed_form():
    # one head, D = 4 (scale 1/2); scores q.k: key 0 gets 2 q0, key 1 gets -q1 ... written out by hand
    q = np.array([[1.0, 0.0, 0.0, 0.0], [0.0, 2.0, 0.0, 0.0], [0.5, 0.5, 0.0, 0.0]])
    k = np.array([[2.0, 0.0, 0.0, 0.0], [0.0, -1.0, 0.0, 0.0]])
    v = np.array([[1.0, 0.0, 3.0, -1.0], [0.0, 1.0, -2.0, 4.0]])
    out = oa.attention_f64(q[None, :, None, :], k[None, :, None, :], v[None, :, None, :])[0, :, 0, :]
    # query 0: scores (1, 0) -> weight of key 0 = 1 / (1 + e^-1)
    # query 1: scores (0, -1) -> weight of key 0 = 1 / (1 + e^-1)
    # query 2: scores (0.5, -0.25) -> weight of key 0 = 1 / (1 + e^-0.75)
    for i, d in enumerate([1.0, 1.0, 0.75]):
        w0 = 1.0 / (1.0 + math.exp(-d))
        np.testing.assert_allclose(out[i], w0 * v[0] + (1 - w0) * v[1], rtol=0, atol=1e-15)


def test_explicit_scale_and_dominant_key():
    rng = np.random.default_rng(1)
    q, k, v = _rand(rng, 1, 5, 2, 8), _rand(rng, 1, 7, 2, 8), _rand(rng, 1, 7, 2, 8)
    # scale 0: every key weighs 1/7
    np.testing.assert_allclose(oa.attention_f64(q, k, v, scale=0.0), np.broadcast_to(v.mean(axis=1, keepdims=True),
                                                                                   (1, 5, 2, 8)), atol=1e-14)
    # a key 1000 ahead in score takes all the weight
    k2 = k.copy()
    k2[0, 3] = 0.0
    q2 = np.zeros_like(q)
    q2[..., 0] = 1.0
    k2[0, 3, :, 0] = 1000.0 * np.sqrt(8)
    out = oa.attention_f64(q2, k2, v)
    np.testing.assert_allclose(out, np.broadcast_to(v[:, 3:4], out.shape), atol=1e-12)


def test_identical_keys_give_the_mean_of_v_and_ones_stay_ones():
    rng = np.random.default_rng(2)
    q, v = _rand(rng, 2, 6, 3, 16), _rand(rng, 2, 9, 3, 16)
    k = np.broadcast_to(_rand(rng, 2, 1, 3, 16), (2, 9, 3, 16))
    np.testing.assert_allclose(oa.attention_f64(q, k, v), np.broadcast_to(v.mean(axis=1, keepdims=True), (2, 6, 3, 16)),
                               atol=1e-14)
    k = _rand(rng, 2, 9, 3, 16)
    np.testing.assert_allclose(oa.attention_f64(q, k, np.ones((2, 9, 3, 16))), np.ones((2, 6, 3, 16)), atol=1e-14)


def test_row_shift_and_permutation_invariance():
    rng = np.random.default_rng(3)
    q, k, v = _rand(rng, 1, 10, 2, 8), _rand(rng, 1, 12, 2, 8), _rand(rng, 1, 12, 2, 8)
    ref = oa.attention_f64(q, k, v)
    # adding one vector to every key shifts each query's scores by a constant: no change
    np.testing.assert_allclose(oa.attention_f64(q, k + _rand(rng, 1, 1, 2, 8), v), ref, atol=1e-12)
    # keys and values permuted together: no change; queries permuted: rows permuted
    pk = rng.permutation(12)
    np.testing.assert_allclose(oa.attention_f64(q, k[:, pk], v[:, pk]), ref, atol=1e-13)
    pq = rng.permutation(10)
    np.testing.assert_allclose(oa.attention_f64(q[:, pq], k, v), ref[:, pq], atol=1e-13)
    # but not keys alone (the weights follow the keys)
    assert np.abs(oa.attention_f64(q, k[:, pk], v) - ref).max() > 1e-3


def test_brute_force_loops():
    rng = np.random.default_rng(4)
    B, Lq, Lk, H, D = 2, 3, 4, 2, 5
    q, k, v = _rand(rng, B, Lq, H, D), _rand(rng, B, Lk, H, D), _rand(rng, B, Lk, H, D)
    got = oa.attention_f64(q, k, v)
    for b in range(B):
        for h in range(H):
            for i in range(Lq):
                e = [math.exp(sum(q[b, i, h, d] * k[b, j, h, d] for d in range(D)) / math.sqrt(D)) for j in range(Lk)]
                z = sum(e)
                for d in range(D):
                    want = sum(e[j] * v[b, j, h, d] for j in range(Lk)) / z
                    assert abs(got[b, i, h, d] - want) < 1e-13


def test_sampled_rows_match_the_full_form():
    rng = np.random.default_rng(5)
    q, k, v = _rand(rng, 2, 20, 3, 8), _rand(rng, 2, 20, 3, 8), _rand(rng, 2, 20, 3, 8)
    full = oa.attention_f64(q, k, v)
    rows = [(0, 0, 0), (1, 19, 2), (1, 7, 1)]
    np.testing.assert_allclose(oa.attention_rows_f64(q, k, v, rows), np.stack([full[b, i, h] for b, i, h in rows]),
                               atol=1e-14)


def test_layer_split_order():
    """q, k, v are taken from W_qkv in that order: W_v = 0 gives 0; W_q = 0 gives uniform weights,
    so the output is the mean over tokens of v, times W_o^T."""
    rng = np.random.default_rng(6)
    B, L, dm, H, D = 1, 6, 8, 2, 4
    u = _rand(rng, B, L, dm)
    wq, wk, wv = _rand(rng, H * D, dm), _rand(rng, H * D, dm), _rand(rng, H * D, dm)
    wo = _rand(rng, dm, H * D)
    out = oa.attention_layer_f64(u, np.concatenate([wq, wk, 0 * wv]), wo, H)
    np.testing.assert_allclose(out, 0.0, atol=1e-14)
    out = oa.attention_layer_f64(u, np.concatenate([0 * wq, wk, wv]), wo, H)
    vbar = (u @ wv.T).mean(axis=1, keepdims=True)          # [B, 1, H D]
    np.testing.assert_allclose(out, np.broadcast_to(vbar @ wo.T, out.shape), atol=1e-12)
    # and with all three, it equals the per-head attention of the split projections
    out = oa.attention_layer_f64(u, np.concatenate([wq, wk, wv]), wo, H)
    q, k, v = ((u @ w.T).reshape(B, L, H, D) for w in (wq, wk, wv))
    np.testing.assert_allclose(out, oa.attention_f64(q, k, v).reshape(B, L, H * D) @ wo.T, atol=1e-12)


@pytest.mark.parametrize("mutant", ["no_scale", "query_axis", "transposed"])
def test_pins_catch_mutants(mutant):
    """Plant a slip in a copy of the oracle's arithmetic: the two-key closed form rejects each one."""
    def bad(q, k, v):
        q, k, v = (np.asarray(a, dtype=np.float64) for a in (q, k, v))
        D = q.shape[-1]
        scale = 1.0 if mutant == "no_scale" else 1.0 / np.sqrt(D)
        if mutant == "transposed":
            s = np.einsum("bihd,bjhd->bhij", k, q) * scale     # s_ij = k_i . q_j
        else:
            s = np.einsum("bihd,bjhd->bhij", q, k) * scale
        axis = -2 if mutant == "query_axis" else -1
        w = np.exp(s - s.max(axis=axis, keepdims=True))
        w = w / w.sum(axis=axis, keepdims=True)
        return np.einsum("bhij,bjhd->bihd", w, v)

    # scores q_i . k_j = [[2, 1], [0, -2]]: not symmetric, so a transposed product differs
    q = np.array([[1.0, 0.0, 0.0, 0.0], [0.0, 2.0, 0.0, 0.0]])
    k = np.array([[2.0, 0.0, 0.0, 0.0], [1.0, -1.0, 0.0, 0.0]])
    v = np.array([[1.0, 0.0, 3.0, -1.0], [0.0, 1.0, -2.0, 4.0]])
    good = oa.attention_f64(q[None, :, None], k[None, :, None], v[None, :, None])
    mut = bad(q[None, :, None], k[None, :, None], v[None, :, None])
    assert np.abs(good - mut).max() > 1e-3
