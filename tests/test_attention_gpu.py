"""The DiffuMamba-H attention mixer on the GPU against the float64 oracle (oracle/attention.py).

Errors are max-abs over max-ref (the spec bar for bf16 io, 2e-2).  The
kernel rounds P to bf16 before the PV product and writes bf16, so its error is
a few bf16 steps; the cases below cover one tile and many, a sequence that
ends inside a tile (keys past the end must not count, rows past it must not be
written), one token, both head sizes, the rescaling of O when a row's maximum
grows along the keys, peaked softmax rows, an explicit scale, q/k/v as views of
one packed projection, sampled rows at the 1.3B shape, and the whole block.
"""
import numpy as np
import pytest
import torch

import oracle
import ssd_inputs as si
from oracle import attention as oa

pytestmark = pytest.mark.gpu
BAR = 2e-2


@pytest.fixture(scope="module")
def ssd():
    import bidirectional_mamba_ssd_bidir_b200 as m
    return m


def _qkv(shape, seed):
    host = si.make_attention(shape, seed)
    return tuple(t.torch("cuda") for t in host), host


def _check(out, ref):
    err = oracle.rel_err(out.double().cpu().numpy(), ref)
    assert err <= BAR, err
    return err


SHAPES = [
    si.AttnShape(1, 128, 2, 128),      # one tile
    si.AttnShape(2, 512, 2, 128),      # four key tiles, four query tiles
    si.AttnShape(2, 300, 3, 64),       # ends inside the third tile
    si.AttnShape(1, 129, 1, 64),       # one key past a tile
    si.AttnShape(1, 1, 2, 128),        # one token
    si.AttnShape(3, 1000, 2, 128),     # 8 tiles, ragged
]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: f"b{s.batch}L{s.seqlen}H{s.nheads}D{s.headdim}")
def test_attention_matches_oracle(ssd, shape):
    (q, k, v), host = _qkv(shape, 11)
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    out = torch.full_like(q, float("nan"))
    ssd.attention(q, k, v, out=out, workspace=ws)
    torch.cuda.synchronize()
    ssd.workspace_status(ws)
    _check(out, oa.attention_f64(*(t.f64() for t in host)))


def test_growing_scores_rescale_the_output(ssd):
    """Keys grow along the sequence, so every row's maximum rises tile after tile (the O rescale path)."""
    shape = si.AttnShape(1, 1024, 2, 128)
    (q, k, v), _ = _qkv(shape, 12)
    ramp = torch.linspace(0.0, 2.0, shape.seqlen, device="cuda").view(1, -1, 1, 1)
    q = (q.float() + 1.0).to(torch.bfloat16)          # a common direction: scores grow with the ramp
    k = (k.float() + ramp).to(torch.bfloat16)
    out = ssd.attention(q, k, v)
    torch.cuda.synchronize()
    _check(out, oa.attention_f64(q.double().cpu().numpy(), k.double().cpu().numpy(), v.double().cpu().numpy()))


def test_peaked_rows_and_explicit_scale(ssd):
    shape = si.AttnShape(2, 384, 2, 64)
    (q, k, v), _ = _qkv(shape, 13)
    qh, kh, vh = (t.double().cpu().numpy() for t in (q, k, v))
    out = ssd.attention(q, k, v, scale=1.0)            # scores of std 8: nearly one-hot rows
    torch.cuda.synchronize()
    _check(out, oa.attention_f64(qh, kh, vh, scale=1.0))
    out = ssd.attention(q, k, v, scale=0.01)           # nearly uniform rows
    torch.cuda.synchronize()
    _check(out, oa.attention_f64(qh, kh, vh, scale=0.01))


def test_packed_projection_views(ssd):
    """q, k, v as column blocks of one [b, L, 3, H, D] tensor (tokens 3 H D elements apart)."""
    b, L, H, D = 2, 256, 2, 128
    g = torch.Generator().manual_seed(14)
    qkv = torch.randn(b, L, 3, H, D, generator=g).to(torch.bfloat16).cuda()
    q, k, v = qkv[:, :, 0], qkv[:, :, 1], qkv[:, :, 2]
    out = ssd.attention(q, k, v)
    torch.cuda.synchronize()
    _check(out, oa.attention_f64(*(t.double().cpu().numpy() for t in (q, k, v))))


def test_full_size_sampled_rows(ssd):
    """The 1.3B attention shape (b4, L8192, 16 heads of 128): sampled rows against the oracle row by row."""
    shape = si.AttnShape(4, 8192, 16, 128)
    (q, k, v), _ = _qkv(shape, 15)
    out = ssd.attention(q, k, v)
    torch.cuda.synchronize()
    rng = np.random.default_rng(0)
    rows = [(int(rng.integers(4)), int(rng.integers(8192)), int(rng.integers(16))) for _ in range(48)]
    rows += [(0, 0, 0), (3, 8191, 15), (1, 127, 3), (2, 128, 7)]
    ref = []
    for b, i, h in rows:       # one (sequence, head) at a time: float64 copies of 8192 x 128 only
        one = [t[b:b + 1, :, h:h + 1].double().cpu().numpy() for t in (q, k, v)]
        ref.append(oa.attention_rows_f64(one[0], one[1], one[2], [(0, i, 0)])[0])
    ref = np.stack(ref)
    got = np.stack([out[b, i, h].double().cpu().numpy() for b, i, h in rows])
    assert np.abs(got - ref).max() / np.abs(ref).max() <= BAR


def test_attention_block_matches_oracle(ssd):
    shape = si.AttnShape(2, 256, 2, 128, d_model=256)
    u, wqkv, wo = si.make_attention_layer(shape, 16)
    out = ssd.attention_block(u.torch("cuda"), wqkv.torch("cuda"), wo.torch("cuda"), shape.nheads, shape.headdim)
    torch.cuda.synchronize()
    ref = oa.attention_layer_f64(u.f64(), wqkv.f64(), wo.f64(), shape.nheads)
    _check(out, ref)


def test_attention_block_at_width_2048(ssd):
    """The 1.3B block width (d_model 2048, 16 heads x 128) on one 2048-token sequence: both
    projections run several 128 x 256 tiles per persistent GEMM CTA."""
    shape = si.AttnShape(1, 2048, 16, 128, d_model=2048)
    u, wqkv, wo = si.make_attention_layer(shape, 17)
    out = ssd.attention_block(u.torch("cuda"), wqkv.torch("cuda"), wo.torch("cuda"), shape.nheads, shape.headdim)
    torch.cuda.synchronize()
    ref = oa.attention_layer_f64(u.f64(), wqkv.f64(), wo.f64(), shape.nheads)
    _check(out, ref)


def test_refuses_other_head_sizes(ssd):
    q = torch.zeros(1, 128, 2, 96, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ssd.SSDError):
        ssd.attention(q, q, q)
