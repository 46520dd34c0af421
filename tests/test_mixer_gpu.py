"""The Mamba-2 mixer around the scan on the GPU, against the float64 oracle (oracle/mixer.py).

The tensor-core GEMM is checked on its own first (bf16 operands are exact
products in float32; the only error is float32 accumulation and the final
bf16 rounding), then the whole bidirectional mixer: two independent layers,
forward and on the reversed sequence, summed, at the spec bar for bf16
io (2e-2, max-normalised).
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import mixer as om
import ssd_inputs as si

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ssd():
    import bidirectional_mamba_ssd_bidir_b200 as m
    return m


# The GEMM is persistent over 128 x 256 output tiles (one CTA per SM, two TMEM accumulators in
# turn): shapes with fewer tiles than SMs, with one or two tiles per CTA (8192 x 1024), and with
# about fourteen per CTA (32768 x 2048), plus ragged last column tiles (N = 8, 200, 264, 1288, 8512).
@pytest.mark.parametrize("M,N,K", [(256, 1288, 256), (384, 200, 128), (128, 64, 64), (512, 8512, 2048),
                                   (128, 8, 64), (256, 264, 192), (8192, 1024, 256), (32768, 2048, 128)])
def test_gemm_matches_float64(ssd, M, N, K):
    g = torch.Generator().manual_seed(M + N + K)
    A = torch.randn(M, K, generator=g).to(torch.bfloat16)
    W = (torch.randn(N, K, generator=g) / K ** 0.5).to(torch.bfloat16)
    D = ssd.gemm_bf16(A.cuda(), W.cuda())
    torch.cuda.synchronize()
    ref = A.double().numpy() @ W.double().numpy().T
    got = D.double().cpu().numpy()
    # within a bf16 rounding step of the float64 product (plus float32 accumulation)
    assert np.all(np.abs(got - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-3 * np.abs(ref).max()), np.abs(got - ref).max()


SHAPES = [
    si.MixerShape(batch=2, seqlen=256, d_model=256, nheads=8),       # d_in_proj 1288: a ragged last N tile
    si.MixerShape(batch=1, seqlen=384, d_model=512, nheads=16),      # 3 blocks of 128, 16 heads
    si.MixerShape(batch=1, seqlen=256, d_model=256, nheads=8, d_conv=2),   # other compiled conv widths
    si.MixerShape(batch=1, seqlen=256, d_model=256, nheads=8, d_conv=3),
    si.MixerShape(batch=1, seqlen=256, d_model=256, nheads=8, d_conv=6),   # the run-time width path
    si.MixerShape(batch=1, seqlen=256, d_model=256, nheads=8, d_conv=1),
]


def _dev_layer(layer):
    return {k: v.torch("cuda") for k, v in layer.items()}


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: f"b{s.batch}L{s.seqlen}dm{s.d_model}H{s.nheads}K{s.d_conv}")
def test_mixer_matches_oracle(ssd, shape):
    u, f, r = si.make_mixer(shape, seed=7)
    ws = torch.zeros(ssd.mixer_workspace_bytes(shape.batch, shape.seqlen, shape.d_model, shape.nheads),
                     dtype=torch.uint8, device="cuda")
    out = ssd.mixer_bidir(u.torch("cuda"), _dev_layer(f), _dev_layer(r), shape.nheads, d_conv=shape.d_conv,
                          workspace=ws)
    torch.cuda.synchronize()
    ssd.workspace_status(ws)
    ref = om.mixer_bidir_f64(u.f64(), om.layer_to_f64(f), om.layer_to_f64(r), shape)
    assert oracle.rel_err(out.double().cpu().numpy(), ref) <= 2e-2


def test_mixer_layers_are_independent(ssd):
    """The reverse layer's weights change only the reverse part: swapping in another reverse layer
    moves the output by exactly that layer's difference (up to bf16 rounding of the sum)."""
    shape = SHAPES[0]
    u, f, r = si.make_mixer(shape, seed=8)
    _, _, r2 = si.make_mixer(shape, seed=9)
    ud = u.torch("cuda")
    a = ssd.mixer_bidir(ud, _dev_layer(f), _dev_layer(r), shape.nheads)
    b = ssd.mixer_bidir(ud, _dev_layer(f), _dev_layer(r2), shape.nheads)
    torch.cuda.synchronize()
    uf = u.f64()
    want = om.layer_f64(uf[:, ::-1], om.layer_to_f64(r), shape)[:, ::-1] - \
        om.layer_f64(uf[:, ::-1], om.layer_to_f64(r2), shape)[:, ::-1]
    assert oracle.rel_err((a.double() - b.double()).cpu().numpy(), want) <= 3e-2
