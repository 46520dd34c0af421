"""GPU parity of ssd_scan_state: the scan with its state carried across the call.

Block-wise decoding (the DiffuMamba page, technical summary, sections 2 and 4:
block diffusion with cache reuse) scans a sequence one block at a time and
hands each block the state the previous one ended with.  These tests scan a
sequence in pieces through the C ABI, pass the float32 state from piece to
piece on the device, and compare every piece's output and the final state with
the float64 oracle run on the whole sequence; and they start a whole scan from
a given state.  Both kernel families: the tensor-core path (bf16, P = 64,
N = 128, 128-token blocks) and the SIMT path (other shapes, float32 io,
single-chunk pieces).

Metric: max|a - ref| / max|ref|, bars 2e-2 (bf16 io) and 1e-4 (float32 io),
applied to y (with D = None, so the scan itself is measured) and to the state.
"""
import numpy as np
import pytest
import torch

import oracle
import ssd_inputs as si

pytestmark = pytest.mark.gpu

TOL = {"bf16": 2e-2, "f32": 1e-4}

CASES = [
    # shape, chunk, split points (token indices), path of the whole-sequence call (1 tensor core,
    # 0 SIMT)
    (si.Shape(2, 512, 8, 64, 128, 1, "bf16"), 256, [256], 1),          # tensor-core path, block-aligned
    (si.Shape(1, 768, 8, 64, 128, 1, "bf16"), 128, [128, 512], 1),     # tensor-core path, three pieces
    (si.Shape(2, 96, 4, 32, 64, 1, "bf16"), 32, [32, 64], 0),          # SIMT, single-chunk pieces
    (si.Shape(1, 64, 2, 16, 16, 1, "f32"), 16, [16], 0),               # SIMT float32
]


def _path(ssd, shape, chunk, lo=0, hi=None):
    io = torch.bfloat16 if shape.io == "bf16" else torch.float32
    n = shape.seqlen if hi is None else hi - lo
    return ssd.path_for((shape.batch, n, shape.nheads, shape.headdim, shape.dstate, shape.ngroups), io, chunk)


@pytest.fixture(scope="module")
def ssd():
    import bidirectional_mamba_ssd_bidir_b200 as m
    return m


def _ids(v):
    return f"b{v.batch}L{v.seqlen}H{v.nheads}P{v.headdim}N{v.dstate}{v.io}" if isinstance(v, si.Shape) else str(v)


def _dev_piece(d, lo, hi):
    return {k: (None if v is None else v[:, lo:hi].contiguous() if k in ("x", "dt", "B", "C") else v)
            for k, v in d.items()}


def _f64_piece(q, lo, hi):
    return {k: (None if v is None else v[:, lo:hi] if k in ("x", "dt", "B", "C") else v) for k, v in q.items()}


def _oracle(q, direction, s0=None):
    return oracle.ssd_scan_state_f64(q["x"], q["dt"], q["A"], q["B"], q["C"], q.get("D"), direction, s0)


@pytest.mark.parametrize("shape,chunk,splits,path", CASES, ids=_ids)
@pytest.mark.parametrize("direction", [1, -1])
def test_pieces_carry_the_state(ssd, shape, chunk, splits, path, direction):
    assert _path(ssd, shape, chunk) == path
    p = si.make_params(shape, seed=31, with_D=False)
    dev = torch.device("cuda")
    d = {k: getattr(p, k).torch(dev) for k in ("x", "dt", "A", "B", "C")}
    d["D"] = None
    q = oracle.params_f64(p)
    y_ref, s_ref = _oracle(q, direction)
    bounds = [0] + splits + [shape.seqlen]
    pieces = list(zip(bounds[:-1], bounds[1:]))
    if direction < 0:
        pieces = pieces[::-1]                 # the reverse scan starts at the right end
    state = None
    ys = {}
    for lo, hi in pieces:
        assert _path(ssd, shape, chunk, lo, hi) == path       # every piece takes the same path
        y, state = ssd.ssd_scan_state(**_dev_piece(d, lo, hi), direction=direction, chunk=chunk, state_in=state)
        ys[lo] = y
    torch.cuda.synchronize()
    y_all = torch.cat([ys[lo] for lo in sorted(ys)], dim=1).double().cpu().numpy()
    assert oracle.rel_err(y_all, y_ref) <= TOL[shape.io]
    assert oracle.rel_err(state.double().cpu().numpy(), s_ref) <= TOL[shape.io]


@pytest.mark.parametrize("shape,chunk,splits,path", CASES, ids=_ids)
@pytest.mark.parametrize("direction", [1, -1])
def test_scan_from_a_given_state(ssd, shape, chunk, splits, path, direction):
    assert _path(ssd, shape, chunk) == path
    p = si.make_params(shape, seed=32, with_D=True)
    dev = torch.device("cuda")
    d = {k: getattr(p, k).torch(dev) for k in ("x", "dt", "A", "B", "C", "D")}
    q = oracle.params_f64(p)
    rng = np.random.default_rng(5)
    s0 = rng.standard_normal((shape.batch, shape.nheads, shape.headdim, shape.dstate)).astype(np.float32)
    y_ref, s_ref = _oracle(q, direction, s0.astype(np.float64))
    y, s = ssd.ssd_scan_state(**d, direction=direction, chunk=chunk, state_in=torch.from_numpy(s0).to(dev))
    torch.cuda.synchronize()
    # the SSD part alone: subtract the exactly known skip term D x in float64
    skip = q["D"][None, None, :, None] * q["x"]
    assert oracle.rel_err(y.double().cpu().numpy(), y_ref) <= TOL[shape.io]
    assert oracle.rel_err(s.double().cpu().numpy(), s_ref) <= TOL[shape.io]
    assert np.abs(y_ref - skip).max() > 0.05 * np.abs(y_ref).max()      # the state term is visible


def test_no_state_in_matches_ssd_scan(ssd):
    shape = si.Shape(2, 512, 8, 64, 128, 1, "bf16")
    assert _path(ssd, shape, 256) == 1
    p = si.make_params(shape, seed=33)
    d = {k: getattr(p, k).torch("cuda") for k in ("x", "dt", "A", "B", "C", "D")}
    for direction in (1, -1):
        y0 = ssd.ssd_scan(**d, direction=direction, chunk=256)
        y1, _ = ssd.ssd_scan_state(**d, direction=direction, chunk=256)
        torch.cuda.synchronize()
        assert torch.equal(y0, y1)


def test_empty_sequence_passes_the_state_through(ssd):
    shape = si.Shape(2, 0, 8, 64, 128, 1, "bf16")
    x = torch.empty(2, 0, 8, 64, dtype=torch.bfloat16, device="cuda")
    dt = torch.empty(2, 0, 8, dtype=torch.bfloat16, device="cuda")
    B = torch.empty(2, 0, 1, 128, dtype=torch.bfloat16, device="cuda")
    A = -torch.ones(8, device="cuda")
    s0 = torch.randn(2, 8, 64, 128, device="cuda")
    _, s = ssd.ssd_scan_state(x, dt, A, B, B, None, direction=1, chunk=256, state_in=s0)
    torch.cuda.synchronize()
    assert torch.equal(s, s0)
