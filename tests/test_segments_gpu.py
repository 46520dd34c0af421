"""Sequences cut into segments that run in parallel (tensor-core path).

When the batch alone gives fewer CTAs than the GPU has SMs, a call cuts each
sequence into segments of whole 128-token blocks: a first kernel forms every
segment's local end state (starting from zero), the scan then runs every
segment at once from the state folded from the segments before it.  The
recurrence is linear in the state, so the result is the whole-sequence scan;
these tests check it against the float64 oracle, against the unsegmented
kernel (the no-allocation entry point never segments), with a ragged last
segment, with a state carried in and out, and with chains the exact kernel
takes (steep decay).
"""
import numpy as np
import pytest
import torch

import oracle
import ssd_inputs as si

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ssd():
    import bidirectional_mamba_ssd_bidir_b200 as m
    return m


def _dev(p, with_D=True):
    d = {k: getattr(p, k).torch("cuda") for k in ("x", "dt", "A", "B", "C")}
    d["D"] = p.D.torch("cuda") if with_D else None
    return d


def _dims(shape):
    return (shape.batch, shape.seqlen, shape.nheads, shape.headdim, shape.dstate, shape.ngroups)


def test_segment_policy(ssd):
    """Segments only when batch x heads leaves SMs idle, at least two blocks each."""
    bf = torch.bfloat16
    assert ssd.segments_for((4, 8192, 64, 64, 128, 1), bf, 256) == 1       # 256 CTAs already
    assert ssd.segments_for((1, 32768, 64, 64, 128, 1), bf, 256) == 2      # 64 CTAs -> 128
    assert ssd.segments_for((1, 131072, 64, 64, 128, 1), bf, 256) == 2
    assert ssd.segments_for((1, 1024, 8, 64, 128, 1), bf, 256) == 4        # 8 blocks, 2 per segment
    assert ssd.segments_for((1, 1408, 8, 64, 128, 1), bf, 128) == 4        # 11 blocks: 3, 3, 3, 2
    assert ssd.segments_for((1, 128, 8, 64, 128, 1), bf, 128) == 1        # a single block
    assert ssd.kernel_launches((4, 8192, 64, 64, 128, 1), bf, 256, "bidir") == 3     # marks, scan, exact


CASES = [
    # shape, chunk; the policy's segment count follows from batch * heads and the block count
    (si.Shape(1, 1024, 8, 64, 128, 1, "bf16"), 256),      # 8 blocks, 4 segments of 2
    (si.Shape(1, 1408, 8, 64, 128, 1, "bf16"), 128),      # 11 blocks: segments of 3, 3, 3, 2
    (si.Shape(2, 2048, 16, 64, 128, 1, "bf16"), 256),     # 16 blocks, 4 segments of 4
]


@pytest.mark.parametrize("shape,chunk", CASES, ids=lambda v: str(v) if isinstance(v, int) else
                         f"b{v.batch}L{v.seqlen}H{v.nheads}")
@pytest.mark.parametrize("with_D", [True, False], ids=["full", "ssd_only"])
def test_segmented_bidir_matches_oracle(ssd, shape, chunk, with_D):
    assert ssd.path_for(_dims(shape), torch.bfloat16, chunk) == 1
    assert ssd.kernel_launches(_dims(shape), torch.bfloat16, chunk, "bidir") == 3     # segmented
    pf, pr = si.make_bidir(shape, seed=3, with_D=with_D)
    y = ssd.bidir_ssd(_dev(pf, with_D), _dev(pr, with_D), chunk=chunk)
    torch.cuda.synchronize()
    ref = oracle.bidir_f64(oracle.params_f64(pf), oracle.params_f64(pr))
    assert oracle.rel_err(y.double().cpu().numpy(), ref) <= 2e-2


@pytest.mark.parametrize("shape,chunk", CASES[:2], ids=["b1L1024", "b1L1408"])
def test_segmented_equals_unsegmented(ssd, shape, chunk):
    """The same call through the no-allocation entry point, which keeps one CTA per sequence."""
    pf, pr = si.make_bidir(shape, seed=4)
    f, r = _dev(pf), _dev(pr)
    y_seg = ssd.bidir_ssd(f, r, chunk=chunk)
    out = torch.empty_like(f["x"])
    area = ssd.bidir_ssd_noalloc(f, r, out, chunk=chunk)
    torch.cuda.synchronize()
    ssd.noalloc_status(area)
    # the state entering a segment is formed in float32 and rounded to bf16 once where the
    # unsegmented kernel carries it block by block: a few bf16 steps apart at most
    err = ((y_seg.float() - out.float()).abs().max() / out.float().abs().max()).item()
    assert err <= 1e-2, err


@pytest.mark.parametrize("direction", [1, -1])
def test_segmented_state_in_and_out(ssd, direction):
    shape, chunk = si.Shape(1, 1408, 8, 64, 128, 1, "bf16"), 128
    assert ssd.kernel_launches(_dims(shape), torch.bfloat16, chunk, "scan") == 3
    p = si.make_params(shape, seed=8, with_D=True)
    d = {k: getattr(p, k).torch("cuda") for k in ("x", "dt", "A", "B", "C", "D")}
    q = oracle.params_f64(p)
    rng = np.random.default_rng(9)
    s0 = rng.standard_normal((shape.batch, shape.nheads, shape.headdim, shape.dstate)).astype(np.float32)
    y_ref, s_ref = oracle.ssd_scan_state_f64(q["x"], q["dt"], q["A"], q["B"], q["C"], q["D"], direction,
                                             s0.astype(np.float64))
    y, s = ssd.ssd_scan_state(**d, direction=direction, chunk=chunk, state_in=torch.from_numpy(s0).cuda())
    torch.cuda.synchronize()
    assert oracle.rel_err(y.double().cpu().numpy(), y_ref) <= 2e-2
    assert oracle.rel_err(s.double().cpu().numpy(), s_ref) <= 2e-2


def test_segmented_steep_chain_goes_to_the_exact_kernel(ssd):
    """One head pair with a decay too steep for the factorised kernel, in a segmented call: the
    segment-state kernel marks the chain, the scan leaves all its segments, the exact kernel
    runs it whole, and the result matches the oracle in both directions."""
    shape, chunk = si.Shape(1, 1024, 8, 64, 128, 1, "bf16"), 256
    pf, pr = si.make_bidir(shape, seed=6)
    for p in (pf, pr):
        A = p.A.data.copy()
        A[2] = -60.0            # |A| dt over a block: hundreds in log2 units (dt ~ 0.01 .. 0.1)
        p.A.data[:] = A
    y = ssd.bidir_ssd(_dev(pf), _dev(pr), chunk=chunk)
    torch.cuda.synchronize()
    ref = oracle.bidir_f64(oracle.params_f64(pf), oracle.params_f64(pr))
    assert oracle.rel_err(y.double().cpu().numpy(), ref) <= 2e-2


def test_bidir_with_one_direction_steep(ssd):
    """The forward layer has a head pair too steep for the factorised kernel, the reverse layer
    does not: the exact kernel runs that pair's forward chain while the shared-score kernel runs
    its reverse chain, and the two parts of every output block still meet once (both kernels take
    the same ticket per head pair and block).  Segmented (bidir_ssd) and whole-sequence
    (bidir_ssd_noalloc) calls."""
    shape, chunk = si.Shape(1, 1024, 8, 64, 128, 1, "bf16"), 256
    pf, pr = si.make_bidir(shape, seed=7)
    A = pf.A.data.copy()
    A[2] = -60.0                # head pair 1 of the forward layer only
    pf.A.data[:] = A
    ref = oracle.bidir_f64(oracle.params_f64(pf), oracle.params_f64(pr))
    y = ssd.bidir_ssd(_dev(pf), _dev(pr), chunk=chunk)
    torch.cuda.synchronize()
    assert oracle.rel_err(y.double().cpu().numpy(), ref) <= 2e-2
    out = torch.empty_like(y)
    area = ssd.bidir_ssd_noalloc(_dev(pf), _dev(pr), out, chunk=chunk)
    torch.cuda.synchronize()
    ssd.noalloc_status(area)
    assert oracle.rel_err(out.double().cpu().numpy(), ref) <= 2e-2
