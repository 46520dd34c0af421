"""The tracing build of the tensor-core kernel (phase_trace.py).

Its output must equal the product library's bit for bit.  Its per-phase
stamps must come in program order: within a block, MMA stream A issues G
before the state product and stream B Y_off before Y_diag; G waits for the
previous block's Y_diag; each CUDA-core warp passes its phase boundaries in
order.  Every CTA must have recorded a start
before its end.
"""
import pytest
import torch

import ssd_inputs as si

pytestmark = pytest.mark.gpu


def test_trace_build_matches_product_and_orders_phases():
    import bidirectional_mamba_ssd_bidir_b200 as ssd
    from bidirectional_mamba_ssd_bidir_b200 import phase_trace as pt

    # 16 blocks per sequence (more than the traced ones, which all have a successor), 80 CTAs:
    # enough that no sequence is cut into segments, so CTA 0 walks every traced block
    shape = si.Shape(10, 2048, 8, 64, 128, 1, "bf16")
    dims = (shape.batch, shape.seqlen, shape.nheads, shape.headdim, shape.dstate, shape.ngroups)
    assert ssd.segments_for(dims, torch.bfloat16, 256) == 1
    pf, pr = si.make_bidir(shape, seed=3)
    dev = lambda p: {k: getattr(p, k).torch("cuda") for k in ("x", "dt", "A", "B", "C", "D")}
    f, r = dev(pf), dev(pr)
    y_ref = ssd.bidir_ssd(f, r, chunk=256)
    y, ph, ctas = pt.run(f, r, chunk=256)
    torch.cuda.synchronize()
    assert torch.equal(y, y_ref)
    order = [k for k, _ in pt.COMPUTE_POINTS]
    A, Bw = pt.WARP_MMA_A, pt.WARP_MMA_B
    for j in range(1, pt.N_BLOCKS):
        assert ph[A, j, 0] <= ph[A, j, 2], j                 # stream A: G, then the state product
        assert ph[Bw, j, 1] <= ph[Bw, j, 3], j               # stream B: Y_off, then Y_diag
        assert ph[A, j, 0] > ph[Bw, j - 1, 3]                # G waits for the previous block's Y_diag
        for w in range(16):
            seq = [ph[w, j, k] for k in order]
            assert all(a <= b for a, b in zip(seq, seq[1:])), (j, w, seq)
    assert len(ctas) == 2 * shape.batch * shape.nheads // 2
    assert (ctas[:, 1] > ctas[:, 0]).all()
    assert "block 3: period" in pt.summary(ph)


def test_trace_of_a_segmented_call():
    """A call cut into segments: the tracing build still matches the product bit for bit, and the
    CTA table covers every segment's CTA."""
    import bidirectional_mamba_ssd_bidir_b200 as ssd
    from bidirectional_mamba_ssd_bidir_b200 import phase_trace as pt

    shape = si.Shape(1, 2048, 8, 64, 128, 1, "bf16")
    dims = (shape.batch, shape.seqlen, shape.nheads, shape.headdim, shape.dstate, shape.ngroups)
    nseg = ssd.segments_for(dims, torch.bfloat16, 256)
    assert nseg > 1
    pf, pr = si.make_bidir(shape, seed=5)
    dev = lambda p: {k: getattr(p, k).torch("cuda") for k in ("x", "dt", "A", "B", "C", "D")}
    f, r = dev(pf), dev(pr)
    y_ref = ssd.bidir_ssd(f, r, chunk=256)
    y, ph, ctas = pt.run(f, r, chunk=256)
    torch.cuda.synchronize()
    assert torch.equal(y, y_ref)
    assert len(ctas) == shape.batch * shape.nheads * nseg
    assert (ctas[:, 1] > ctas[:, 0]).all()
