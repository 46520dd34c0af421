"""Failure detection on the GPU without faulting it.

The tensor-core bidirectional mixer hands each output block from one
direction to the other through a flag in the workspace, and every wait in the
kernel is bounded.  A test hook makes the first direction skip publishing, so
the other direction's wait runs out: the call must report SSD_ERR_TIMEOUT
through the workspace status word, and the context must stay usable (the next
normal call is correct).  No trap, assert, bad address or endless loop.
"""
import pytest
import torch

import oracle
import ssd_inputs as si

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ssd():
    import bidirectional_mamba_ssd_bidir_b200 as m
    return m


def _dev(p):
    return {k: getattr(p, k).torch("cuda") for k in ("x", "dt", "A", "B", "C", "D")}


def test_handoff_timeout_is_reported_and_recoverable(ssd):
    shape = si.Shape(1, 512, 8, 64, 128, 1, "bf16")
    dims = (1, 512, 8, 64, 128, 1)
    if ssd.path_for(dims, torch.bfloat16, 256) != 1:
        pytest.skip("tensor-core path not available")
    pf, pr = si.make_bidir(shape, seed=3)
    df, dr = _dev(pf), _dev(pr)
    ws = torch.zeros(ssd.workspace_bytes(dims, torch.bfloat16, 256), dtype=torch.uint8, device="cuda")
    try:
        assert ssd.lib.ssd_debug_fault(1, 0.02) == 0
        ssd.bidir_ssd(df, dr, chunk=256, workspace=ws)
        torch.cuda.synchronize()
        with pytest.raises(ssd.SSDError) as ei:
            ssd.workspace_status(ws)
        assert ei.value.status == 4
    finally:
        assert ssd.lib.ssd_debug_fault(0, 2.0) == 0
    # the status word was cleared by the read, and the GPU still computes correctly
    y = ssd.bidir_ssd(df, dr, chunk=256, workspace=ws)
    torch.cuda.synchronize()
    ssd.workspace_status(ws)
    ref = oracle.bidir_f64(oracle.params_f64(pf), oracle.params_f64(pr))
    assert oracle.rel_err(y.double().cpu().numpy(), ref) <= 2e-2


def test_debug_hook_rejects_bad_arguments(ssd):
    assert ssd.lib.ssd_debug_fault(7, 1.0) == 1
    assert ssd.lib.ssd_debug_fault(0, 0.0) == 1
    assert ssd.lib.ssd_debug_fault(0, 2.0) == 0
