"""Full-size workloads on the GPU, in the launch configuration the bench times, checked on sampled outputs.

The oracle cannot afford a whole 1.3B-layer-shape call in a test, so for a few
sampled (batch, head) pairs it recomputes the full sequence of both
directions from the same stored inputs and the GPU output is compared on
those slices, full output and SSD-only (D = None).  The R2L sidecar workload
is small enough to check every step.
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


def _slice(q: dict, b: int, h: int, G: int, H: int) -> dict:
    g = h // (H // G)
    return {"x": q["x"][b:b + 1, :, h:h + 1], "dt": q["dt"][b:b + 1, :, h:h + 1], "A": q["A"][h:h + 1],
            "B": q["B"][b:b + 1, :, g:g + 1], "C": q["C"][b:b + 1, :, g:g + 1],
            "D": None if q["D"] is None else q["D"][h:h + 1]}


def _pairs(shape, k=3, seed=1):
    rng = np.random.default_rng(seed)
    pairs = {(0, 0), (shape.batch - 1, shape.nheads - 1)}
    while len(pairs) < k + 2:
        pairs.add((int(rng.integers(shape.batch)), int(rng.integers(shape.nheads))))
    return sorted(pairs)


@pytest.mark.parametrize("name", ["diffumamba_240m_L2048", "diffumamba_1p3b_L8192", "long_L32768", "long_L131072"])
def test_fullsize_sampled(ssd, name):
    w = si.WORKLOADS[name]
    shape, chunk = w["shape"], w["chunk"]
    for with_D in (True, False):
        pf, pr = si.make_bidir(shape, seed=0, with_D=with_D)
        y = ssd.bidir_ssd(_dev(pf, with_D), _dev(pr, with_D), chunk=chunk)
        torch.cuda.synchronize()
        qf, qr = oracle.params_f64(pf), oracle.params_f64(pr)
        for (b, h) in _pairs(shape):
            ref = oracle.bidir_f64(_slice(qf, b, h, shape.ngroups, shape.nheads),
                                   _slice(qr, b, h, shape.ngroups, shape.nheads))
            got = y[b:b + 1, :, h:h + 1].double().cpu().numpy()
            err = oracle.rel_err(got, ref)
            assert err <= 2e-2, f"{name} D={with_D} (b={b}, h={h}): rel err {err:.3e}"
        del y
        torch.cuda.empty_cache()


def test_r2l_workload_all_steps(ssd):
    """The R2L sidecar decode workload: 256 denoising steps, fresh seeded inputs per step.

    Each step is checked twice: the full output (residual + gate * reverse scan), and the scan
    alone (zero residual and no D), where the SSD term is the whole output and cannot hide
    behind the residual."""
    w = si.WORKLOADS["r2l_block_L32"]
    shape, chunk = w["shape"], w["chunk"]
    zero = torch.zeros(shape.batch, shape.seqlen, shape.nheads * shape.headdim, dtype=torch.bfloat16, device="cuda")
    zero64 = np.zeros(zero.shape)
    worst = worst_ssd = 0.0
    for step in range(w["steps"]):
        p = si.make_params(shape, seed=0, offset=si.STEP_STRIDE * step + si.REV_OFFSET)
        res = si.make_residual(shape, seed=0, step=step)
        gate = si.make_gate(0, step)
        out = ssd.r2l_block_scan(_dev(p), gate, res.torch("cuda"), chunk=chunk)
        ref = oracle.r2l_block_f64(oracle.params_f64(p), gate, res.f64())
        worst = max(worst, oracle.rel_err(out.double().cpu().numpy(), ref))
        q = si.make_params(shape, seed=0, offset=si.STEP_STRIDE * step + si.REV_OFFSET, with_D=False)
        o2 = ssd.r2l_block_scan(_dev(q, False), gate, zero, chunk=chunk)
        ref2 = oracle.r2l_block_f64(oracle.params_f64(q), gate, zero64)
        if gate != 0:
            worst_ssd = max(worst_ssd, oracle.rel_err(o2.double().cpu().numpy(), ref2))
        else:
            assert not o2.any(), f"step {step}: gate 0 must give the zero residual back"
    assert worst <= 2e-2
    assert worst_ssd <= 2e-2
