"""GPU parity of ssd_scan_bwd: the scan's gradients against the float64 oracle.

The oracle takes the reverse-mode derivative of the recurrence position by
position (and is itself pinned by central differences and exact identities on
the CPU); the GPU evaluates the same derivatives in chunked form in float32.
Inputs are the exact stored bf16/float32 values, so the only differences are
float32 rounding.  Metric per gradient: max|g - g_ref| / max|g_ref|; bars
1e-3 (bf16 inputs, long float32 sums) and 1e-4 (float32 io, short sums).
"""
import numpy as np
import pytest
import torch

import oracle
import ssd_inputs as si

pytestmark = pytest.mark.gpu

TOL = {"bf16": 1e-3, "f32": 1e-4}

CASES = [
    (si.Shape(1, 64, 2, 16, 16, 1, "f32"), 16),
    (si.Shape(1, 96, 3, 16, 32, 1, "f32"), 32),
    (si.Shape(2, 256, 4, 64, 128, 1, "bf16"), 256),     # 4 chunks of 64
    (si.Shape(2, 192, 4, 32, 64, 2, "bf16"), 64),       # two groups
    (si.Shape(1, 1024, 2, 64, 128, 1, "bf16"), 128),    # 16 chunks
    (si.Shape(1, 128, 2, 64, 16, 1, "f32"), 32),         # wide x, narrow state, 32-position chunks
    (si.Shape(1, 48, 2, 32, 128, 1, "bf16"), 16),        # 16-position chunks, wide state
    # tensor-core shapes (bf16, P 64, N 128, heads a multiple of 8): 128-position chunks on tcgen05
    (si.Shape(2, 256, 8, 64, 128, 1, "bf16"), 256),     # 2 chunks
    (si.Shape(1, 1024, 8, 64, 128, 1, "bf16"), 128),    # 8 chunks
    (si.Shape(1, 384, 16, 64, 128, 1, "bf16"), 128),    # 3 chunks, 16 heads
]


@pytest.fixture(scope="module")
def ssd():
    import bidirectional_mamba_ssd_bidir_b200 as m
    return m


def _ids(v):
    return f"b{v.batch}L{v.seqlen}H{v.nheads}P{v.headdim}N{v.dstate}G{v.ngroups}{v.io}" if isinstance(v, si.Shape) \
        else str(v)


@pytest.mark.parametrize("shape,chunk", CASES, ids=_ids)
@pytest.mark.parametrize("direction", [1, -1])
@pytest.mark.parametrize("with_D", [True, False], ids=["D", "noD"])
def test_gradients_match_oracle(ssd, shape, chunk, direction, with_D):
    dims = (shape.batch, shape.seqlen, shape.nheads, shape.headdim, shape.dstate, shape.ngroups)
    tc = shape.io == "bf16" and shape.headdim == 64 and shape.dstate == 128 and shape.ngroups == 1 and \
        shape.nheads % 8 == 0 and chunk % 128 == 0
    assert ssd.path_for(dims, torch.bfloat16 if shape.io == "bf16" else torch.float32, chunk) == (1 if tc else 0)
    p = si.make_params(shape, seed=41, with_D=with_D)
    dev = torch.device("cuda")
    d = {k: getattr(p, k).torch(dev) for k in ("x", "dt", "A", "B", "C")}
    d["D"] = p.D.torch(dev) if with_D else None
    rng = np.random.default_rng(7)
    gy64 = rng.standard_normal(p.x.shape)
    gy = torch.from_numpy(gy64).to(dev, torch.bfloat16 if shape.io == "bf16" else torch.float32)
    gy64 = gy.double().cpu().numpy()          # the exact stored values
    g = ssd.ssd_scan_bwd(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], gy, direction=direction, chunk=chunk)
    torch.cuda.synchronize()
    q = oracle.params_f64(p)
    ref = oracle.ssd_scan_bwd_f64(q["x"], q["dt"], q["A"], q["B"], q["C"], q["D"] if with_D else None,
                                  direction, gy64)
    for name in ("x", "dt", "A", "B", "C") + (("D",) if with_D else ()):
        err = oracle.rel_err(g[name].double().cpu().numpy(), ref[name])
        assert err <= TOL[shape.io], (name, err)


def test_bidirectional_gradient_is_the_sum_of_directions(ssd):
    """y = y_fwd + y_rev with the same inputs: the gradient wrt x is the sum of the two directions'."""
    shape = si.Shape(1, 256, 2, 64, 128, 1, "bf16")
    p = si.make_params(shape, seed=42)
    d = {k: getattr(p, k).torch("cuda") for k in ("x", "dt", "A", "B", "C", "D")}
    gy = torch.randn(d["x"].shape, device="cuda").to(torch.bfloat16)
    gf = ssd.ssd_scan_bwd(**d, gy=gy, direction=1, chunk=256)
    gr = ssd.ssd_scan_bwd(**d, gy=gy, direction=-1, chunk=256)
    torch.cuda.synchronize()
    q = oracle.params_f64(p)
    g64 = gy.double().cpu().numpy()
    rf = oracle.ssd_scan_bwd_f64(q["x"], q["dt"], q["A"], q["B"], q["C"], q["D"], 1, g64)
    rr = oracle.ssd_scan_bwd_f64(q["x"], q["dt"], q["A"], q["B"], q["C"], q["D"], -1, g64)
    got = (gf["x"] + gr["x"]).double().cpu().numpy()
    assert oracle.rel_err(got, rf["x"] + rr["x"]) <= TOL["bf16"]


def test_empty_inputs_give_zero_parameter_gradients(ssd):
    """No token: dA and dD are zero (dx, ddt, dB, dC are empty)."""
    for b, L in ((0, 256), (2, 0)):
        x = torch.empty(b, L, 4, 64, dtype=torch.bfloat16, device="cuda")
        dt = torch.empty(b, L, 4, dtype=torch.bfloat16, device="cuda")
        B = torch.empty(b, L, 1, 128, dtype=torch.bfloat16, device="cuda")
        A = -torch.ones(4, device="cuda")
        D = torch.ones(4, device="cuda")
        g = ssd.ssd_scan_bwd(x, dt, A, B, B, D, torch.empty_like(x), direction=1, chunk=256)
        torch.cuda.synchronize()
        assert torch.equal(g["A"], torch.zeros(4, device="cuda"))
        assert torch.equal(g["D"], torch.zeros(4, device="cuda"))
        assert g["x"].numel() == 0 and g["B"].numel() == 0


def test_gradients_at_the_bench_layer_shape(ssd):
    """The 1.3B layer shape at L = 8192 (one sequence of the bench workload), forward direction,
    every gradient against the oracle's adjoint over the whole sequence (about half a minute of
    single-threaded oracle; the reverse direction is covered at smaller sizes)."""
    direction = 1
    shape = si.Shape(1, 8192, 64, 64, 128, 1, "bf16")
    assert ssd.path_for((1, 8192, 64, 64, 128, 1), torch.bfloat16, 256) == 1       # tensor-core gradients
    p = si.make_params(shape, seed=43)
    d = {k: getattr(p, k).torch("cuda") for k in ("x", "dt", "A", "B", "C", "D")}
    gy = torch.randn(d["x"].shape, device="cuda", generator=torch.Generator("cuda").manual_seed(5)).to(torch.bfloat16)
    g = ssd.ssd_scan_bwd(**d, gy=gy, direction=direction, chunk=256)
    torch.cuda.synchronize()
    q = oracle.params_f64(p)
    ref = oracle.ssd_scan_bwd_f64(q["x"], q["dt"], q["A"], q["B"], q["C"], q["D"], direction,
                                  gy.double().cpu().numpy())
    for name in ("x", "dt", "A", "B", "C", "D"):
        err = oracle.rel_err(g[name].double().cpu().numpy(), ref[name])
        assert err <= TOL["bf16"], (name, err)
