"""GPU parity: the CUDA path (through the C ABI) against the float64 oracle on the same seeded inputs.

Metric: max|y - y_ref| / max|y_ref| over the output.  Bars: 2e-2 for bf16 io
(float32 state), 1e-4 for float32 io.  Every bf16/f32 case is checked twice:
on the full output and on the "SSD-only" output (D = None on both sides),
because the skip term D*x dominates |y| and would hide an error in the scan.
"""
import numpy as np
import pytest
import torch

import oracle
import ssd_inputs as si

pytestmark = pytest.mark.gpu

TOL = {"bf16": 2e-2, "f32": 1e-4}


@pytest.fixture(scope="module")
def ssd():
    import bidirectional_mamba_ssd_bidir_b200 as m
    return m


def _dev(p, with_D=True):
    dev = torch.device("cuda")
    d = {k: getattr(p, k).torch(dev) for k in ("x", "dt", "A", "B", "C")}
    d["D"] = p.D.torch(dev) if with_D else None
    return d


def _f64(y):
    return y.detach().double().cpu().numpy()


def _bidir_case(ssd, shape, chunk, with_D, seed=0):
    pf, pr = si.make_bidir(shape, seed=seed, with_D=with_D)
    y = ssd.bidir_ssd(_dev(pf, with_D), _dev(pr, with_D), chunk=chunk)
    torch.cuda.synchronize()
    ref = oracle.bidir_f64(oracle.params_f64(pf), oracle.params_f64(pr))
    return oracle.rel_err(_f64(y), ref)


SHAPES = [
    # (batch, L, H, P, N, G, io), chunk, path the call must take (1 tensor core, 0 SIMT)
    (si.Shape(1, 64, 2, 16, 16, 1, "f32"), 16, 0),            # the tiny float32 workload
    (si.Shape(2, 512, 8, 64, 128, 1, "bf16"), 256, 1),        # layer shape, tensor-core path, 4 blocks
    (si.Shape(1, 128, 8, 64, 128, 1, "bf16"), 128, 1),        # tensor-core path, a single block
    (si.Shape(3, 384, 16, 64, 128, 1, "bf16"), 128, 1),       # tensor-core path, odd block count, 8 head pairs
    (si.Shape(1, 1280, 24, 64, 128, 1, "bf16"), 256, 1),      # tensor-core path, 10 blocks, 12 head pairs
    (si.Shape(1, 768, 6, 64, 128, 1, "bf16"), 256, 0),        # SIMT path (6 heads), odd chunk count
    (si.Shape(3, 384, 4, 64, 128, 1, "bf16"), 128, 0),        # SIMT path, 3 chunks of 128
    (si.Shape(2, 256, 4, 32, 64, 1, "bf16"), 64, 0),
    (si.Shape(1, 256, 4, 16, 16, 1, "bf16"), 16, 0),
    (si.Shape(2, 192, 4, 64, 64, 2, "bf16"), 64, 0),          # two groups
    (si.Shape(1, 96, 3, 16, 32, 1, "f32"), 32, 0),
    (si.Shape(2, 256, 2, 64, 128, 1, "f32"), 128, 0),
]


def _dims(shape):
    return (shape.batch, shape.seqlen, shape.nheads, shape.headdim, shape.dstate, shape.ngroups)


@pytest.mark.parametrize("shape,chunk,path", SHAPES, ids=lambda v: str(v) if isinstance(v, int) else
                         f"b{v.batch}L{v.seqlen}H{v.nheads}P{v.headdim}N{v.dstate}G{v.ngroups}{v.io}")
@pytest.mark.parametrize("with_D", [True, False], ids=["full", "ssd_only"])
def test_bidir_parity(ssd, shape, chunk, path, with_D):
    io = torch.bfloat16 if shape.io == "bf16" else torch.float32
    assert ssd.path_for(_dims(shape), io, chunk) == path
    err = _bidir_case(ssd, shape, chunk, with_D)
    assert err <= TOL[shape.io], f"rel err {err:.3e}"


@pytest.mark.parametrize("direction", [1, -1])
@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_single_direction_parity(ssd, direction, io):
    shape = si.Shape(2, 512, 8, 64, 128, 1, io)
    p = si.make_params(shape, seed=3, with_D=False)
    y = ssd.ssd_scan(**_dev(p, False), direction=direction, chunk=128)
    torch.cuda.synchronize()
    q = oracle.params_f64(p)
    ref = oracle.ssd_scan_f64(q["x"], q["dt"], q["A"], q["B"], q["C"], None, direction)
    assert oracle.rel_err(_f64(y), ref) <= TOL[io]


@pytest.mark.parametrize("chunk", [16, 32, 64, 128, 256])
def test_chunk_size_invariance(ssd, chunk):
    shape = si.Shape(1, 512, 8, 64, 128, 1, "bf16")
    err = _bidir_case(ssd, shape, chunk, with_D=False, seed=5)
    assert err <= TOL["bf16"]


def _flip(p):
    q = {}
    for k, v in p.items():
        q[k] = v.flip(1).contiguous() if (v is not None and k in ("x", "dt", "B", "C")) else v
    return q


@pytest.mark.parametrize("io,chunk", [("f32", 16), ("bf16", 64), ("bf16", 256)])
def test_reverse_is_flip_forward_flip(ssd, io, chunk):
    shape = si.Shape(2, 512, 8, 64, 128, 1, io)
    p = _dev(si.make_params(shape, seed=6))
    yr = ssd.ssd_scan(**p, direction=-1, chunk=chunk)
    yf = ssd.ssd_scan(**_flip(p), direction=1, chunk=chunk).flip(1)
    torch.cuda.synchronize()
    if ssd.path_for((2, 512, 8, 64, 128, 1), p["x"].dtype, chunk) == 0:
        assert torch.equal(yr, yf)      # same arithmetic in scan order: bit for bit
    else:
        assert oracle.rel_err(_f64(yr), _f64(yf)) <= 1e-2


@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_bidir_is_sum_of_directions(ssd, io):
    shape = si.Shape(2, 512, 8, 64, 128, 1, io)
    pf, pr = si.make_bidir(shape, seed=8)
    df, dr = _dev(pf), _dev(pr)
    yb = ssd.bidir_ssd(df, dr, chunk=128).double()
    yf = ssd.ssd_scan(**df, direction=1, chunk=128).double()
    yr = ssd.ssd_scan(**dr, direction=-1, chunk=128).double()
    torch.cuda.synchronize()
    s = yf + yr
    if io == "f32":
        assert torch.max(torch.abs(yb - s)).item() <= 1e-5 * torch.max(torch.abs(s)).item()
    else:
        # two roundings to bf16 (8-bit significand) on each side
        bound = 2.0 ** -7 * torch.maximum(torch.maximum(yf.abs(), yr.abs()), s.abs())
        assert bool(torch.all(torch.abs(yb - s) <= bound))


def test_dt_zero_gives_skip_term_bitwise(ssd):
    shape = si.Shape(1, 128, 8, 64, 128, 1, "f32")
    p = _dev(si.make_params(shape, seed=9))
    p["dt"] = torch.zeros_like(p["dt"])
    for d in (1, -1):
        y = ssd.ssd_scan(**p, direction=d, chunk=64)
        torch.cuda.synchronize()
        assert torch.equal(y, p["D"][None, None, :, None] * p["x"])


def test_dt_zero_tensor_core_path(ssd):
    """dt = 0 on the tensor-core path: the state never moves, y = bf16(D x)."""
    shape = si.Shape(1, 256, 8, 64, 128, 1, "bf16")
    p = _dev(si.make_params(shape, seed=9))
    p["dt"] = torch.zeros_like(p["dt"])
    for d in (1, -1):
        y = ssd.ssd_scan(**p, direction=d, chunk=128)
        torch.cuda.synchronize()
        ref = (p["D"][None, None, :, None] * p["x"].float()).to(torch.bfloat16)
        assert torch.equal(y, ref)


def test_steep_decay(ssd):
    """Decays steep enough that a 16-token window falls below 2^-120 (dt = 3, A = -16 on even
    heads): the tensor-core path's factorised decay mask must switch to its exact form there."""
    shape = si.Shape(1, 512, 8, 64, 128, 1, "bf16")
    p = si.make_params(shape, seed=21, with_D=False)
    q = oracle.params_f64(p)
    q["dt"][:, 40:56, :] = 3.0          # inside one 16-row sub-block of the first block
    q["dt"][:, 300:340, :] = 2.0        # across sub-block and quarter boundaries of the third block
    q["A"][0::2] = -16.0
    dev = torch.device("cuda")
    d = {"x": p.x.torch(dev), "dt": torch.from_numpy(q["dt"]).to(dev, torch.bfloat16),
         "A": torch.from_numpy(q["A"]).to(dev, torch.float32), "B": p.B.torch(dev), "C": p.C.torch(dev), "D": None}
    for direction in (1, -1):
        y = ssd.ssd_scan(**d, direction=direction, chunk=256)
        torch.cuda.synchronize()
        assert torch.isfinite(y.float()).all()
        ref = oracle.ssd_scan_f64(q["x"], q["dt"], q["A"], q["B"], q["C"], None, direction)
        assert oracle.rel_err(_f64(y), ref) <= TOL["bf16"], direction


def test_paths_agree(ssd):
    """The tensor-core path (chunk 128) and the SIMT path (chunk 64) on the same inputs."""
    shape = si.Shape(2, 512, 8, 64, 128, 1, "bf16")
    dims = (2, 512, 8, 64, 128, 1)
    assert ssd.path_for(dims, torch.bfloat16, 64) == 0
    pf, pr = si.make_bidir(shape, seed=12, with_D=False)
    df, dr = _dev(pf, False), _dev(pr, False)
    a = ssd.bidir_ssd(df, dr, chunk=128).double()
    b = ssd.bidir_ssd(df, dr, chunk=64).double()
    torch.cuda.synchronize()
    assert oracle.rel_err(a.cpu().numpy(), b.cpu().numpy()) <= 2e-2


def test_deterministic(ssd):
    shape = si.Shape(2, 512, 8, 64, 128, 1, "bf16")
    pf, pr = si.make_bidir(shape, seed=10)
    df, dr = _dev(pf), _dev(pr)
    y1 = ssd.bidir_ssd(df, dr, chunk=256)
    y2 = ssd.bidir_ssd(df, dr, chunk=256)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)


@pytest.mark.parametrize("dims,chunk", [((2, 512, 8, 64, 128, 1), 256), ((2, 256, 4, 32, 64, 1), 64)],
                         ids=["tensor_core", "simt"])
def test_output_canaries(ssd, dims, chunk):
    """The kernels write exactly the output tensor: sentinel words before and after it survive."""
    shape = si.Shape(*dims, "bf16")
    pf, pr = si.make_bidir(shape, seed=14)
    df, dr = _dev(pf), _dev(pr)
    n, pad = df["x"].numel(), 8192
    buf = torch.full((n + 2 * pad,), float("nan"), dtype=torch.bfloat16, device="cuda")
    sentinel = buf[:pad].clone()
    y = buf[pad:pad + n].view(df["x"].shape)
    ssd.bidir_ssd(df, dr, chunk=chunk, out=y)
    torch.cuda.synchronize()
    assert torch.equal(buf[:pad].view(torch.int16), sentinel.view(torch.int16))
    assert torch.equal(buf[pad + n:].view(torch.int16), sentinel.view(torch.int16))
    assert torch.isfinite(y.float()).all()


def test_empty_batch(ssd):
    shape = si.Shape(0, 256, 4, 64, 128, 1, "bf16")
    x = torch.empty(0, 256, 4, 64, dtype=torch.bfloat16, device="cuda")
    B = torch.empty(0, 256, 1, 128, dtype=torch.bfloat16, device="cuda")
    dt = torch.empty(0, 256, 4, dtype=torch.bfloat16, device="cuda")
    A = -torch.ones(4, device="cuda")
    y = ssd.ssd_scan(x, dt, A, B, B, None, 1, 256)
    assert y.shape == x.shape


def test_refuses_unsupported_shape(ssd):
    x = torch.zeros(1, 64, 2, 48, dtype=torch.bfloat16, device="cuda")
    B = torch.zeros(1, 64, 1, 16, dtype=torch.bfloat16, device="cuda")
    dt = torch.zeros(1, 64, 2, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ssd.SSDError):
        ssd.ssd_scan(x, dt, -torch.ones(2, device="cuda"), B, B, None, 1, 16)


# ------------------------------------------------------------------ R2L sidecar

def _r2l_step(ssd, shape, chunk, step, s=None):
    p = si.make_params(shape, seed=0, offset=si.STEP_STRIDE * step + si.REV_OFFSET)
    res = si.make_residual(shape, seed=0, step=step)
    gate = si.make_gate(0, step) if s is None else s
    out = ssd.r2l_block_scan(_dev(p), gate, res.torch("cuda"), chunk=chunk)
    torch.cuda.synchronize()
    return p, res, gate, out


def test_r2l_gate_zero_is_bit_identical(ssd):
    shape = si.WORKLOADS["r2l_block_L32"]["shape"]
    p, res, _, out = _r2l_step(ssd, shape, 32, 0, s=0.0)
    assert torch.equal(out.cpu().view(torch.int16), res.torch().view(torch.int16))
    # in place: out is the residual buffer itself
    r = res.torch("cuda")
    ref = r.clone()
    o = ssd.r2l_block_scan(_dev(p), 0.0, r, chunk=32, out=r)
    torch.cuda.synchronize()
    assert torch.equal(o.view(torch.int16), ref.view(torch.int16))


@pytest.mark.parametrize("chunk", [32, 16])
def test_r2l_block_parity(ssd, chunk):
    """Full output against the oracle, then the scan alone: zero residual and no D, so out = s * y_rev."""
    shape = si.WORKLOADS["r2l_block_L32"]["shape"]
    for step in range(4):
        p, res, gate, out = _r2l_step(ssd, shape, chunk, step)
        ref = oracle.r2l_block_f64(oracle.params_f64(p), gate, res.f64())
        assert oracle.rel_err(_f64(out), ref) <= TOL["bf16"]
        q = si.make_params(shape, seed=0, offset=si.STEP_STRIDE * step + si.REV_OFFSET, with_D=False)
        zero = torch.zeros(shape.batch, shape.seqlen, shape.nheads * shape.headdim,
                           dtype=torch.bfloat16, device="cuda")
        o2 = ssd.r2l_block_scan(_dev(q, False), gate, zero, chunk=chunk)
        torch.cuda.synchronize()
        ref2 = oracle.r2l_block_f64(oracle.params_f64(q), gate, np.zeros(zero.shape))
        assert oracle.rel_err(_f64(o2), ref2) <= TOL["bf16"]


def test_homogeneous_in_x_bitwise_tensor_core(ssd):
    """y is linear in x.  Doubling x doubles every bf16 operand and float32 partial sum exactly,
    so on the tensor-core path y(2x) is 2 y(x) bit for bit, in both directions and for the sum."""
    shape = si.Shape(2, 512, 8, 64, 128, 1, "bf16")
    pf, pr = si.make_bidir(shape, seed=12)
    df, dr = _dev(pf), _dev(pr)
    df2, dr2 = dict(df, x=df["x"] * 2), dict(dr, x=dr["x"] * 2)
    for d in (1, -1):
        p, p2 = (df, df2) if d > 0 else (dr, dr2)
        y, y2 = ssd.ssd_scan(**p, direction=d, chunk=256), ssd.ssd_scan(**p2, direction=d, chunk=256)
        torch.cuda.synchronize()
        assert torch.equal(y2, y * 2)
    yb, yb2 = ssd.bidir_ssd(df, dr, chunk=256), ssd.bidir_ssd(df2, dr2, chunk=256)
    torch.cuda.synchronize()
    assert torch.equal(yb2, yb * 2)


def test_additive_in_x_float32(ssd):
    """y(a x1 + b x2) = a y(x1) + b y(x2) for fixed dt, A, B, C, D, on the float32 path."""
    shape = si.Shape(1, 256, 4, 32, 64, 1, "f32")
    p1 = _dev(si.make_params(shape, seed=13))
    x2 = _dev(si.make_params(shape, seed=14))["x"]
    a, b = 0.75, -1.5
    for d in (1, -1):
        y1 = ssd.ssd_scan(**p1, direction=d, chunk=64)
        y2 = ssd.ssd_scan(**dict(p1, x=x2), direction=d, chunk=64)
        y3 = ssd.ssd_scan(**dict(p1, x=a * p1["x"] + b * x2), direction=d, chunk=64)
        torch.cuda.synchronize()
        ref = a * y1.double() + b * y2.double()
        assert torch.max(torch.abs(y3.double() - ref)).item() <= 1e-5 * torch.max(torch.abs(ref)).item()


@pytest.mark.parametrize("dims,chunk", [((2, 1024, 8, 64, 128, 1), 256), ((1, 256, 4, 32, 64, 1), 64)])
def test_workspace_needs_only_its_status_word_zeroed(ssd, dims, chunk):
    """Apart from the status word (first 256 bytes), a workspace may hold anything before a call:
    the hand-off flags are epoch-tagged and the chunk states are written before they are read."""
    shape = si.Shape(*dims, "bf16")
    pf, pr = si.make_bidir(shape, seed=15)
    df, dr = _dev(pf), _dev(pr)
    n = ssd.workspace_bytes(dims, torch.bfloat16, chunk)
    clean = torch.zeros(n, dtype=torch.uint8, device="cuda")
    y_ref = ssd.bidir_ssd(df, dr, chunk=chunk, workspace=clean)
    for fill in (0xFF, 0xA5):
        ws = torch.full((n,), fill, dtype=torch.uint8, device="cuda")
        ws[:256] = 0
        for _ in range(2):
            y = ssd.bidir_ssd(df, dr, chunk=chunk, workspace=ws)
            torch.cuda.synchronize()
            ssd.workspace_status(ws)
            assert torch.equal(y, y_ref)


ONE_CHUNK = [
    # sequences of one chunk (seqlen == chunk <= 64) with no state: the single-chunk kernel
    (si.Shape(2, 16, 3, 16, 16, 1, "f32"), 16),
    (si.Shape(2, 32, 4, 64, 128, 2, "f32"), 32),
    (si.Shape(3, 64, 4, 64, 128, 1, "bf16"), 64),
    (si.Shape(1, 64, 6, 32, 64, 3, "bf16"), 64),
    (si.Shape(2, 32, 5, 16, 128, 1, "bf16"), 32),
]


@pytest.mark.parametrize("shape,chunk", ONE_CHUNK, ids=lambda v: str(v) if isinstance(v, int) else
                         f"b{v.batch}L{v.seqlen}H{v.nheads}P{v.headdim}N{v.dstate}G{v.ngroups}{v.io}")
def test_single_chunk_calls(ssd, shape, chunk):
    """Every output mode of a one-chunk call: each direction alone (write), the bidirectional sum
    (write, then add) and the R2L gate (residual + s y_rev), with and without the skip term."""
    io = torch.bfloat16 if shape.io == "bf16" else torch.float32
    assert ssd.path_for(_dims(shape), io, chunk) == 0
    tol = TOL[shape.io]
    for with_D in (True, False):
        assert _bidir_case(ssd, shape, chunk, with_D, seed=21) <= tol
        p = si.make_params(shape, seed=22, with_D=with_D)
        q = oracle.params_f64(p)
        for direction in (1, -1):
            y = ssd.ssd_scan(**_dev(p, with_D), direction=direction, chunk=chunk)
            torch.cuda.synchronize()
            ref = oracle.ssd_scan_f64(q["x"], q["dt"], q["A"], q["B"], q["C"], q.get("D"), direction)
            assert oracle.rel_err(_f64(y), ref) <= tol, (with_D, direction)
        gate = 0.37
        res = si.make_residual(shape, seed=23)
        for r_dev, r_ref in ((res.torch("cuda"), res.f64()),
                             (torch.zeros(res.torch().shape, dtype=io, device="cuda"), np.zeros(res.torch().shape))):
            out = ssd.r2l_block_scan(_dev(p, with_D), gate, r_dev, chunk=chunk)
            torch.cuda.synchronize()
            assert oracle.rel_err(_f64(out), oracle.r2l_block_f64(q, gate, r_ref)) <= tol, with_D
