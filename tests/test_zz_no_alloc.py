"""bidir_ssd_noalloc: the bidirectional mixer without a caller-supplied workspace.

Some callers cannot allocate device memory at the point of the call: a host
program that has handed out all of its device memory up front, or a
latency-bound loop that cannot afford cudaMalloc/cudaFree (which may
synchronise the whole device).  For them the library keeps the scratch in a
fixed array of its own.  These tests call that entry point through the C ABI
and check it against bidir_ssd (caller workspace) on the same inputs, twice in
a row, so the second call also shows that the scratch left by the first one is
cleared correctly.  The file is named to be collected last, and passes on its
own in a fresh process as well as after the rest of the suite.
"""
import pytest
import torch

import oracle
import ssd_inputs as si

pytestmark = pytest.mark.gpu

# max |y_noalloc - y_workspace| / max |y_workspace|: both sides run the same
# kernels in float32 and round to bf16 once; the order in which the forward
# and reverse halves are added may differ, which moves a value by at most one
# bf16 rounding step of the sum.
TOL = 1e-2


@pytest.fixture(scope="module")
def ssd():
    import bidirectional_mamba_ssd_bidir_b200 as m
    return m


def _dev(p):
    return {k: getattr(p, k).torch("cuda") for k in ("x", "dt", "A", "B", "C", "D")}


def _rel(a, b):
    return ((a.float() - b.float()).abs().max() / b.float().abs().max().clamp_min(1e-30)).item()


@pytest.mark.parametrize("dims,chunk", [
    ((2, 1024, 8, 64, 128, 1), 256),     # tensor-core path, 8 blocks of 128 rows per sequence
    ((1, 384, 4, 64, 128, 1), 128),      # tensor-core path, 3 blocks
    ((2, 96, 4, 32, 64, 1), 32),         # SIMT path (headdim 32), three chunks
])
def test_matches_workspace_entry_point_twice(ssd, dims, chunk):
    shape = si.Shape(*dims, "bf16")
    pf, pr = si.make_bidir(shape, seed=11)
    f, r = _dev(pf), _dev(pr)
    ws = torch.zeros(ssd.workspace_bytes(dims, torch.bfloat16, chunk), dtype=torch.uint8, device="cuda")
    y_ref = ssd.bidir_ssd(f, r, chunk=chunk, workspace=ws)
    torch.cuda.synchronize()
    ssd.workspace_status(ws)

    out = torch.empty_like(f["x"])
    for call in range(2):
        out.fill_(float("nan"))
        area = ssd.bidir_ssd_noalloc(f, r, out, chunk=chunk)
        torch.cuda.synchronize()
        ssd.noalloc_status(area)
        assert torch.isfinite(out.float()).all(), f"call {call}: output not fully written"
        assert _rel(out, y_ref) <= TOL, f"call {call}"

    # and both agree with the float64 oracle on one (batch, head) slice
    q = oracle.params_f64(pf), oracle.params_f64(pr)
    def sl(d):   # batch 0, head 0 (x, dt: [b, L, H, ...]; A, D: [H]; B, C: [b, L, G, N] with G = 1)
        return {k: None if v is None else v[0:1, :, 0:1] if k in ("x", "dt") else v[0:1] for k, v in d.items()}
    ref = oracle.bidir_f64(sl(q[0]), sl(q[1]))
    assert oracle.rel_err(out[0:1, :, 0:1].double().cpu().numpy(), ref) <= 2e-2


def test_allocates_nothing_through_torch(ssd):
    dims, chunk = (1, 512, 8, 64, 128, 1), 256
    pf, pr = si.make_bidir(si.Shape(*dims, "bf16"), seed=5)
    f, r = _dev(pf), _dev(pr)
    out = torch.empty_like(f["x"])
    ssd.bidir_ssd_noalloc(f, r, out, chunk=chunk)      # first call on this device: looks up the scratch
    torch.cuda.synchronize()
    before = (torch.cuda.memory_allocated(), torch.cuda.memory_reserved())
    area = ssd.bidir_ssd_noalloc(f, r, out, chunk=chunk)
    torch.cuda.synchronize()
    assert (torch.cuda.memory_allocated(), torch.cuda.memory_reserved()) == before
    ssd.noalloc_status(area)


def test_refuses_shapes_beyond_the_scratch(ssd):
    # tensor-core path: 64 heads x 2048 blocks of 128 rows, 16 B of hand-off flags each, is
    # 2 MiB plus the status area; the SIMT path's chunk states would need far more
    dims, chunk = (1, 262144, 64, 64, 128, 1), 256
    assert ssd.workspace_bytes(dims, torch.bfloat16, chunk) > 2 << 20
    shape = ssd._Shape(*dims, ssd.SSD_BF16)
    prm = ssd._Params(16, 16, 16, 16, 16, None)     # never dereferenced: the size check comes first
    area = ssd.ctypes.c_void_p()
    st = ssd.lib.bidir_ssd_noalloc(ssd.ctypes.byref(shape), ssd.ctypes.byref(prm), ssd.ctypes.byref(prm),
                                   chunk, 16, None, ssd.ctypes.byref(area))
    assert st == 2 and area.value is None
    assert "bidir_ssd with a workspace" in ssd.lib.ssd_last_error().decode()
