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


@pytest.mark.parametrize("dims,chunk,path", [
    ((2, 1024, 8, 64, 128, 1), 256, 1),     # tensor-core path, 8 blocks of 128 rows per sequence
    ((1, 384, 8, 64, 128, 1), 128, 1),      # tensor-core path, 3 blocks
    ((1, 384, 4, 64, 128, 1), 128, 0),      # SIMT path (4 heads), 3 chunks
    ((2, 96, 4, 32, 64, 1), 32, 0),         # SIMT path (headdim 32), three chunks
])
def test_matches_workspace_entry_point_twice(ssd, dims, chunk, path):
    assert ssd.path_for(dims, torch.bfloat16, chunk) == path
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


def test_allocates_nothing(ssd):
    dims, chunk = (1, 512, 8, 64, 128, 1), 256
    assert ssd.path_for(dims, torch.bfloat16, chunk) == 1
    pf, pr = si.make_bidir(si.Shape(*dims, "bf16"), seed=5)
    f, r = _dev(pf), _dev(pr)
    out = torch.empty_like(f["x"])
    ssd.bidir_ssd_noalloc(f, r, out, chunk=chunk)      # first call on this device: loads the kernels
    torch.cuda.synchronize()
    before = (torch.cuda.memory_allocated(), torch.cuda.memory_reserved())
    free_before = torch.cuda.mem_get_info()[0]          # cudaMemGetInfo: sees any cudaMalloc, not only torch's
    area = ssd.bidir_ssd_noalloc(f, r, out, chunk=chunk)
    torch.cuda.synchronize()
    free_after = torch.cuda.mem_get_info()[0]
    assert (torch.cuda.memory_allocated(), torch.cuda.memory_reserved()) == before
    # device allocations come in pages of at least 2 MiB: any allocation would show
    assert free_before - free_after < (2 << 20), (free_before, free_after)
    ssd.noalloc_status(area)


# Runs without torch: two driver-API contexts on the same device, one after the other, each
# with its own buffers.  In each, the no-allocation call must match bidir_ssd with a workspace:
# the scratch's address is the one in the context current at the call, not a leftover from the
# first context (whose memory is gone once that context is destroyed).
_TWO_CONTEXTS = r"""
import ctypes, sys
import numpy as np
root = sys.argv[1]
sys.path.insert(0, root)
import ssd_inputs as si

cu = ctypes.CDLL("libcuda.so.1")
U64, VP = ctypes.c_uint64, ctypes.c_void_p
cu.cuCtxCreate_v2.argtypes = [ctypes.POINTER(VP), ctypes.c_uint, ctypes.c_int]
cu.cuCtxDestroy_v2.argtypes = [VP]
cu.cuMemAlloc_v2.argtypes = [ctypes.POINTER(U64), ctypes.c_size_t]
cu.cuMemFree_v2.argtypes = [U64]
cu.cuMemcpyHtoD_v2.argtypes = [U64, VP, ctypes.c_size_t]
cu.cuMemcpyDtoH_v2.argtypes = [VP, U64, ctypes.c_size_t]
cu.cuMemsetD8_v2.argtypes = [U64, ctypes.c_ubyte, ctypes.c_size_t]

def ck(rc, what):
    if rc != 0:
        raise SystemExit(f"{what} returned {rc}")

ck(cu.cuInit(0), "cuInit")
dev = ctypes.c_int()
ck(cu.cuDeviceGet(ctypes.byref(dev), 0), "cuDeviceGet")

lib = ctypes.CDLL(root + "/bidirectional_mamba_ssd_bidir_b200/libbidirssd.so")
class Shape(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in ("batch", "seqlen", "nheads", "headdim", "dstate", "ngroups", "io")]
class Params(ctypes.Structure):
    _fields_ = [(n, VP) for n in ("x", "dt", "A", "B", "C", "D")]
PS, PP = ctypes.POINTER(Shape), ctypes.POINTER(Params)
lib.ssd_workspace_bytes.argtypes = [PS, ctypes.c_int]
lib.ssd_workspace_bytes.restype = ctypes.c_size_t
lib.bidir_ssd.argtypes = [PS, PP, PP, ctypes.c_int, VP, VP, ctypes.c_size_t, VP]
lib.bidir_ssd_noalloc.argtypes = [PS, PP, PP, ctypes.c_int, VP, VP, ctypes.POINTER(VP)]
lib.ssd_workspace_status.argtypes = [VP, ctypes.c_size_t, VP]
lib.ssd_last_error.restype = ctypes.c_char_p

dims, chunk = (2, 384, 8, 64, 128, 1), 128
pf, pr = si.make_bidir(si.Shape(*dims, "bf16"), seed=17)
sh = Shape(*dims, 0)
ny = dims[0] * dims[1] * dims[2] * dims[3]

def one_context():
    ctx = VP()
    ck(cu.cuCtxCreate_v2(ctypes.byref(ctx), 0, dev.value), "cuCtxCreate")      # now current
    bufs = []
    def alloc(n):
        p = U64()
        ck(cu.cuMemAlloc_v2(ctypes.byref(p), n), "cuMemAlloc")
        bufs.append(p.value)
        return p.value
    def up(stored):
        a = np.ascontiguousarray(stored.data)
        p = alloc(a.nbytes)
        ck(cu.cuMemcpyHtoD_v2(p, a.ctypes.data, a.nbytes), "cuMemcpyHtoD")
        return p
    f = Params(*(up(getattr(pf, k)) for k in ("x", "dt", "A", "B", "C", "D")))
    r = Params(*(up(getattr(pr, k)) for k in ("x", "dt", "A", "B", "C", "D")))
    y_ws, y_na = alloc(2 * ny), alloc(2 * ny)
    nws = lib.ssd_workspace_bytes(ctypes.byref(sh), chunk)
    ws = alloc(nws)
    ck(cu.cuMemsetD8_v2(ws, 0, nws), "cuMemsetD8")
    if lib.bidir_ssd(ctypes.byref(sh), ctypes.byref(f), ctypes.byref(r), chunk, y_ws, ws, nws, None) != 0:
        raise SystemExit("bidir_ssd: " + lib.ssd_last_error().decode())
    area = VP()
    if lib.bidir_ssd_noalloc(ctypes.byref(sh), ctypes.byref(f), ctypes.byref(r), chunk, y_na, None,
                             ctypes.byref(area)) != 0:
        raise SystemExit("bidir_ssd_noalloc: " + lib.ssd_last_error().decode())
    ck(cu.cuCtxSynchronize(), "cuCtxSynchronize")
    for w in (ws, area.value):
        if lib.ssd_workspace_status(w, 256, None) != 0:
            raise SystemExit("status: " + lib.ssd_last_error().decode())
    out = []
    for y in (y_ws, y_na):
        h = np.empty(ny, np.uint16)
        ck(cu.cuMemcpyDtoH_v2(h.ctypes.data, y, 2 * ny), "cuMemcpyDtoH")
        out.append(si.bf16_bits_to_f32(h).astype(np.float64))
    for p in bufs:
        ck(cu.cuMemFree_v2(p), "cuMemFree")
    ck(cu.cuCtxDestroy_v2(ctx), "cuCtxDestroy")
    return out

rel = lambda a, b: float(np.abs(a - b).max() / np.abs(b).max())
(a_ws, a_na), (b_ws, b_na) = one_context(), one_context()
errs = [rel(a_na, a_ws), rel(b_na, b_ws), rel(b_ws, a_ws)]
print("errs", errs)
assert all(np.isfinite(v).all() for v in (a_ws, a_na, b_ws, b_na))
assert max(errs) <= 1e-2, errs
print("TWO_CONTEXTS_OK")
"""


def test_scratch_address_follows_the_current_context():
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, "-c", _TWO_CONTEXTS, root], capture_output=True, text=True, timeout=600)
    assert r.returncode == 0 and "TWO_CONTEXTS_OK" in r.stdout, r.stdout[-2000:] + r.stderr[-2000:]


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
