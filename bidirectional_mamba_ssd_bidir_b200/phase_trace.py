"""Per-phase timeline of the tensor-core kernel, from its tracing build.

The tracing build (``libbidirssd_trace.so``: the same sources compiled with
``-DSSD_TRACE``) records two things.

* In CTA 0, for its first 8 blocks of 128 tokens, each warp's SM-cycle clock
  at its phase boundaries: points 0..23 per (warp, block).
* For every CTA, its start and end on the global timer (ns) and its SM.

The kernel traced is the shared-score kernel (ssd_tcs.cu), the one that runs
every chain whose decay it can factorise.  This module builds that library on demand and runs one bidirectional call
through it.  The marshalling is the package's own and the call is the same
C ABI entry point, so the output equals the product library's bit for bit.
It returns the stamps; ``summary`` prints when each phase of a block ended,
relative to the issue of that block's score product G = C B^T (MMA stream A).

The product library carries none of this code.  Tracing changes the timing
a little (one store per warp per point).
"""
from __future__ import annotations

import ctypes

import numpy as np
import torch

from . import _check, _params, _shape_of, _stream, _workspace, lib as _lib
from . import build as _build

N_WARPS, N_BLOCKS, N_POINTS = 20, 8, 24
N_CTA_SLOTS = 4096
WARP_MMA_A, WARP_MMA_B = 17, 19
WARP_MMA = WARP_MMA_A

# the points each role records, in program order within a block
COMPUTE_POINTS = [(0, "block start"), (1, "scores G ready"), (2, "masked scores Gc written"),
                  (3, "tables two blocks ahead built"), (4, "state product done"), (5, "state hand-off done"),
                  (7, "Y ready"), (8, "epilogue done"), (6, "next block's cX and Y start written")]
# (warp, point): stream A (warp 17) issues G and the state product, stream B (warp 19) Y_off and Y_diag
MMA_POINTS = [(17, 0, "G issued"), (19, 1, "Y_off issued"), (17, 2, "state product issued"), (19, 3, "Y_diag issued")]
# (warp, point, name) of the load and hand-off warps
LOAD_POINTS = [(16, 0, "x stage free, x loads issued"), (16, 1, "B loads issued (store warp)"),
               (16, 2, "C buffer free, C loads issued"), (16, 3, "decay tables built"),
               (18, 3, "iteration start (ticket next)"), (18, 4, "ticket taken"),
               (18, 0, "y tiles written, store issued"), (18, 2, "y tiles read"),
               (18, 5, "previous store completed"), (18, 1, "first part published")]
# per-block timeline of CTAs 0 and 1, every block (see block_times)
BLOCK_POINTS = ["G issued", "y store issued", "y tiles read", "B load issued"]
N_ALL_BLOCKS = 1024

_trace_lib = None


def library(force_build: bool = False) -> ctypes.CDLL:
    """The tracing build of the library, compiled first if it is missing or older than the sources."""
    global _trace_lib
    if _trace_lib is None or force_build:
        path = _build.build(force=force_build, trace=True)
        t = ctypes.CDLL(path)
        for name in ("bidir_ssd", "ssd_workspace_bytes", "ssd_workspace_status", "ssd_segments_for"):
            getattr(t, name).argtypes = getattr(_lib, name).argtypes
            getattr(t, name).restype = getattr(_lib, name).restype
        t.ssd_debug_trace.argtypes = [ctypes.POINTER(ctypes.c_ulonglong), ctypes.c_int]
        t.ssd_debug_trace.restype = ctypes.c_int
        t.ssd_debug_blocks.argtypes = [ctypes.POINTER(ctypes.c_ulonglong), ctypes.c_int]
        t.ssd_debug_blocks.restype = ctypes.c_int
        t.ssd_debug_cta_times.argtypes = [ctypes.POINTER(ctypes.c_ulonglong), ctypes.c_int]
        t.ssd_debug_cta_times.restype = ctypes.c_int
        _trace_lib = t
    return _trace_lib


def run(fwd: dict, rev: dict, chunk: int = 256):
    """One bidirectional call through the tracing build.

    Returns ``(y, phases, ctas)``.
    * ``phases`` is a float64 array [warp][block][point] of SM cycles, NaN where nothing was recorded.
    * ``ctas`` is an int64 array [cta][start ns, end ns, SM] for the CTAs of the call.
    The shapes must take the tensor-core path (bf16, headdim 64, d_state 128).
    """
    t = library()
    shape = _shape_of(fwd["x"], fwd["B"])
    pf = _params(fwd["x"], fwd["dt"], fwd["A"], fwd["B"], fwd["C"], fwd.get("D"))
    pr = _params(rev["x"], rev["dt"], rev["A"], rev["B"], rev["C"], rev.get("D"))
    y = torch.empty_like(fwd["x"])
    ws, nbytes = _workspace(shape, chunk, fwd["x"].device, None)
    _check(t.bidir_ssd(ctypes.byref(shape), ctypes.byref(pf), ctypes.byref(pr), int(chunk), y.data_ptr(),
                       ws.data_ptr(), nbytes, _stream(fwd["x"].device)))
    torch.cuda.synchronize(fwd["x"].device)
    _check(t.ssd_workspace_status(ws.data_ptr(), nbytes, None))
    n = N_WARPS * N_BLOCKS * N_POINTS
    buf = (ctypes.c_ulonglong * n)()
    if t.ssd_debug_trace(buf, n) != n:
        raise RuntimeError("could not read the phase stamps")
    phases = np.array(buf[:], dtype=np.float64).reshape(N_WARPS, N_BLOCKS, N_POINTS)
    phases[phases == 0] = np.nan
    cbuf = (ctypes.c_ulonglong * (3 * N_CTA_SLOTS))()
    if t.ssd_debug_cta_times(cbuf, 3 * N_CTA_SLOTS) != N_CTA_SLOTS:
        raise RuntimeError("could not read the CTA times")
    nseg = max(1, int(t.ssd_segments_for(ctypes.byref(shape), int(chunk))))
    ncta = min(N_CTA_SLOTS, 2 * shape.batch * (shape.nheads // 2) * nseg)
    ctas = np.array(cbuf[:], dtype=np.int64).reshape(N_CTA_SLOTS, 3)[:ncta]
    return y, phases, ctas


def block_times() -> np.ndarray:
    """Per-block timeline of CTAs 0 and 1 of the last traced call: float64 [cta][block][point]
    of SM cycles (points in ``BLOCK_POINTS``), NaN where nothing was recorded."""
    n = 2 * N_ALL_BLOCKS * len(BLOCK_POINTS)
    buf = (ctypes.c_ulonglong * n)()
    if library().ssd_debug_blocks(buf, n) != n:
        raise RuntimeError("could not read the block timeline")
    out = np.array(buf[:], dtype=np.float64).reshape(2, N_ALL_BLOCKS, len(BLOCK_POINTS))
    out[out == 0] = np.nan
    return out


def summary(phases: np.ndarray, clock_mhz: float = 1965.0, blocks=(3, 4, 5, 6)) -> str:
    """Per block: when each phase ended, in microseconds after the MMA warp issued that block's G."""
    lines = []
    for j in blocks:
        ref = phases[WARP_MMA, j, 0]
        nxt = phases[WARP_MMA, j + 1, 0] if j + 1 < N_BLOCKS else np.nan
        lines.append(f"block {j}: period {(nxt - ref) / clock_mhz:.3f} us")
        for w, k, name in MMA_POINTS:
            lines.append(f"  mma {w:2d}   {name:40s} {(phases[w, j, k] - ref) / clock_mhz:8.3f}")
        for w, k, name in LOAD_POINTS:
            lines.append(f"  warp {w:2d}  {name:40s} {(phases[w, j, k] - ref) / clock_mhz:8.3f}")
        for k, name in COMPUTE_POINTS:
            v = (phases[:16, j, k] - ref) / clock_mhz
            if np.all(np.isnan(v)):
                continue
            lines.append(f"  compute  {name:40s} min {np.nanmin(v):7.3f} median {np.nanmedian(v):7.3f} "
                         f"max {np.nanmax(v):7.3f}")
    return "\n".join(lines)


__all__ = ["library", "run", "summary", "block_times", "COMPUTE_POINTS", "MMA_POINTS", "LOAD_POINTS",
           "BLOCK_POINTS"]
