"""Float64 CPU oracle for the bidirectional SSD scan.

TEST INFRASTRUCTURE ONLY.  The tests, the smoke check and the bench's CPU
baseline may import this package; the library (``bidirectional_mamba_ssd_bidir_b200``)
never does, and this package never imports the library.  The two share no
code: the only thing both sides see is the seeded input generator
(``ssd_inputs``), which holds none of the scan's arithmetic.

Contents
--------
``ssd_scan_f64``   the plain sequential recurrence (C, ``ssd_oracle.c``), one
                   direction.  Pinned by the tests against the brute-force
                   semiseparable matrix form, closed forms and invariants.
``bidir_f64``      DiffuMamba mixer: two independent layers, forward and
                   reverse, combined by summation ("DiffuMamba", technical
                   summary section 2: a forward and a reverse Mamba layer,
                   independent of each other, give a symmetric context).
``r2l_block_f64``  R2LM sidecar: reverse scan (flip, scan, flip back), scaled
                   by the scalar gate s and added to the residual
                   ("Bifocal Diffusion Language Models", section 2,
                   mechanism and integration).  s = 0 returns the residual
                   itself, so the model is unchanged at initialisation.
``ssd_scan_bwd_f64`` the gradients of the scan (reverse-mode, position by
                   position), for training the layers that run it.
``ssd_scan_state_f64`` the recurrence with the state carried across the call
                   (state in, state out), for block-wise decoding.
``ssd_chunked_f64`` the chunked (state-passing) form of the same scan, the
                   decomposition the GPU kernels use; pinned against the
                   recurrence for several chunk sizes.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ssd_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libssd_oracle.so")
_lib = None
_lock = threading.Lock()


def build(force: bool = False) -> str:
    """Compile the C oracle (gcc, IEEE float64, no fast-math)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-pthread",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def load_library(path: str | None = None):
    """Load the oracle library; ``path`` overrides it (the mutation tests load planted-bug builds)."""
    global _lib
    if path is not None:
        lib = ctypes.CDLL(path)
    else:
        with _lock:
            if _lib is None:
                _lib = ctypes.CDLL(build())
            lib = _lib
    f = lib.ssd_oracle_scan
    dp = ctypes.POINTER(ctypes.c_double)
    f.argtypes = [ctypes.c_int] * 6 + [dp] * 6 + [ctypes.c_int, dp, ctypes.c_int]
    f.restype = ctypes.c_int
    if hasattr(lib, "ssd_oracle_scan_bwd"):
        k = lib.ssd_oracle_scan_bwd
        k.argtypes = [ctypes.c_int] * 6 + [dp] * 6 + [ctypes.c_int, dp] + [dp] * 6 + [ctypes.c_int]
        k.restype = ctypes.c_int
    if hasattr(lib, "ssd_oracle_scan_state"):
        g = lib.ssd_oracle_scan_state
        g.argtypes = [ctypes.c_int] * 6 + [dp] * 6 + [ctypes.c_int, dp, dp, dp, ctypes.c_int]
        g.restype = ctypes.c_int
    return lib


def _ptr(a):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double)) if a is not None else None


def default_threads() -> int:
    return len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else (os.cpu_count() or 1)


def ssd_scan_f64(x, dt, A, B, C, D=None, direction=1, nthreads=None, lib=None):
    """Plain recurrence, float64.  x [b,L,H,P], dt [b,L,H], A [H], B/C [b,L,G,N], D [H] or None."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    dt = np.ascontiguousarray(dt, dtype=np.float64)
    A = np.ascontiguousarray(A, dtype=np.float64)
    B = np.ascontiguousarray(B, dtype=np.float64)
    C = np.ascontiguousarray(C, dtype=np.float64)
    D = None if D is None else np.ascontiguousarray(D, dtype=np.float64)
    b, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    assert dt.shape == (b, L, H) and A.shape == (H,) and B.shape == (b, L, G, N) and C.shape == B.shape
    y = np.zeros_like(x)
    lib = lib or load_library()
    rc = lib.ssd_oracle_scan(b, L, H, P, N, G, _ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C),
                             _ptr(D), int(direction), _ptr(y), int(nthreads or default_threads()))
    if rc != 0:
        raise RuntimeError(f"ssd_oracle_scan failed with {rc}")
    return y


def ssd_scan_state_f64(x, dt, A, B, C, D=None, direction=1, init_state=None, nthreads=None, lib=None):
    """The recurrence with the state carried across the call: returns (y, final_state).

    ``init_state`` [b, H, P, N] (None = zero) is the state before the first token in scan order;
    ``final_state`` is the state after the last one.  Block-wise decoding with cache reuse
    ("DiffuMamba", technical summary, sections 2 and 4) carries this state from one block
    to the next."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    dt = np.ascontiguousarray(dt, dtype=np.float64)
    A = np.ascontiguousarray(A, dtype=np.float64)
    B = np.ascontiguousarray(B, dtype=np.float64)
    C = np.ascontiguousarray(C, dtype=np.float64)
    D = None if D is None else np.ascontiguousarray(D, dtype=np.float64)
    b, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    assert dt.shape == (b, L, H) and A.shape == (H,) and B.shape == (b, L, G, N) and C.shape == B.shape
    s_in = None if init_state is None else np.ascontiguousarray(init_state, dtype=np.float64)
    if s_in is not None:
        assert s_in.shape == (b, H, P, N)
    y = np.zeros_like(x)
    s_out = np.zeros((b, H, P, N))
    lib = lib or load_library()
    rc = lib.ssd_oracle_scan_state(b, L, H, P, N, G, _ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C), _ptr(D),
                                   int(direction), _ptr(s_in), _ptr(y), _ptr(s_out),
                                   int(nthreads or default_threads()))
    if rc != 0:
        raise RuntimeError(f"ssd_oracle_scan_state failed with {rc}")
    return y, s_out


def ssd_scan_bwd_f64(x, dt, A, B, C, D, direction, gy, nthreads=None, lib=None):
    """Gradients of L = sum(gy * y) for the scan from a zero state: dict with x, dt, A, B, C, D.

    The reverse-mode derivative of the recurrence, taken position by position
    (oracle header); D's entry is None when D is None."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    dt = np.ascontiguousarray(dt, dtype=np.float64)
    A = np.ascontiguousarray(A, dtype=np.float64)
    B = np.ascontiguousarray(B, dtype=np.float64)
    C = np.ascontiguousarray(C, dtype=np.float64)
    D = None if D is None else np.ascontiguousarray(D, dtype=np.float64)
    gy = np.ascontiguousarray(gy, dtype=np.float64)
    b, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    assert gy.shape == x.shape
    g = {"x": np.zeros_like(x), "dt": np.zeros_like(dt), "A": np.zeros(H), "B": np.zeros_like(B),
         "C": np.zeros_like(C), "D": None if D is None else np.zeros(H)}
    lib = lib or load_library()
    rc = lib.ssd_oracle_scan_bwd(b, L, H, P, N, G, _ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C), _ptr(D),
                                 int(direction), _ptr(gy), _ptr(g["x"]), _ptr(g["dt"]), _ptr(g["A"]),
                                 _ptr(g["B"]), _ptr(g["C"]), _ptr(g["D"]), int(nthreads or default_threads()))
    if rc != 0:
        raise RuntimeError(f"ssd_oracle_scan_bwd failed with {rc}")
    return g


def bidir_f64(pf: dict, pr: dict, nthreads=None, lib=None):
    """y = y_fwd(pf) + y_rev(pr); each dict holds float64 x, dt, A, B, C and D (or None)."""
    yf = ssd_scan_f64(pf["x"], pf["dt"], pf["A"], pf["B"], pf["C"], pf.get("D"), 1, nthreads, lib)
    yr = ssd_scan_f64(pr["x"], pr["dt"], pr["A"], pr["B"], pr["C"], pr.get("D"), -1, nthreads, lib)
    return yf + yr


def r2l_block_f64(p: dict, s: float, residual, nthreads=None, lib=None):
    """out = residual + s * y_rev, residual laid out [b, L, H*P]; s == 0 returns residual exactly."""
    residual = np.asarray(residual, dtype=np.float64)
    if s == 0.0:
        return residual.copy()
    yr = ssd_scan_f64(p["x"], p["dt"], p["A"], p["B"], p["C"], p.get("D"), -1, nthreads, lib)
    return residual + float(s) * yr.reshape(residual.shape)


def ssd_chunked_f64(x, dt, A, B, C, D=None, direction=1, chunk=16):
    """Chunked (state-passing) form of the scan, float64, one direction.

    The sequence is cut into chunks of ``chunk`` tokens.  Inside chunk c, with
    cs_t = A * (sum of dt over the chunk's tokens up to and including t):
      intra-chunk: Y_diag[t] = sum_{s<=t} (C_t . B_s) exp(cs_t - cs_s) dt_s x_s
      chunk state: S_c      = sum_s exp(cs_last - cs_s) dt_s x_s (outer) B_s
      passing:     Sin_0 = 0,  Sin_{c+1} = exp(cs_last) Sin_c + S_c
      from state:  Y_off[t] = exp(cs_t) * (C_t applied to Sin_c)
      output:      y = Y_diag + Y_off + D x
    The reverse direction is flip, forward, flip.  Exact arithmetic gives the
    recurrence's result for every chunk size.
    """
    x = np.asarray(x, np.float64); dt = np.asarray(dt, np.float64)
    A = np.asarray(A, np.float64); B = np.asarray(B, np.float64); C = np.asarray(C, np.float64)
    if direction < 0:
        y = ssd_chunked_f64(x[:, ::-1], dt[:, ::-1], A, B[:, ::-1], C[:, ::-1], D, 1, chunk)
        return np.ascontiguousarray(y[:, ::-1])
    b, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    assert L % chunk == 0
    nc = L // chunk
    hg = np.arange(H) // (H // G)
    Bh = B[:, :, hg, :]                      # [b, L, H, N]
    Ch = C[:, :, hg, :]
    xc = x.reshape(b, nc, chunk, H, P)
    dtc = dt.reshape(b, nc, chunk, H)
    Bc = Bh.reshape(b, nc, chunk, H, N)
    Cc = Ch.reshape(b, nc, chunk, H, N)
    cs = np.cumsum(dtc, axis=2) * A          # [b, nc, Q, H]
    seg = cs[:, :, :, None, :] - cs[:, :, None, :, :]          # [b,nc,t,s,H]
    causal = np.tril(np.ones((chunk, chunk), dtype=bool))[None, None, :, :, None]
    decay = np.where(causal, np.exp(np.where(causal, seg, 0.0)), 0.0)
    CB = np.einsum("bctHn,bcsHn->bctsH", Cc, Bc)
    Mmat = CB * decay * dtc[:, :, None, :, :]
    y_diag = np.einsum("bctsH,bcsHp->bctHp", Mmat, xc)
    w = np.exp(cs[:, :, -1:, :] - cs) * dtc                   # [b,nc,Q,H]
    S = np.einsum("bcsH,bcsHp,bcsHn->bcHpn", w, xc, Bc)
    a = np.exp(cs[:, :, -1, :])                                # [b,nc,H]
    Sin = np.zeros((b, nc, H, P, N))
    run = np.zeros((b, H, P, N))
    for c in range(nc):
        Sin[:, c] = run
        run = a[:, c, :, None, None] * run + S[:, c]
    y_off = np.einsum("bctHn,bcHpn->bctHp", Cc, Sin) * np.exp(cs)[..., None]
    y = (y_diag + y_off).reshape(b, L, H, P)
    if D is not None:
        y = y + np.asarray(D, np.float64)[None, None, :, None] * x
    return y


def rel_err(y, y_ref) -> float:
    """max|y - y_ref| / max|y_ref| over the whole tensor, in float64."""
    y = np.asarray(y, np.float64); y_ref = np.asarray(y_ref, np.float64)
    den = np.max(np.abs(y_ref)) if y_ref.size else 0.0
    num = np.max(np.abs(y - y_ref)) if y_ref.size else 0.0
    return float(num / den) if den > 0 else float(num)


def params_f64(p) -> dict:
    """float64 view of a generated parameter set (``ssd_inputs.Params``): the exact stored values."""
    return {"x": p.x.f64(), "dt": p.dt.f64(), "A": p.A.f64(), "B": p.B.f64(), "C": p.C.f64(),
            "D": p.D.f64() if p.extra.get("with_D", True) else None}
