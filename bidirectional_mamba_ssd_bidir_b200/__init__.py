"""Bidirectional Mamba-2 SSD scan for NVIDIA B200 (sm_100a).

Thin Python binding over the C ABI of ``libbidirssd.so`` (declared in
``include/bidir_ssd.h``).  This module only marshals arguments: it checks
dtypes, shapes and devices, takes device memory for the output and the
workspace from PyTorch, and passes raw pointers and the current CUDA stream
to the library.  Every step of the scan runs in the library's CUDA kernels;
there is no CPU or PyTorch fallback, and importing this package fails if the
library has not been built.

Entry points (same names as the C ABI):
  ssd_scan(x, dt, A, B, C, D=None, direction=1, chunk=256)   one direction
  ssd_scan_state(..., state_in=None)                          one direction, state in and out
  ssd_scan_bwd(x, dt, A, B, C, D, gy, direction, chunk)       gradients of one direction
  bidir_ssd(fwd, rev, chunk=256)                              y_fwd + flip(scan(flip(.)))
  r2l_block_scan(p, s, residual, chunk=32)                    residual + s * y_rev
  bidir_ssd_noalloc(fwd, rev, out, chunk=256)                 bidir_ssd into a caller-owned `out`,
                                                              scratch inside the library
"""
from __future__ import annotations

import ctypes
import os

import torch

__all__ = ["ssd_scan", "ssd_scan_state", "ssd_scan_bwd", "bidir_ssd", "r2l_block_scan", "bidir_ssd_noalloc", "noalloc_status", "NoallocArea", "workspace_bytes", "path_for",
           "segments_for", "kernel_launches", "mixer_bidir", "mixer_workspace_bytes", "gemm_bf16", "attention",
           "attention_block", "attention_block_workspace_bytes", "workspace_status", "SSDError", "library_path", "lib"]

_HERE = os.path.dirname(os.path.abspath(__file__))
library_path = os.path.join(_HERE, "libbidirssd.so")

if not os.path.exists(library_path):
    raise ImportError(
        f"{library_path} is missing: build the CUDA library first "
        "(python -c 'import __graft_entry__ as g; g.build()' from the repository root)")

lib = ctypes.CDLL(library_path)

SSD_BF16, SSD_F32 = 0, 1
_STATUS = {0: "ok", 1: "invalid argument", 2: "unsupported shape", 3: "CUDA error", 4: "device wait timed out"}


class _Shape(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int), ("seqlen", ctypes.c_int), ("nheads", ctypes.c_int),
                ("headdim", ctypes.c_int), ("dstate", ctypes.c_int), ("ngroups", ctypes.c_int),
                ("io", ctypes.c_int)]


class _Params(ctypes.Structure):
    _fields_ = [("x", ctypes.c_void_p), ("dt", ctypes.c_void_p), ("A", ctypes.c_void_p),
                ("B", ctypes.c_void_p), ("C", ctypes.c_void_p), ("D", ctypes.c_void_p)]


class _MixerShape(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in ("batch", "seqlen", "d_model", "nheads", "headdim", "dstate", "ngroups",
                                            "d_conv")]


class _MixerLayer(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("W_in", "conv_w", "conv_b", "dt_bias", "A", "D", "norm_w", "W_out")]


class _AttnShape(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in ("batch", "seqlen", "nheads", "headdim")]


_SP, _PP, _VP, _SZ = ctypes.POINTER(_Shape), ctypes.POINTER(_Params), ctypes.c_void_p, ctypes.c_size_t
_ASP, _LL = ctypes.POINTER(_AttnShape), ctypes.c_longlong
lib.ssd_attention.argtypes = [_ASP, _VP, _LL, _VP, _LL, _VP, _LL, _VP, _LL, ctypes.c_float, _VP, _SZ, _VP]
lib.ssd_attention.restype = ctypes.c_int
lib.ssd_attention_block_workspace_bytes.argtypes = [_ASP]
lib.ssd_attention_block_workspace_bytes.restype = _SZ
lib.attention_block.argtypes = [_ASP, ctypes.c_int, _VP, _VP, _VP, _VP, _VP, _SZ, _VP]
lib.attention_block.restype = ctypes.c_int
_MSP, _MLP = ctypes.POINTER(_MixerShape), ctypes.POINTER(_MixerLayer)
lib.ssd_mixer_workspace_bytes.argtypes = [_MSP]
lib.ssd_mixer_workspace_bytes.restype = _SZ
lib.mamba2_mixer_bidir.argtypes = [_MSP, _VP, _MLP, _MLP, _VP, _VP, _SZ, _VP]
lib.mamba2_mixer_bidir.restype = ctypes.c_int
lib.ssd_gemm_bf16.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, _VP, _VP, _VP, _VP, _SZ, _VP]
lib.ssd_gemm_bf16.restype = ctypes.c_int
lib.ssd_workspace_bytes.argtypes = [_SP, ctypes.c_int]
lib.ssd_workspace_bytes.restype = _SZ
lib.ssd_path_for.argtypes = [_SP, ctypes.c_int]
lib.ssd_path_for.restype = ctypes.c_int
lib.ssd_kernel_launches.argtypes = [_SP, ctypes.c_int, ctypes.c_int]
lib.ssd_kernel_launches.restype = ctypes.c_int
lib.ssd_segments_for.argtypes = [_SP, ctypes.c_int]
lib.ssd_segments_for.restype = ctypes.c_int
lib.ssd_scan.argtypes = [_SP, _PP, ctypes.c_int, ctypes.c_int, _VP, _VP, _SZ, _VP]
lib.ssd_scan.restype = ctypes.c_int
lib.bidir_ssd.argtypes = [_SP, _PP, _PP, ctypes.c_int, _VP, _VP, _SZ, _VP]
lib.ssd_scan_state.argtypes = [_SP, _PP, ctypes.c_int, ctypes.c_int, _VP, _VP, _VP, _VP, _SZ, _VP]
lib.ssd_scan_state.restype = ctypes.c_int
lib.ssd_bwd_workspace_bytes.argtypes = [_SP, ctypes.c_int]
lib.ssd_bwd_workspace_bytes.restype = _SZ
lib.ssd_scan_bwd.argtypes = [_SP, _PP, ctypes.c_int, ctypes.c_int, _VP] + [_VP] * 6 + [_VP, _SZ, _VP]
lib.ssd_scan_bwd.restype = ctypes.c_int
lib.bidir_ssd.restype = ctypes.c_int
lib.r2l_block_scan.argtypes = [_SP, _PP, ctypes.c_float, _VP, ctypes.c_int, _VP, _VP, _SZ, _VP]
lib.r2l_block_scan.restype = ctypes.c_int
lib.ssd_workspace_status.argtypes = [_VP, _SZ, _VP]
lib.bidir_ssd_noalloc.argtypes = [_SP, _PP, _PP, ctypes.c_int, _VP, _VP, ctypes.POINTER(ctypes.c_void_p)]
lib.bidir_ssd_noalloc.restype = ctypes.c_int
lib.ssd_workspace_status.restype = ctypes.c_int
lib.ssd_status_string.argtypes = [ctypes.c_int]
lib.ssd_status_string.restype = ctypes.c_char_p
lib.ssd_debug_fault.argtypes = [ctypes.c_int, ctypes.c_double]
lib.ssd_debug_fault.restype = ctypes.c_int
lib.ssd_last_error.argtypes = []
lib.ssd_last_error.restype = ctypes.c_char_p


class SSDError(RuntimeError):
    def __init__(self, status: int):
        self.status = status
        msg = lib.ssd_last_error().decode() or ""
        super().__init__(f"{_STATUS.get(status, status)}: {msg}")


def _check(status: int):
    if status != 0:
        raise SSDError(status)


def _io(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return SSD_BF16
    if t.dtype == torch.float32:
        return SSD_F32
    raise TypeError(f"unsupported io dtype {t.dtype} (bfloat16 or float32)")


def _shape_of(x, B) -> _Shape:
    if x.dim() != 4 or B.dim() != 4:
        raise ValueError("x must be [batch, seqlen, nheads, headdim] and B/C [batch, seqlen, ngroups, dstate]")
    b, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    return _Shape(b, L, H, P, N, G, _io(x))


def _params(x, dt, A, B, C, D) -> _Params:
    """The six parameter pointers, after checking shapes, dtypes, device and layout.

    The common case is checked with few tensor calls (a per-call cost of decode-sized
    launches); if anything is off, the checks run one by one for the error message."""
    b, L, H, P = x.shape
    io, dev = x.dtype, x.get_device()
    if (dev >= 0 and dt.shape == (b, L, H) and B.dim() == 4 and C.shape == B.shape and B.shape[:2] == (b, L)
            and dt.dtype is io and B.dtype is io and C.dtype is io
            and A.dtype is torch.float32 and A.shape == (H,)
            and (D is None or (D.dtype is torch.float32 and D.shape == (H,)))
            and dt.get_device() == dev and A.get_device() == dev and B.get_device() == dev
            and C.get_device() == dev and (D is None or D.get_device() == dev)
            and x.is_contiguous() and dt.is_contiguous() and A.is_contiguous() and B.is_contiguous()
            and C.is_contiguous() and (D is None or D.is_contiguous())):
        return _Params(x.data_ptr(), dt.data_ptr(), A.data_ptr(), B.data_ptr(), C.data_ptr(),
                       D.data_ptr() if D is not None else None)
    return _params_checked(x, dt, A, B, C, D)


def _params_checked(x, dt, A, B, C, D) -> _Params:
    b, L, H, P = x.shape
    io = x.dtype
    for name, t, shp in (("dt", dt, (b, L, H)), ("B", B, None), ("C", C, tuple(B.shape))):
        if shp is not None and tuple(t.shape) != shp:
            raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {shp}")
    if B.shape[:2] != x.shape[:2]:
        raise ValueError("B must be [batch, seqlen, ngroups, dstate]")
    for name, t in (("x", x), ("dt", dt), ("B", B), ("C", C)):
        if t.dtype != io:
            raise TypeError(f"{name} is {t.dtype}; x, dt, B, C must share one dtype")
    for name, t in (("A", A), ("D", D)):
        if t is not None and (t.dtype != torch.float32 or tuple(t.shape) != (H,)):
            raise TypeError(f"{name} must be float32 of shape ({H},)")
    dev = x.device
    for name, t in (("x", x), ("dt", dt), ("A", A), ("B", B), ("C", C), ("D", D)):
        if t is None:
            continue
        if t.device != dev or dev.type != "cuda":
            raise ValueError(f"{name} must be a CUDA tensor on {dev}")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    return _Params(x.data_ptr(), dt.data_ptr(), A.data_ptr(), B.data_ptr(), C.data_ptr(),
                   D.data_ptr() if D is not None else None)


# the current stream's handle without building a torch Stream object (about 2 us a call less)
_raw_stream = getattr(torch._C, "_cuda_getCurrentRawStream", None)


def _stream(dev) -> int:
    if _raw_stream is not None:
        return int(_raw_stream(dev.index if dev.index is not None else torch.cuda.current_device()))
    return torch.cuda.current_stream(dev).cuda_stream


def workspace_bytes(shape: tuple, io: torch.dtype, chunk: int) -> int:
    """Workspace size for (batch, seqlen, nheads, headdim, dstate, ngroups) at this chunk."""
    s = _Shape(*shape, SSD_BF16 if io == torch.bfloat16 else SSD_F32)
    return int(lib.ssd_workspace_bytes(ctypes.byref(s), int(chunk)))


def path_for(shape: tuple, io: torch.dtype, chunk: int) -> int:
    """1 = tensor-core path, 0 = SIMT path, -1 = refused."""
    s = _Shape(*shape, SSD_BF16 if io == torch.bfloat16 else SSD_F32)
    return int(lib.ssd_path_for(ctypes.byref(s), int(chunk)))


def segments_for(shape: tuple, io: torch.dtype, chunk: int) -> int:
    """Segments per sequence on the tensor-core path (1 = none), 0 on the SIMT path, -1 = refused."""
    s = _Shape(*shape, SSD_BF16 if io == torch.bfloat16 else SSD_F32)
    return int(lib.ssd_segments_for(ctypes.byref(s), int(chunk)))


def kernel_launches(shape: tuple, io: torch.dtype, chunk: int, op: str) -> int:
    """Kernels one call launches: op in {"scan", "bidir", "r2l"}."""
    s = _Shape(*shape, SSD_BF16 if io == torch.bfloat16 else SSD_F32)
    return int(lib.ssd_kernel_launches(ctypes.byref(s), int(chunk), {"scan": 0, "bidir": 1, "r2l": 2}[op]))


def _workspace(shape: _Shape, chunk: int, dev, workspace):
    need = int(lib.ssd_workspace_bytes(ctypes.byref(shape), int(chunk)))
    if workspace is None:
        # only the status word (the first 256 bytes) must start at zero
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
        workspace[:256].zero_()
    return workspace, workspace.numel() * workspace.element_size()


def ssd_scan(x, dt, A, B, C, D=None, direction: int = 1, chunk: int = 256, out=None, workspace=None):
    """One direction of the scan; returns y shaped like x."""
    shape = _shape_of(x, B)
    prm = _params(x, dt, A, B, C, D)
    y = torch.empty_like(x) if out is None else out
    ws, nbytes = _workspace(shape, chunk, x.device, workspace)
    _check(lib.ssd_scan(ctypes.byref(shape), ctypes.byref(prm), int(direction), int(chunk),
                        y.data_ptr(), ws.data_ptr(), nbytes, _stream(x.device)))
    return y


def ssd_scan_state(x, dt, A, B, C, D=None, direction: int = 1, chunk: int = 256, state_in=None,
                   out=None, state_out=None, workspace=None):
    """One direction with the state carried across the call: returns (y, state_out).

    ``state_in`` (float32 [batch, nheads, headdim, dstate], or None = zero) is the state before
    the first token in scan order; the returned state is the one after the last token."""
    shape = _shape_of(x, B)
    prm = _params(x, dt, A, B, C, D)
    b, L, H, P = x.shape
    N = B.shape[3]
    for name, t in (("state_in", state_in), ("state_out", state_out)):
        if t is not None and (t.dtype != torch.float32 or tuple(t.shape) != (b, H, P, N) or
                              t.device != x.device or not t.is_contiguous()):
            raise ValueError(f"{name} must be contiguous float32 of shape {(b, H, P, N)} on {x.device}")
    y = torch.empty_like(x) if out is None else out
    so = torch.empty((b, H, P, N), dtype=torch.float32, device=x.device) if state_out is None else state_out
    ws, nbytes = _workspace(shape, chunk, x.device, workspace)
    _check(lib.ssd_scan_state(ctypes.byref(shape), ctypes.byref(prm), int(direction), int(chunk),
                              state_in.data_ptr() if state_in is not None else None, so.data_ptr(),
                              y.data_ptr(), ws.data_ptr(), nbytes, _stream(x.device)))
    return y, so


def ssd_scan_bwd(x, dt, A, B, C, D, gy, direction: int = 1, chunk: int = 256, workspace=None) -> dict:
    """Gradients of ssd_scan for dL/dy = gy: dict with float32 x, dt, A, B, C and D (None if D is None)."""
    shape = _shape_of(x, B)
    prm = _params(x, dt, A, B, C, D)
    if gy.shape != x.shape or gy.dtype != x.dtype or gy.device != x.device or not gy.is_contiguous():
        raise ValueError(f"gy must be a contiguous {x.dtype} tensor of shape {tuple(x.shape)} on {x.device}")
    dev = x.device
    f32 = dict(dtype=torch.float32, device=dev)
    g = {"x": torch.empty(x.shape, **f32), "dt": torch.empty(dt.shape, **f32), "A": torch.empty(A.shape, **f32),
         "B": torch.empty(B.shape, **f32), "C": torch.empty(C.shape, **f32),
         "D": torch.empty(A.shape, **f32) if D is not None else None}
    need = int(lib.ssd_bwd_workspace_bytes(ctypes.byref(shape), int(chunk)))
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
        workspace[:256].zero_()
    ptr = lambda t: t.data_ptr() if t is not None else None
    _check(lib.ssd_scan_bwd(ctypes.byref(shape), ctypes.byref(prm), int(direction), int(chunk), gy.data_ptr(),
                            ptr(g["x"]), ptr(g["dt"]), ptr(g["A"]), ptr(g["B"]), ptr(g["C"]), ptr(g["D"]),
                            workspace.data_ptr(), workspace.numel(), _stream(dev)))
    return g


def bidir_ssd(fwd: dict, rev: dict, chunk: int = 256, out=None, workspace=None):
    """DiffuMamba mixer: y = scan(fwd, +1) + scan(rev, -1).  Each dict holds x, dt, A, B, C and D (or None)."""
    shape = _shape_of(fwd["x"], fwd["B"])
    if tuple(rev["x"].shape) != tuple(fwd["x"].shape) or tuple(rev["B"].shape) != tuple(fwd["B"].shape):
        raise ValueError("forward and reverse parameters must have the same shapes")
    pf = _params(fwd["x"], fwd["dt"], fwd["A"], fwd["B"], fwd["C"], fwd.get("D"))
    pr = _params(rev["x"], rev["dt"], rev["A"], rev["B"], rev["C"], rev.get("D"))
    y = torch.empty_like(fwd["x"]) if out is None else out
    ws, nbytes = _workspace(shape, chunk, fwd["x"].device, workspace)
    _check(lib.bidir_ssd(ctypes.byref(shape), ctypes.byref(pf), ctypes.byref(pr), int(chunk),
                         y.data_ptr(), ws.data_ptr(), nbytes, _stream(fwd["x"].device)))
    return y


def r2l_block_scan(p: dict, s: float, residual, chunk: int = 32, out=None, workspace=None):
    """R2LM sidecar block: out = residual + s * scan(p, -1); s == 0 returns the residual bit for bit."""
    shape = _shape_of(p["x"], p["B"])
    prm = _params(p["x"], p["dt"], p["A"], p["B"], p["C"], p.get("D"))
    b, L, H, P = p["x"].shape
    if tuple(residual.shape) != (b, L, H * P) or residual.dtype != p["x"].dtype or not residual.is_contiguous():
        raise ValueError(f"residual must be contiguous {p['x'].dtype} of shape {(b, L, H * P)}")
    o = torch.empty_like(residual) if out is None else out
    ws, nbytes = _workspace(shape, chunk, p["x"].device, workspace)
    _check(lib.r2l_block_scan(ctypes.byref(shape), ctypes.byref(prm), ctypes.c_float(s), residual.data_ptr(),
                              int(chunk), o.data_ptr(), ws.data_ptr(), nbytes, _stream(p["x"].device)))
    return o


_MIXER_KEYS = ("W_in", "conv_w", "conv_b", "dt_bias", "A", "D", "norm_w", "W_out")


def _mixer_layer(layer: dict) -> _MixerLayer:
    for k in ("W_in", "W_out"):
        if layer[k].dtype != torch.bfloat16 or not layer[k].is_contiguous():
            raise ValueError(f"{k} must be contiguous bf16")
    for k in ("conv_w", "conv_b", "dt_bias", "A", "D", "norm_w"):
        if layer[k].dtype != torch.float32 or not layer[k].is_contiguous():
            raise ValueError(f"{k} must be contiguous float32")
    return _MixerLayer(*(layer[k].data_ptr() for k in _MIXER_KEYS))


def mixer_workspace_bytes(batch: int, seqlen: int, d_model: int, nheads: int, headdim: int = 64,
                          dstate: int = 128, ngroups: int = 1, d_conv: int = 4) -> int:
    s = _MixerShape(batch, seqlen, d_model, nheads, headdim, dstate, ngroups, d_conv)
    return int(lib.ssd_mixer_workspace_bytes(ctypes.byref(s)))


def mixer_bidir(u, fwd: dict, rev: dict, nheads: int, headdim: int = 64, dstate: int = 128, d_conv: int = 4,
                out=None, workspace=None):
    """The DiffuMamba mixer: two independent Mamba-2 layers (forward, and on the reversed sequence), summed.

    u [batch, seqlen, d_model] bf16; each layer a dict of W_in, conv_w, conv_b, dt_bias, A, D, norm_w, W_out."""
    if u.dtype != torch.bfloat16 or u.dim() != 3 or not u.is_contiguous():
        raise ValueError("u must be contiguous bf16 [batch, seqlen, d_model]")
    b, L, dm = u.shape
    s = _MixerShape(b, L, dm, nheads, headdim, dstate, 1, d_conv)
    need = int(lib.ssd_mixer_workspace_bytes(ctypes.byref(s)))
    if need == 0:
        raise SSDError(2)
    o = torch.empty_like(u) if out is None else out
    if workspace is None:
        workspace = torch.zeros(need, dtype=torch.uint8, device=u.device)
    f, r = _mixer_layer(fwd), _mixer_layer(rev)
    _check(lib.mamba2_mixer_bidir(ctypes.byref(s), u.data_ptr(), ctypes.byref(f), ctypes.byref(r), o.data_ptr(),
                                  workspace.data_ptr(), workspace.numel(), _stream(u.device)))
    return o


def gemm_bf16(A, W, out=None):
    """A [M, K] @ W[N, K]^T on the tensor core (bf16 in and out, float32 accumulation)."""
    if A.dtype != torch.bfloat16 or W.dtype != torch.bfloat16 or not A.is_contiguous() or not W.is_contiguous():
        raise ValueError("A and W must be contiguous bf16")
    M, K = A.shape
    N = W.shape[0]
    o = torch.empty(M, N, dtype=torch.bfloat16, device=A.device) if out is None else out
    ws = torch.zeros(256, dtype=torch.uint8, device=A.device)
    _check(lib.ssd_gemm_bf16(M, N, K, A.data_ptr(), W.data_ptr(), o.data_ptr(), ws.data_ptr(), 256, _stream(A.device)))
    return o


def attention(q, k, v, out=None, scale: float = 0.0, workspace=None):
    """Unmasked multi-head softmax attention on the tensor core: q, k, v [batch, seqlen, nheads,
    headdim] bf16 (headdim 64 or 128; the last two dimensions contiguous, tokens any multiple of 8
    elements apart, so q, k, v may be views of one packed projection).  scale 0: 1/sqrt(headdim)."""
    for t in (q, k, v):
        if t.dtype != torch.bfloat16 or t.dim() != 4 or t.stride(3) != 1 or t.stride(2) != t.shape[3]:
            raise ValueError("q, k, v must be bf16 [batch, seqlen, nheads, headdim] with contiguous heads")
        if t.shape != q.shape or (t.shape[0] > 1 and t.stride(0) != t.shape[1] * t.stride(1)):
            raise ValueError("q, k, v must have one shape and sequences one after another")
    b, L, H, D = q.shape
    o = torch.empty(b, L, H, D, dtype=torch.bfloat16, device=q.device) if out is None else out
    if workspace is None:
        workspace = torch.zeros(256, dtype=torch.uint8, device=q.device)
    s = _AttnShape(b, L, H, D)
    _check(lib.ssd_attention(ctypes.byref(s), q.data_ptr(), q.stride(1), k.data_ptr(), k.stride(1), v.data_ptr(),
                             v.stride(1), o.data_ptr(), o.stride(1), float(scale), workspace.data_ptr(),
                             workspace.numel(), _stream(q.device)))
    return o


def attention_block_workspace_bytes(batch: int, seqlen: int, nheads: int, headdim: int) -> int:
    s = _AttnShape(batch, seqlen, nheads, headdim)
    return int(lib.ssd_attention_block_workspace_bytes(ctypes.byref(s)))


def attention_block(u, W_qkv, W_o, nheads: int, headdim: int = 128, out=None, workspace=None):
    """The DiffuMamba-H attention block: out = attention(split(u W_qkv^T)) W_o^T; u [batch, seqlen,
    d_model] bf16, W_qkv [3 nheads headdim, d_model], W_o [d_model, nheads headdim]."""
    if u.dtype != torch.bfloat16 or u.dim() != 3 or not u.is_contiguous():
        raise ValueError("u must be contiguous bf16 [batch, seqlen, d_model]")
    b, L, dm = u.shape
    s = _AttnShape(b, L, nheads, headdim)
    need = int(lib.ssd_attention_block_workspace_bytes(ctypes.byref(s)))
    if need == 0:
        raise SSDError(2)
    o = torch.empty_like(u) if out is None else out
    if workspace is None:
        workspace = torch.zeros(need, dtype=torch.uint8, device=u.device)
    _check(lib.attention_block(ctypes.byref(s), dm, u.data_ptr(), W_qkv.data_ptr(), W_o.data_ptr(), o.data_ptr(),
                               workspace.data_ptr(), workspace.numel(), _stream(u.device)))
    return o


def workspace_status(workspace) -> None:
    """Raise SSDError if a bounded device-side wait gave up in a call that used ``workspace``."""
    dev = workspace.device
    _check(lib.ssd_workspace_status(workspace.data_ptr(), workspace.numel(), _stream(dev)))


class NoallocArea(int):
    """Device address of the no-allocation scratch's status area, with the device the call ran on."""

    def __new__(cls, address: int, device: int):
        obj = super().__new__(cls, address)
        obj.device = device
        return obj


def bidir_ssd_noalloc(fwd: dict, rev: dict, out, chunk: int = 256) -> NoallocArea:
    """``bidir_ssd`` for callers that cannot allocate device memory at the call.

    Writes y into ``out`` (preallocated, contiguous, shaped like ``fwd["x"]``).
    The scratch the kernels need is a fixed array inside the library, so
    neither this function nor the library allocates anything; shapes whose
    scratch exceeds that array raise SSDError (unsupported shape).  Calls
    that overlap on the GPU share the array and race: order them on one
    stream.  Returns the device address of the scratch's status area (with the
    device it lives on), for ``noalloc_status``.
    """
    shape = _shape_of(fwd["x"], fwd["B"])
    if tuple(rev["x"].shape) != tuple(fwd["x"].shape) or tuple(rev["B"].shape) != tuple(fwd["B"].shape):
        raise ValueError("forward and reverse parameters must have the same shapes")
    x = fwd["x"]
    if out.shape != x.shape or out.dtype != x.dtype or out.device != x.device or not out.is_contiguous():
        raise ValueError(f"out must be a contiguous {x.dtype} tensor of shape {tuple(x.shape)} on {x.device}")
    pf = _params(x, fwd["dt"], fwd["A"], fwd["B"], fwd["C"], fwd.get("D"))
    pr = _params(rev["x"], rev["dt"], rev["A"], rev["B"], rev["C"], rev.get("D"))
    area = ctypes.c_void_p()
    dev = x.device.index if x.device.index is not None else torch.cuda.current_device()
    with torch.cuda.device(dev):
        _check(lib.bidir_ssd_noalloc(ctypes.byref(shape), ctypes.byref(pf), ctypes.byref(pr), int(chunk),
                                     out.data_ptr(), _stream(x.device), ctypes.byref(area)))
    return NoallocArea(int(area.value or 0), dev)


def noalloc_status(area: NoallocArea) -> None:
    """Raise SSDError if a bounded device-side wait gave up in the ``bidir_ssd_noalloc`` call that
    returned ``area`` (read on that call's device, whatever device is current now)."""
    if not isinstance(area, NoallocArea):
        raise TypeError("pass the value bidir_ssd_noalloc returned (it carries the device of the call)")
    if area:
        with torch.cuda.device(area.device):
            _check(lib.ssd_workspace_status(int(area), 256, _stream(torch.device("cuda", area.device))))
