"""Seeded synthetic inputs for the bidirectional SSD scan.

This module is shared by the tests, the bench and the smoke check.  It draws
random numbers and rounds them to the storage dtypes; it holds none of the
scan's arithmetic.

Generator
---------
Every tensor has its own counter-based stream: element ``i`` of tensor
``tensor_id`` under ``seed`` is a pure function of ``(seed, tensor_id, i)``,
so any element (or any sampled subset) can be regenerated on its own.

* 64-bit mixing: the SplitMix64 finaliser (Steele, Lea & Flood, "Fast
  splittable pseudorandom number generators", OOPSLA 2014): add the golden
  gamma 0x9E3779B97F4A7C15, then ``z ^= z >> 30; z *= 0xBF58476D1CE4E5B9;
  z ^= z >> 27; z *= 0x94D049BB133111EB; z ^= z >> 31``.
* uniforms: the top 53 bits of a mixed word, offset by half an ulp, give a
  double in the open interval (0, 1).
* normals: Box-Muller, ``sqrt(-2 ln u1) * cos(2 pi u2)``, in float64.

Distributions (the layer-shape workloads of the bidirectional SSD mixer):
x ~ N(0,1); dt = softplus(N(0,1) - 4) (dt arrives positive, so the scan does
no softplus of its own); A_h = -exp(U(0, ln 16)) in [-16, -1];
B, C ~ N(0,1)/sqrt(d_state); D ~ U(0,1); residual ~ N(0,1); gate s ~ U(0, 0.5).

Rounding: values are drawn in float64, rounded to float32 (round to nearest
even), and, for bf16 tensors, rounded again float32 -> bf16 (nearest even).
A and D are always float32.

Tensor ids: forward {x:0, dt:1, A:2, B:3, C:4, D:5}; reverse adds 16;
residual 32; gate 33; step k of a multi-step workload adds 64*k.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
import threading
from dataclasses import dataclass, field

import numpy as np

_GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)

TENSOR_IDS = {"x": 0, "dt": 1, "A": 2, "B": 3, "C": 4, "D": 5}
REV_OFFSET = 16
RESIDUAL_ID = 32
GATE_ID = 33
STEP_STRIDE = 64

def _mix64(z: np.ndarray) -> np.ndarray:
    z = z ^ (z >> np.uint64(30))
    z = z * _M1
    z = z ^ (z >> np.uint64(27))
    z = z * _M2
    return z ^ (z >> np.uint64(31))


def _stream_key(seed: int, tensor_id: int) -> np.uint64:
    with np.errstate(over="ignore"):
        k = np.array([(seed << 32) | tensor_id], dtype=np.uint64)
        return _mix64(k + _GOLDEN)[0]


def _uniform_pair(key: np.uint64, idx: np.ndarray):
    """Two independent uniforms in (0,1) for each flat index in ``idx`` (numpy restatement of gen.c)."""
    with np.errstate(over="ignore"):
        base = idx.astype(np.uint64) * np.uint64(2)
        w1 = _mix64(key + (base + np.uint64(1)) * _GOLDEN)
        w2 = _mix64(key + (base + np.uint64(2)) * _GOLDEN)
    scale = 2.0 ** -53
    u1 = ((w1 >> np.uint64(11)).astype(np.float64) + 0.5) * scale
    u2 = ((w2 >> np.uint64(11)).astype(np.float64) + 0.5) * scale
    return u1, u2


_GEN_SRC = os.path.join(os.path.dirname(os.path.abspath(__file__)), "gen.c")
_GEN_LIB = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libssdgen.so")
_gen = None
_gen_lock = threading.Lock()


def _genlib():
    """The compiled bulk generator (gcc, built on first use)."""
    global _gen
    with _gen_lock:
        if _gen is None:
            if (not os.path.exists(_GEN_LIB)) or os.path.getmtime(_GEN_LIB) < os.path.getmtime(_GEN_SRC):
                tmp = _GEN_LIB + f".tmp{os.getpid()}"
                subprocess.check_call(["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-pthread",
                                       "-o", tmp, _GEN_SRC, "-lm"])
                os.replace(tmp, _GEN_LIB)
            lib = ctypes.CDLL(_GEN_LIB)
            lib.gen_stream.argtypes = [ctypes.c_uint64, ctypes.c_uint64, ctypes.c_int, ctypes.c_int64,
                                       ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p, ctypes.c_int]
            lib.gen_stream.restype = ctypes.c_int
            _gen = lib
    return _gen


def _threads() -> int:
    return len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else (os.cpu_count() or 1)


def _stream(seed: int, tensor_id: int, normal_dist: bool, n: int, idx, start: int = 0) -> np.ndarray:
    if idx is not None:
        idx = np.ascontiguousarray(np.asarray(idx, dtype=np.int64))
        n = idx.size
    out = np.empty(n, dtype=np.float64)
    rc = _genlib().gen_stream(seed, tensor_id, 1 if normal_dist else 0, start,
                              idx.ctypes.data if idx is not None else None, n, out.ctypes.data, _threads())
    if rc != 0:
        raise MemoryError("input generator failed")
    return out


def uniform(seed: int, tensor_id: int, n: int, idx=None) -> np.ndarray:
    """Uniform(0,1) stream: n elements, or the elements at flat indices ``idx``."""
    return _stream(seed, tensor_id, False, n, idx)


def normal(seed: int, tensor_id: int, n: int, idx=None) -> np.ndarray:
    """Standard normal stream (Box-Muller): n elements, or the elements at flat indices ``idx``."""
    return _stream(seed, tensor_id, True, n, idx)


# ---------------------------------------------------------------- rounding

def f64_to_f32(a: np.ndarray) -> np.ndarray:
    return np.asarray(a, dtype=np.float64).astype(np.float32)  # IEEE RNE


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit patterns (uint16), round to nearest even (finite inputs)."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    r = (u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


# ---------------------------------------------------------------- tensors

@dataclass
class Stored:
    """One stored tensor: its storage dtype, the stored bits and the exact value as float64."""
    dtype: str                 # "bf16" or "f32"
    shape: tuple
    data: np.ndarray           # uint16 bit patterns (bf16) or float32 values

    def f64(self) -> np.ndarray:
        if self.dtype == "bf16":
            return bf16_bits_to_f32(self.data).astype(np.float64).reshape(self.shape)
        return self.data.astype(np.float64).reshape(self.shape)

    def torch(self, device="cpu"):
        import torch
        if self.dtype == "bf16":
            t = torch.from_numpy(self.data.view(np.int16).reshape(self.shape)).view(torch.bfloat16)
        else:
            t = torch.from_numpy(self.data.reshape(self.shape))
        return t.to(device) if device != "cpu" else t


def _store(vals64: np.ndarray, dtype: str, shape) -> Stored:
    f32 = f64_to_f32(vals64)
    if dtype == "bf16":
        return Stored("bf16", tuple(shape), f32_to_bf16_bits(f32))
    return Stored("f32", tuple(shape), f32)


_SLICE = 1 << 25


def _gen_tensor(seed: int, tensor_id: int, shape, dtype: str, normal_dist: bool, transform=None) -> Stored:
    """Draws a whole tensor slice by slice (bounded float64 temporaries) and rounds it to ``dtype``."""
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.uint16 if dtype == "bf16" else np.float32)
    for s0 in range(0, n, _SLICE):
        m = min(_SLICE, n - s0)
        v = _stream(seed, tensor_id, normal_dist, m, None, start=s0)
        if transform is not None:
            v = transform(v)
        f32 = f64_to_f32(v)
        out[s0:s0 + m] = f32_to_bf16_bits(f32) if dtype == "bf16" else f32
    return Stored(dtype, tuple(shape), out)


@dataclass
class Shape:
    batch: int
    seqlen: int
    nheads: int
    headdim: int
    dstate: int
    ngroups: int = 1
    io: str = "bf16"           # dtype of x, dt, B, C, y, residual

    @property
    def tokens(self) -> int:
        return self.batch * self.seqlen


@dataclass
class Params:
    """One direction's parameter set (x, dt, A, B, C, D)."""
    x: Stored
    dt: Stored
    A: Stored
    B: Stored
    C: Stored
    D: Stored
    extra: dict = field(default_factory=dict)


def make_params(shape: Shape, seed: int = 0, offset: int = 0, with_D: bool = True) -> Params:
    """Generate one direction's parameters; ``offset`` is added to every tensor id."""
    b, L, H, P, N, G = (shape.batch, shape.seqlen, shape.nheads, shape.headdim,
                        shape.dstate, shape.ngroups)
    tid = {k: v + offset for k, v in TENSOR_IDS.items()}
    io = shape.io
    A = -np.exp(uniform(seed, tid["A"], H) * math.log(16.0))
    D = uniform(seed, tid["D"], H) if with_D else np.zeros(H)
    return Params(
        x=_gen_tensor(seed, tid["x"], (b, L, H, P), io, True),
        dt=_gen_tensor(seed, tid["dt"], (b, L, H), io, True, lambda z: np.log1p(np.exp(z - 4.0))),
        A=_store(A, "f32", (H,)),
        B=_gen_tensor(seed, tid["B"], (b, L, G, N), io, True, lambda z: z / math.sqrt(N)),
        C=_gen_tensor(seed, tid["C"], (b, L, G, N), io, True, lambda z: z / math.sqrt(N)),
        D=_store(D, "f32", (H,)),
        extra={"with_D": with_D},
    )


def make_bidir(shape: Shape, seed: int = 0, step: int = 0, with_D: bool = True):
    """Forward and reverse parameter sets (independent draws, as two separate layers)."""
    base = STEP_STRIDE * step
    return (make_params(shape, seed, base, with_D),
            make_params(shape, seed, base + REV_OFFSET, with_D))


def make_residual(shape: Shape, seed: int = 0, step: int = 0) -> Stored:
    b, L, H, P = shape.batch, shape.seqlen, shape.nheads, shape.headdim
    return _gen_tensor(seed, RESIDUAL_ID + STEP_STRIDE * step, (b, L, H * P), shape.io, True)


def make_gate(seed: int = 0, step: int = 0) -> float:
    """Gate scalar s ~ U(0, 0.5), stored as float32."""
    u = uniform(seed, GATE_ID + STEP_STRIDE * step, 1)[0]
    return float(np.float32(0.5 * u))


# ------------------------------------------------------------- the Mamba-2 mixer around the scan

MIXER_U_ID = 200            # the layer input, shared by both layers
MIXER_IDS = {"W_in": 201, "conv_w": 202, "conv_b": 203, "dt_bias": 204, "A": 205, "D": 206, "norm_w": 207,
             "W_out": 208}
MIXER_REV_OFFSET = 16


@dataclass
class MixerShape:
    batch: int
    seqlen: int
    d_model: int
    nheads: int
    headdim: int = 64
    dstate: int = 128
    ngroups: int = 1
    d_conv: int = 4

    @property
    def d_inner(self) -> int:
        return self.nheads * self.headdim

    @property
    def conv_dim(self) -> int:
        return self.d_inner + 2 * self.ngroups * self.dstate

    @property
    def d_in_proj(self) -> int:
        return 2 * self.d_inner + 2 * self.ngroups * self.dstate + self.nheads

    @property
    def tokens(self) -> int:
        return self.batch * self.seqlen


def make_mixer_input(shape: MixerShape, seed: int = 0) -> Stored:
    """The layer input u [b, L, d_model] ~ N(0, 1), bf16."""
    return _gen_tensor(seed, MIXER_U_ID, (shape.batch, shape.seqlen, shape.d_model), "bf16", True)


def make_mixer_layer(shape: MixerShape, seed: int = 0, offset: int = 0) -> dict:
    """One Mamba-2 layer's weights.  Projections bf16 (N(0, 1/fan_in)); conv taps U(-1/2, 1/2) and
    bias 0.1 N(0, 1), float32; dt_bias the inverse softplus of dt ~ exp(U(ln 1e-3, ln 1e-1));
    A = -exp(U(0, ln 16)); D ~ U(0, 1); norm weight 1 + 0.1 N(0, 1)."""
    t = {k: v + offset for k, v in MIXER_IDS.items()}
    H, dm, di, cd, K = shape.nheads, shape.d_model, shape.d_inner, shape.conv_dim, shape.d_conv
    dt0 = np.exp(math.log(1e-3) + uniform(seed, t["dt_bias"], H) * (math.log(1e-1) - math.log(1e-3)))
    return {
        "W_in": _gen_tensor(seed, t["W_in"], (shape.d_in_proj, dm), "bf16", True, lambda z: z / math.sqrt(dm)),
        "conv_w": _store(uniform(seed, t["conv_w"], cd * K) - 0.5, "f32", (cd, K)),
        "conv_b": _store(0.1 * normal(seed, t["conv_b"], cd), "f32", (cd,)),
        "dt_bias": _store(dt0 + np.log(-np.expm1(-dt0)), "f32", (H,)),
        "A": _store(-np.exp(uniform(seed, t["A"], H) * math.log(16.0)), "f32", (H,)),
        "D": _store(uniform(seed, t["D"], H), "f32", (H,)),
        "norm_w": _store(1.0 + 0.1 * normal(seed, t["norm_w"], di), "f32", (di,)),
        "W_out": _gen_tensor(seed, t["W_out"], (dm, di), "bf16", True, lambda z: z / math.sqrt(di)),
    }


def make_mixer(shape: MixerShape, seed: int = 0):
    """Input and the forward and reverse layers' weights (two independent layers)."""
    return (make_mixer_input(shape, seed), make_mixer_layer(shape, seed, 0),
            make_mixer_layer(shape, seed, MIXER_REV_OFFSET))


# ------------------------------------------------------------- the DiffuMamba-H attention mixer

ATTN_IDS = {"q": 300, "k": 301, "v": 302, "u": 303, "W_qkv": 304, "W_o": 305}


@dataclass
class AttnShape:
    batch: int
    seqlen: int
    nheads: int
    headdim: int = 128
    d_model: int = 0          # the block's width (0: nheads * headdim)

    @property
    def width(self) -> int:
        return self.nheads * self.headdim

    @property
    def model(self) -> int:
        return self.d_model or self.width


def make_attention(shape: AttnShape, seed: int = 0):
    """q, k, v [b, L, H, D] ~ N(0, 1), bf16: projections of unit-variance activations, so the
    scaled scores q.k / sqrt(D) have unit variance."""
    dims = (shape.batch, shape.seqlen, shape.nheads, shape.headdim)
    return tuple(_gen_tensor(seed, ATTN_IDS[n], dims, "bf16", True) for n in ("q", "k", "v"))


def make_attention_layer(shape: AttnShape, seed: int = 0):
    """The block input u [b, L, d_model] ~ N(0, 1) and its weights W_qkv [3 H D, d_model],
    W_o [d_model, H D] ~ N(0, 1/fan_in), all bf16."""
    dm, w = shape.model, shape.width
    u = _gen_tensor(seed, ATTN_IDS["u"], (shape.batch, shape.seqlen, dm), "bf16", True)
    wqkv = _gen_tensor(seed, ATTN_IDS["W_qkv"], (3 * w, dm), "bf16", True, lambda z: z / math.sqrt(dm))
    wo = _gen_tensor(seed, ATTN_IDS["W_o"], (dm, w), "bf16", True, lambda z: z / math.sqrt(w))
    return u, wqkv, wo


# ------------------------------------------------------------- workloads

# The five workloads: a tiny fp32 case the oracle checks exhaustively, two
# bidirectional layer shapes of the DiffuMamba mixer (~240M and ~1.3B
# models), a batch-1 long-sequence scaling case, and the R2L sidecar block.
WORKLOADS = {
    "tiny_f32": dict(shape=Shape(1, 64, 2, 16, 16, 1, "f32"), chunk=16, kind="bidir"),
    "diffumamba_240m_L2048": dict(shape=Shape(8, 2048, 32, 64, 128, 1, "bf16"), chunk=256, kind="bidir"),
    "diffumamba_1p3b_L8192": dict(shape=Shape(4, 8192, 64, 64, 128, 1, "bf16"), chunk=256, kind="bidir"),
    "long_L32768": dict(shape=Shape(1, 32768, 64, 64, 128, 1, "bf16"), chunk=256, kind="bidir"),
    "long_L131072": dict(shape=Shape(1, 131072, 64, 64, 128, 1, "bf16"), chunk=256, kind="bidir"),
    "r2l_block_L32": dict(shape=Shape(8, 32, 32, 64, 64, 1, "bf16"), chunk=32, kind="r2l", steps=256),
}
