"""C-ABI host logic: exported symbols, argument checks, workspace sizing, path choice (CPU only).

Nothing here launches a kernel: every call either fails validation on the
host or is a pure host query.
"""
import ctypes
import glob
import os
import re
import subprocess

import pytest
import torch

import bidirectional_mamba_ssd_bidir_b200 as ssd

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        text = re.sub(r"//[^\n]*", "", text)
        for m in re.finditer(r"^[A-Za-z_][\w\s\*]*?\b([A-Za-z_]\w*)\s*\(", text, flags=re.M):
            if m.group(1) not in ("if", "while", "sizeof"):
                names.add(m.group(1))
    return sorted(names)


def test_header_declares_the_entry_points():
    names = _declared_functions()
    for n in ("ssd_scan", "bidir_ssd", "r2l_block_scan", "ssd_workspace_bytes", "ssd_status_string"):
        assert n in names


def test_library_exports_every_declared_symbol():
    names = _declared_functions()
    lib = ctypes.CDLL(ssd.library_path)
    for n in names:
        assert hasattr(lib, n), f"{n} declared in include/ but not exported"
    out = subprocess.run(["nm", "-D", "--defined-only", ssd.library_path], capture_output=True, text=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    assert set(names) <= exported


def test_tracing_code_only_in_the_tracing_build():
    """The product library exports no trace readers; the tracing build exports them and every ABI symbol."""
    out = subprocess.run(["nm", "-D", "--defined-only", ssd.library_path], capture_output=True, text=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    assert not {"ssd_debug_trace", "ssd_debug_cta_times"} & exported
    trace_path = os.path.join(os.path.dirname(ssd.library_path), "libbidirssd_trace.so")
    if not os.path.exists(trace_path):
        pytest.skip("tracing build not compiled")
    out = subprocess.run(["nm", "-D", "--defined-only", trace_path], capture_output=True, text=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    assert {"ssd_debug_trace", "ssd_debug_cta_times"} <= exported
    assert set(_declared_functions()) <= exported


def _shape(b=1, L=64, H=2, P=16, N=16, G=1, io=1):
    return ssd._Shape(b, L, H, P, N, G, io)


def _ws(shape, chunk):
    return ssd.lib.ssd_workspace_bytes(ctypes.byref(shape), chunk)


def test_workspace_bytes_and_refusals():
    assert _ws(_shape(), 16) >= 256
    assert _ws(_shape(L=60), 16) == 0            # seqlen not a multiple of chunk
    assert _ws(_shape(P=48), 16) == 0            # unsupported headdim
    assert _ws(_shape(N=256), 16) == 0           # unsupported dstate
    assert _ws(_shape(H=3, G=2), 16) == 0        # heads not divisible by groups
    assert _ws(_shape(), 24) == 0                # unsupported chunk
    # SIMT workspace holds one fp32 state per (batch, head, chunk) plus decays
    s = _shape(b=2, L=128, H=4, P=64, N=128, io=1)
    units = 2 * 4 * (128 // 32)
    assert _ws(s, 32) >= units * 64 * 128 * 4
    # a single chunk still gets the state buffer: ssd_scan_state carries a state into and out
    # of it (block-wise decoding of one chunk-sized block)
    assert _ws(_shape(b=8, L=32, H=32, P=64, N=64, io=0), 32) >= 256 + 8 * 32 * 64 * 64 * 4


def test_path_choice():
    assert ssd.path_for((1, 64, 2, 16, 16, 1), torch.float32, 16) == 0
    assert ssd.path_for((1, 60, 2, 16, 16, 1), torch.float32, 16) == -1


def _call_scan(shape, params, chunk=16, direction=1, y=None, ws=None, wsb=0):
    return ssd.lib.ssd_scan(ctypes.byref(shape), ctypes.byref(params) if params else None, direction, chunk,
                            y, ws, wsb, None)


def _fake_params(ptr=1 << 20):
    return ssd._Params(ptr, ptr, ptr, ptr, ptr, None)


def test_validation_statuses():
    s = _shape()
    good = 1 << 20
    need = _ws(s, 16)
    assert _call_scan(s, _fake_params(), chunk=24, y=good, ws=good, wsb=need) == 2         # unsupported chunk
    assert _call_scan(_shape(L=60), _fake_params(), y=good, ws=good, wsb=need) == 1       # ragged length
    assert b"multiple of chunk" in ssd.lib.ssd_last_error()
    assert _call_scan(s, None, y=good, ws=good, wsb=need) == 1                            # NULL params
    assert _call_scan(s, _fake_params(), y=None, ws=good, wsb=need) == 1                  # NULL output
    assert _call_scan(s, _fake_params(), y=good + 4, ws=good, wsb=need) == 1              # misaligned output
    assert _call_scan(s, _fake_params(), y=good, ws=good, wsb=need - 1) == 1              # short workspace
    assert _call_scan(s, _fake_params(), y=good, ws=good + 16, wsb=need) == 1             # misaligned workspace
    assert _call_scan(s, _fake_params(), direction=0, y=good, ws=good, wsb=need) == 1     # bad direction
    assert _call_scan(s, _fake_params(good + 8), y=good, ws=good, wsb=need) == 1          # misaligned x
    assert _call_scan(_shape(P=48), _fake_params(), y=good, ws=good, wsb=need) == 2
    assert ssd.lib.ssd_status_string(4) == b"device wait timed out"


def test_empty_problem_is_a_no_op():
    s = _shape(b=0)
    assert _call_scan(s, _fake_params(), y=1 << 20, ws=1 << 20, wsb=_ws(s, 16)) == 0
    assert _call_scan(s, None, y=None, ws=None, wsb=0) == 0   # nothing to compute: pointers unused


def test_python_binding_refuses_cpu_tensors():
    x = torch.zeros(1, 16, 2, 16)
    with pytest.raises(ValueError):
        ssd.ssd_scan(x, torch.zeros(1, 16, 2), torch.zeros(2), torch.zeros(1, 16, 1, 16),
                     torch.zeros(1, 16, 1, 16), chunk=16)


def test_python_binding_checks_dtypes():
    x = torch.zeros(1, 16, 2, 16, dtype=torch.float16)
    with pytest.raises(TypeError):
        ssd.ssd_scan(x, torch.zeros(1, 16, 2), torch.zeros(2), torch.zeros(1, 16, 1, 16),
                     torch.zeros(1, 16, 1, 16), chunk=16)


def test_segment_query():
    # float32 and small head dims take the SIMT path, which never segments; refused shapes say -1
    assert ssd.segments_for((1, 64, 2, 16, 16, 1), torch.float32, 16) == 0
    assert ssd.segments_for((1, 60, 2, 16, 16, 1), torch.float32, 16) == -1


def test_mixer_and_attention_refusals():
    """Host-side refusals of the mixer, attention and GEMM entry points (no kernel is launched)."""
    ms = ssd._MixerShape(1, 256, 256, 8, 64, 128, 1, 4)
    assert ssd.lib.ssd_mixer_workspace_bytes(ctypes.byref(ms)) > 0
    for bad in (ssd._MixerShape(1, 256, 256, 8, 32, 128, 1, 4),      # headdim 32
                ssd._MixerShape(1, 200, 256, 8, 64, 128, 1, 4),      # seqlen not a multiple of 128
                ssd._MixerShape(1, 256, 256, 12, 64, 128, 1, 4),     # heads not a multiple of 8
                ssd._MixerShape(1, 256, 256, 264, 64, 128, 1, 4),    # more than 256 heads
                ssd._MixerShape(1, 256, 256, 8, 64, 128, 1, 9)):     # conv wider than 8
        assert ssd.lib.ssd_mixer_workspace_bytes(ctypes.byref(bad)) == 0
    good = 1 << 20
    a = ssd._AttnShape(1, 128, 2, 96)                                  # headdim 96: refused
    assert ssd.lib.ssd_attention(ctypes.byref(a), good, 192, good, 192, good, 192, good, 192, 0.0, good, 256,
                                 None) == 2
    assert ssd.lib.ssd_attention_block_workspace_bytes(ctypes.byref(a)) == 0
    assert ssd.lib.ssd_attention(None, good, 256, good, 256, good, 256, good, 256, 0.0, good, 256, None) == 1
    neg = ssd._AttnShape(-1, 128, 2, 128)
    assert ssd.lib.ssd_attention(ctypes.byref(neg), good, 256, good, 256, good, 256, good, 256, 0.0, good, 256,
                                 None) == 1
    assert ssd.lib.ssd_gemm_bf16(-1, 8, 64, good, good, good, good, 256, None) == 1
    assert ssd.lib.ssd_gemm_bf16(0, 8, 64, good, good, good, good, 256, None) == 0     # empty: a no-op
