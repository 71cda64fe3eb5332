"""The C-ABI library loads, exports every declared symbol, and rejects bad
arguments on the host before any CUDA call (no GPU needed)."""
import ctypes
import os
import re

import pytest

from channel_gated_delta_b200 import _native

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gdelta.h")


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"GDELTA_API\s+[\w\s\*]*?\b(gdelta_\w+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(_native.LIB_PATH):
        from channel_gated_delta_b200 import build
        build.build()
    return _native.load()


def test_every_declared_symbol_is_exported(lib):
    names = declared_symbols()
    assert len(names) >= 8
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(_native.EXPORTED)


def test_abi_version_and_status_strings(lib):
    assert lib.gdelta_abi_version() == 4
    for code in range(8):
        s = lib.gdelta_status_string(code)
        assert s and s != b"unknown status"
    assert lib.gdelta_status_string(99) == b"unknown status"


def _args(**kw):
    a = _native.FwdArgs()
    a.B, a.T, a.H, a.dk, a.dv, a.chunk, a.dtype, a.path = 1, 64, 1, 128, 128, 64, 1, 0
    fake = 0x10000
    for i, n in enumerate(("q", "k", "z", "b", "v", "w", "g", "log_alpha", "y")):
        setattr(a, n, fake + 256 * i)
    a.eps = 1e-6
    for key, val in kw.items():
        setattr(a, key, val)
    return a


def test_host_validation_codes(lib):
    f = lib.gdelta_fwd_chunked
    assert f(None, None) == 1
    assert f(ctypes.byref(_args(B=0)), None) == 1
    assert f(ctypes.byref(_args(T=-1)), None) == 1
    assert f(ctypes.byref(_args(dk=96)), None) == 2
    assert f(ctypes.byref(_args(chunk=48)), None) == 2
    assert f(ctypes.byref(_args(dtype=7)), None) == 2
    assert f(ctypes.byref(_args(path=9)), None) == 1
    assert f(ctypes.byref(_args(q=None)), None) == 1
    assert f(ctypes.byref(_args(k=0x10001)), None) == 3
    assert f(ctypes.byref(_args(eps=float("nan"))), None) == 1
    assert lib.gdelta_fwd_selected_path(ctypes.byref(_args(B=0))) == -1
    assert lib.gdelta_fwd_workspace_bytes(ctypes.byref(_args(B=0))) == 0
    assert lib.gdelta_state_init(None, 1, 1, 128, 128, None, None) == 1
    assert lib.gdelta_state_init(0x10000, 1, 1, 100, 128, None, None) == 2
    assert lib.gdelta_state_init(0x10004, 1, 1, 128, 128, None, None) == 3
    # overlapping, unequal source and destination
    assert lib.gdelta_state_init(0x10000, 1, 1, 128, 128, 0x10010, None) == 1
    d = _native.DecodeArgs()
    d.B, d.H, d.dk, d.dv, d.dtype, d.reserved = 1, 1, 128, 128, 1, 0
    assert lib.gdelta_decode_step(ctypes.byref(d), None) == 1       # null tensors
    d.reserved = 3
    assert lib.gdelta_decode_step(ctypes.byref(d), None) == 1


def test_reduced_gate_forms_are_validated_on_the_host(lib):
    f = lib.gdelta_fwd_chunked
    beta = 0x20000
    # beta stands for b and w: giving it beside either is ambiguous
    assert f(ctypes.byref(_args(beta=beta)), None) == 1
    assert f(ctypes.byref(_args(beta=beta, b=None)), None) == 1
    assert f(ctypes.byref(_args(beta=beta, w=None)), None) == 1
    # without beta both per-channel gates are needed
    assert f(ctypes.byref(_args(b=None)), None) == 1
    assert f(ctypes.byref(_args(w=None)), None) == 1
    assert f(ctypes.byref(_args(decay_per_token=2)), None) == 1
    assert f(ctypes.byref(_args(qk_raw=2)), None) == 1
    assert lib.gdelta_fwd_selected_path(ctypes.byref(_args(beta=beta))) == -1
    assert f(ctypes.byref(_args(b=None, w=None, beta=beta + 2)), None) == 3     # beta 16-byte aligned too
    # accepted forms: no z; beta alone; beta with a per-token decay
    for kw in ({"z": None}, {"qk_raw": 1}, {"b": None, "w": None, "beta": beta},
               {"b": None, "w": None, "beta": beta, "decay_per_token": 1, "z": None}):
        assert lib.gdelta_fwd_selected_path(ctypes.byref(_args(**kw))) in (1, 2), kw
        assert lib.gdelta_fwd_workspace_bytes(ctypes.byref(_args(**kw))) >= 0
    d = _native.DecodeArgs()
    d.B, d.H, d.dk, d.dv, d.dtype = 1, 1, 128, 128, 1
    for i, n in enumerate(("q", "k", "b", "v", "w", "g", "log_alpha", "S", "y")):
        setattr(d, n, 0x10000 + 256 * i)
    d.eps = 1e-6
    d.beta = beta
    assert lib.gdelta_decode_step(ctypes.byref(d), None) == 1       # beta beside b and w
    d.beta, d.qk_raw = None, 2
    assert lib.gdelta_decode_step(ctypes.byref(d), None) == 1
    d.qk_raw, d.decay_per_token = 0, 5
    assert lib.gdelta_decode_step(ctypes.byref(d), None) == 1
    d.decay_per_token, d.b = 0, None
    assert lib.gdelta_decode_step(ctypes.byref(d), None) == 1       # b missing, no beta


def test_state_affine_validation(lib):
    f = lib.gdelta_state_affine
    S, A, S_in, D = 0x100000, 0x200000, 0x300000, 0x400000
    n = 128 * 128 * 4
    assert f(None, A, S_in, D, 1, 1, 128, 128, None) == 1
    assert f(S, None, S_in, D, 1, 1, 128, 128, None) == 1
    assert f(S, A, S_in, D, 0, 1, 128, 128, None) == 1
    assert f(S, A, S_in, D, 1, 1, 96, 128, None) == 2
    assert f(S, A + 4, S_in, D, 1, 1, 128, 128, None) == 3
    assert f(S, A, S + n // 2, D, 1, 1, 128, 128, None) == 1        # S_in overlaps S_out
    assert f(S, S + 16, S_in, D, 1, 1, 128, 128, None) == 1          # A overlaps S_out
    assert f(S, A, S_in, S + 16, 1, 1, 128, 128, None) == 1          # D partly over S_out


def _bwd_args(**kw):
    a = _native.BwdArgs()
    a.B, a.T, a.H, a.dk, a.dv, a.dtype = 1, 64, 1, 128, 128, 1
    names = ("q", "k", "z", "b", "v", "w", "g", "log_alpha", "grad_y", "grad_q", "grad_k", "grad_z",
             "grad_b", "grad_log_alpha", "grad_v", "grad_w", "grad_g")
    for i, n in enumerate(names):
        setattr(a, n, 0x100000 + 0x1000 * i)
    a.eps = 1e-6
    for key, val in kw.items():
        setattr(a, key, val)
    return a


def test_backward_validation(lib):
    f, wsb = lib.gdelta_bwd, lib.gdelta_bwd_workspace_bytes
    assert f(None, None) == 1
    assert f(ctypes.byref(_bwd_args(dk=64)), None) == 2                # d_k = d_v = 128 only
    assert f(ctypes.byref(_bwd_args(dtype=5)), None) == 2
    assert f(ctypes.byref(_bwd_args(grad_y=None)), None) == 1
    assert f(ctypes.byref(_bwd_args(grad_k=None)), None) == 1
    assert f(ctypes.byref(_bwd_args(q=0x100004)), None) == 3
    assert f(ctypes.byref(_bwd_args(eps=float("inf"))), None) == 1
    need = wsb(ctypes.byref(_bwd_args()))
    # per value half of the head: checkpoints (2 for 64 tokens, plus one spare) and
    # 33 chunk states of 32 KiB, and 128 floats; per token: 8 floats of RMS partials
    # and, per value half, the token's o and r on that half's 64 columns
    assert need == 2 * ((3 + 33) * 128 * 64 * 4 + 128 * 4) + 64 * 8 * 4 + 2 * 64 * 128 * 4
    assert f(ctypes.byref(_bwd_args(workspace=0x900000, workspace_bytes=need - 1)), None) == 6
    assert wsb(ctypes.byref(_bwd_args(dk=64))) == 0
    # no tokens: token tensors may be null
    empty = {n: None for n in ("q", "k", "z", "b", "v", "w", "g", "log_alpha", "grad_y")}
    assert wsb(ctypes.byref(_bwd_args(T=0, **empty))) > 0


def test_path_selection_is_host_logic(lib):
    a = _args()
    assert lib.gdelta_fwd_selected_path(ctypes.byref(a)) in (1, 2)
    assert lib.gdelta_fwd_selected_path(ctypes.byref(_args(dtype=0))) == 1
    assert lib.gdelta_fwd_selected_path(ctypes.byref(_args(path=1))) == 1
