"""The allocation-free forward, gdelta_fwd_chunked_noalloc.

Callers that cannot allocate device memory when they run the forward (a
runtime that plans all device memory in advance, or latency-critical code
that must not call cudaMalloc, which synchronises the device and can fail)
use this entry point; its scratch is a fixed array inside the library.  These
tests call it through the C ABI and compare it with gdelta_fwd_chunked given a
torch-allocated workspace.  Both run the same kernels on the same inputs, so
the outputs must be identical bit for bit; two calls in a row with different
inputs would show scratch left over from the first call.

The file name sorts last so that pytest collects it after every other test: if
it fails, a run that stops at the first failure has already run the rest.
"""
import ctypes

import pytest
import torch

import synth
from channel_gated_delta_b200 import _fwd_struct, _native, gdelta_fwd_chunked, gdelta_fwd_workspace_bytes
from tests.gpu_util import to_dev

pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 32 << 20
OK, UNSUPPORTED, WORKSPACE = 0, 2, 6


def _struct(d, y, S, o, path="auto"):
    return _fwd_struct(d["q"], d["k"], d["v"], d["b"], d["w"], d["z"], d["g"], d["log_alpha"], d["gamma_stat"],
                       None, S, y, o, 64, 1e-6, path, None)


def _run_noalloc(a):
    return _native.load().gdelta_fwd_chunked_noalloc(ctypes.byref(a), torch.cuda.current_stream().cuda_stream)


def _outputs(B, T, H, dtype):
    y = torch.empty(B, T, H, 128, dtype=dtype, device="cuda")
    S = torch.empty(B, H, 128, 128, device="cuda")
    o = torch.empty(B, T, H, 128, device="cuda")
    return y, S, o


def _compare_with_workspace_entry_point(d, B, T, H, dtype, path="auto"):
    y, S, o = _outputs(B, T, H, dtype)
    assert _run_noalloc(_struct(d, y, S, o, path)) == OK
    o_ref = torch.empty_like(o)
    y_ref, S_ref = gdelta_fwd_chunked(d["q"], d["k"], d["v"], d["b"], d["w"], d["z"], d["g"], d["log_alpha"],
                                      gamma_stat=d["gamma_stat"], o_raw=o_ref, path=path)
    torch.cuda.synchronize()
    assert torch.equal(y, y_ref)
    assert torch.equal(o, o_ref)
    assert torch.equal(S, S_ref)


def test_noalloc_matches_workspace_entry_point_bit_for_bit_twice():
    for seed, T in [(21, 1000), (22, 777)]:
        d = to_dev(synth.generate(synth.GdnShape(B=2, T=T, H=4, dk=128, dv=128, dtype="bf16", hot_channels=6,
                                                 seed=seed)))
        _compare_with_workspace_entry_point(d, 2, T, 4, torch.bfloat16)


def test_noalloc_without_scratch_on_the_fp32_path():
    # fp32 tokens run the CUDA-core kernel, which needs no scratch at all
    d = to_dev(synth.generate(synth.GdnShape(B=1, T=150, H=2, dk=128, dv=128, dtype="f32", seed=23)))
    assert gdelta_fwd_workspace_bytes(d["q"], d["k"], d["v"], d["b"], d["w"], d["z"], d["g"], d["log_alpha"]) == 0
    _compare_with_workspace_entry_point(d, 1, 150, 2, torch.float32)


def test_noalloc_passes_argument_errors_through():
    d = to_dev(synth.generate(synth.GdnShape(B=1, T=64, H=2, dk=128, dv=128, dtype="bf16", seed=24)))
    y, S, o = _outputs(1, 64, 2, torch.bfloat16)
    a = _struct(d, y, S, o)
    a.dk = 96                                               # not a supported head size
    lib = _native.load()
    expect = lib.gdelta_fwd_chunked(ctypes.byref(a), torch.cuda.current_stream().cuda_stream)
    assert expect == UNSUPPORTED
    assert _run_noalloc(a) == expect
    assert lib.gdelta_fwd_chunked_noalloc(None, None) == 1  # GDELTA_ERR_INVALID_ARG


def _need(B, T, H):
    q = torch.empty(B, T, H, 128, dtype=torch.bfloat16, device="cuda")
    la = torch.empty(B, T, H, 128, device="cuda")
    return gdelta_fwd_workspace_bytes(q, q, q, q, q, q, q, la)


def test_noalloc_capacity_edge():
    """The largest T that fits the fixed scratch runs and matches; one more
    token (one more window per head) is rejected before any launch."""
    B, H = 2, 4
    T = 64
    while _need(B, T + 64, H) <= SCRATCH_BYTES:
        T += 64
    assert _need(B, T, H) <= SCRATCH_BYTES < _need(B, T + 1, H)
    d = to_dev(synth.generate(synth.GdnShape(B=B, T=T + 1, H=H, dk=128, dv=128, dtype="bf16", seed=25)))
    y, S, o = _outputs(B, T + 1, H, torch.bfloat16)
    assert _run_noalloc(_struct(d, y, S, o)) == WORKSPACE
    d_fit = {k: (v[:, :T].contiguous() if v.dim() == 4 else v) for k, v in d.items()}
    _compare_with_workspace_entry_point(d_fit, B, T, H, torch.bfloat16)
