"""The allocation-free forward, gdelta_fwd_chunked_noalloc.

Callers that cannot allocate device memory when they run the forward (a
runtime that plans all device memory in advance, or latency-critical code
that must not call cudaMalloc) use this entry point; its scratch is a fixed
array inside the library.  These tests call it through the C ABI and compare
it with gdelta_fwd_chunked given a torch-allocated workspace, on two calls in
a row (the second with different inputs, so stale scratch from the first call
would show).  This file is collected last on purpose.
"""
import ctypes

import pytest
import torch

import synth
from channel_gated_delta_b200 import _fwd_struct, _native, gdelta_fwd_chunked
from tests.gpu_util import TOL_BF16, err, to_dev

pytestmark = pytest.mark.gpu


def _run_noalloc(d, y, S, o):
    lib = _native.load()
    a = _fwd_struct(d["q"], d["k"], d["v"], d["b"], d["w"], d["z"], d["g"], d["log_alpha"], d["gamma_stat"],
                    None, S, y, o, 64, 1e-6, "auto", None)
    st = lib.gdelta_fwd_chunked_noalloc(ctypes.byref(a), torch.cuda.current_stream().cuda_stream)
    return st


def _shape(seed, T):
    return synth.GdnShape(B=2, T=T, H=4, dk=128, dv=128, dtype="bf16", hot_channels=6, seed=seed)


def test_noalloc_matches_workspace_entry_point_twice():
    for call, (seed, T) in enumerate([(21, 1000), (22, 777)]):
        d = to_dev(synth.generate(_shape(seed, T)))
        B, H = 2, 4
        y = torch.empty(B, T, H, 128, dtype=torch.bfloat16, device="cuda")
        S = torch.empty(B, H, 128, 128, device="cuda")
        o = torch.empty(B, T, H, 128, device="cuda")
        assert _run_noalloc(d, y, S, o) == 0, f"call {call}"
        o_ref = torch.empty_like(o)
        y_ref, S_ref = gdelta_fwd_chunked(d["q"], d["k"], d["v"], d["b"], d["w"], d["z"], d["g"], d["log_alpha"],
                                          gamma_stat=d["gamma_stat"], o_raw=o_ref)
        torch.cuda.synchronize()
        assert err(o.cpu(), o_ref.cpu().double().numpy()) <= TOL_BF16
        assert err(S.cpu(), S_ref.cpu().double().numpy()) <= TOL_BF16
        assert err(y.float().cpu(), y_ref.float().cpu().double().numpy()) <= TOL_BF16


def test_noalloc_rejects_problems_beyond_its_scratch():
    # 8 heads x 2500 tokens needs 8 x 40 windows x 105 KiB > 32 MiB
    d = to_dev(synth.generate(synth.GdnShape(B=2, T=2500, H=4, dk=128, dv=128, dtype="bf16", seed=3)))
    y = torch.empty(2, 2500, 4, 128, dtype=torch.bfloat16, device="cuda")
    assert _run_noalloc(d, y, None, None) == 6          # GDELTA_ERR_WORKSPACE
