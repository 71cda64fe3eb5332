"""Device-side failure paths of the tensor-core forward, made to happen without
faulting the GPU.

* A bounded wait that runs out: ``gdelta_set_wait_timeout_test(1)`` makes the
  kernels first wait on an mbarrier that nothing completes, with the wait limit
  forced down by ``gdelta_set_wait_limit``; the call must come back, report
  GDELTA_ERR_TIMEOUT through the device status word, and leave the device
  usable (the next call matches the oracle).
* An fp16 operand out of range: keys scaled far beyond unit norm push the
  pivot-scaled operands past 6e4; the kernels must report GDELTA_ERR_RANGE.
* The same bounded-wait failure in the five-gate projection kernel and in the
  backward pass.
"""
import ctypes

import pytest
import torch

import oracle
import synth
from channel_gated_delta_b200 import (_fwd_struct, _native, gdelta_fwd_chunked, gdelta_gate_proj,
                                      gdelta_get_last_device_error, gdelta_set_wait_limit,
                                      gdelta_set_wait_timeout_test)
from tests.gpu_util import TOL_BF16, err, err_stored, sel_heads, to_dev

pytestmark = pytest.mark.gpu

TIMEOUT, RANGE = 5, 7


def _inputs(seed=11, T=300):
    return synth.generate(synth.GdnShape(B=2, T=T, H=2, dk=128, dv=128, dtype="bf16", hot_channels=6, seed=seed))


def _fwd(d, **kw):
    return gdelta_fwd_chunked(d["q"], d["k"], d["v"], d["b"], d["w"], d["z"], d["g"], d["log_alpha"],
                              gamma_stat=d["gamma_stat"], path="tc", **kw)


def _parity(inp):
    d = to_dev(inp)
    o = torch.empty(2, inp["q"].shape[1], 2, 128, device="cuda")
    y, S = _fwd(d, o_raw=o)
    assert gdelta_get_last_device_error() == 0
    heads = oracle.all_heads(2, 2)
    ref = oracle.forward(inp, heads=heads)
    assert err_stored(sel_heads(y.cpu(), heads), ref["y"], "bf16") <= TOL_BF16
    assert err(sel_heads(o.cpu(), heads), ref["o_raw"]) <= TOL_BF16
    assert err(torch.stack([S.cpu()[b, h] for b, h in heads]), ref["S"]) <= TOL_BF16


@pytest.fixture
def restore_failure_controls():
    yield
    gdelta_set_wait_timeout_test(False)
    gdelta_set_wait_limit(0)


@pytest.mark.parametrize("polls", [8, 4096])
def test_wait_that_runs_out_reports_timeout_and_device_stays_usable(polls, restore_failure_controls):
    inp = _inputs()
    d = to_dev(inp)
    assert gdelta_get_last_device_error() == 0
    gdelta_set_wait_limit(polls)
    gdelta_set_wait_timeout_test(True)
    _fwd(d)                                           # queued without error; the kernels give up on the wait
    assert gdelta_get_last_device_error() == TIMEOUT
    assert gdelta_get_last_device_error() == 0        # reading clears the word
    gdelta_set_wait_timeout_test(False)
    gdelta_set_wait_limit(0)
    _parity(inp)                                      # the context is intact


def test_wait_timeout_through_the_allocation_free_entry_point(restore_failure_controls):
    d = to_dev(_inputs(seed=12, T=200))
    y = torch.empty(2, 200, 2, 128, dtype=torch.bfloat16, device="cuda")
    gdelta_set_wait_limit(64)
    gdelta_set_wait_timeout_test(True)
    a = _fwd_struct(d["q"], d["k"], d["v"], d["b"], d["w"], d["z"], d["g"], d["log_alpha"], d["gamma_stat"],
                    None, None, y, None, 64, 1e-6, "tc", None)
    lib = _native.load()
    assert lib.gdelta_fwd_chunked_noalloc(ctypes.byref(a), torch.cuda.current_stream().cuda_stream) == 0
    assert gdelta_get_last_device_error() == TIMEOUT


def test_out_of_range_operand_reports_range_error():
    inp = _inputs(seed=13, T=200)
    d = to_dev(inp)
    d["k"] = (d["k"].float() * 1e5).to(torch.bfloat16)   # |k| ~ 1e4 .. 4e4 before the decay factors
    assert gdelta_get_last_device_error() == 0
    _fwd(d)
    assert gdelta_get_last_device_error() == RANGE
    _parity(inp)


def test_wait_limit_setters_validate_and_restore(restore_failure_controls):
    lib = _native.load()
    assert lib.gdelta_set_wait_timeout_test(2) == 1    # GDELTA_ERR_INVALID_ARG
    assert lib.gdelta_set_wait_limit(0) == 0
    assert lib.gdelta_set_wait_limit(123) == 0
    assert lib.gdelta_set_wait_limit(0) == 0           # back to the default
    _parity(_inputs(seed=14, T=130))



def test_gate_projection_wait_that_runs_out(restore_failure_controls):
    inp = {k: v.cuda() for k, v in synth.gate_proj_inputs(200, 256, seed=15).items()}
    gdelta_set_wait_limit(32)
    gdelta_set_wait_timeout_test(True)
    gdelta_gate_proj(inp["x"], inp["w_down"], inp["w_up"], inp["bias"])
    assert gdelta_get_last_device_error() == TIMEOUT
    gdelta_set_wait_timeout_test(False)
    gdelta_set_wait_limit(0)
    out = gdelta_gate_proj(inp["x"], inp["w_down"], inp["w_up"], inp["bias"])
    assert gdelta_get_last_device_error() == 0
    from oracle import gate_proj as ogp
    ref = ogp.project(inp["x"].cpu(), inp["w_down"].cpu(), inp["w_up"].cpu(), inp["bias"].cpu())
    assert err(out["log_alpha"].cpu(), ref["log_alpha"]) <= TOL_BF16


def test_backward_wait_that_runs_out_reports_timeout(restore_failure_controls):
    """gdelta_bwd reports a bounded wait that runs out through the same status
    word (both CTAs of each cluster leave before any cluster barrier), and the
    next call matches the float64 autograd oracle."""
    import channel_gated_delta_b200 as gd
    from oracle import backward as ob
    inp = synth.generate(synth.GdnShape(B=1, T=40, H=1, dk=128, dv=128, dtype="bf16", hot_channels=6, seed=21))
    d = to_dev(inp)
    dy = torch.randn(1, 40, 1, 128, generator=torch.Generator().manual_seed(21))

    def call():
        return gd.gdelta_bwd(d["q"], d["k"], d["v"], d["b"], d["w"], d["z"], d["g"], d["log_alpha"], dy.cuda(),
                             gamma_stat=d["gamma_stat"])

    assert gdelta_get_last_device_error() == 0
    gdelta_set_wait_limit(64)
    gdelta_set_wait_timeout_test(True)
    call()
    assert gdelta_get_last_device_error() == TIMEOUT
    gdelta_set_wait_timeout_test(False)
    gdelta_set_wait_limit(0)
    g = call()
    torch.cuda.synchronize()
    assert gdelta_get_last_device_error() == 0
    ref = ob.backward(inp, dy.numpy(), heads=oracle.all_heads(1, 1))
    for key in ("q", "k", "v", "b", "w", "z", "g", "log_alpha"):
        assert err(sel_heads(g[key].cpu(), oracle.all_heads(1, 1)), ref["d" + key]) <= 1e-4, key
