"""Five-gate low-rank projection (Muir review §2.3) on the GPU against the
float64 oracle (``oracle.gate_proj``): the activated gates element by element
on a ragged token count and several column tiles, sampled rows of the Muir
1.34B-scale layer (N = 4 x 4096 tokens, d = 2048), other rank splits, and the
projection feeding the chunked forward, compared with the oracle projection
feeding the oracle recurrence."""
import numpy as np
import pytest
import torch

import oracle
import synth
from channel_gated_delta_b200 import gdelta_fwd_chunked, gdelta_gate_proj, gdelta_get_last_device_error
from oracle import gate_proj as ogp
from tests.gpu_util import TOL_BF16, err, err_stored, sel_heads

pytestmark = pytest.mark.gpu


def _check(out, ref, rows=None):
    sel = (lambda t: t.cpu()) if rows is None else (lambda t: t.cpu()[rows])
    assert err(sel(out["log_alpha"]), ref["log_alpha"]) <= TOL_BF16
    for n in ("b", "g", "w", "z"):
        assert err_stored(sel(out[n]), ref[n], "bf16") <= TOL_BF16, n


def _run(inp, ranks=synth.GATE_RANKS):
    d = {k: v.cuda() for k, v in inp.items()}
    out = gdelta_gate_proj(d["x"], d["w_down"], d["w_up"], d["bias"], ranks=ranks)
    torch.cuda.synchronize()
    assert gdelta_get_last_device_error() == 0
    return out


@pytest.mark.parametrize("N,d", [(300, 512), (128, 256), (1, 768)])
def test_gate_proj_matches_oracle(N, d):
    inp = synth.gate_proj_inputs(N, d, seed=N + d)
    out = _run(inp)
    _check(out, ogp.project(inp["x"], inp["w_down"], inp["w_up"], inp["bias"]))


@pytest.mark.parametrize("ranks", [(64, 64, 64, 64, 256), (128, 128, 128, 128, 256)])
def test_gate_proj_other_rank_splits(ranks):
    inp = synth.gate_proj_inputs(200, 512, ranks=ranks, seed=5)
    out = _run(inp, ranks)
    _check(out, ogp.project(inp["x"], inp["w_down"], inp["w_up"], inp["bias"], ranks))


def test_gate_proj_full_layer_sampled_rows():
    """The Muir 1.34B-scale layer in the benchmark's launch: N = 16384 tokens,
    d = 2048; rows are independent, so the oracle recomputes a sample (first,
    last, and rows across tile boundaries)."""
    inp = synth.gate_proj_inputs(4 * 4096, 2048, seed=1)
    out = _run(inp)
    rows = [0, 1, 127, 128, 5000, 8191, 12345, 16256, 16383]
    ref = ogp.project(inp["x"][rows], inp["w_down"], inp["w_up"], inp["bias"])
    _check(out, ref, rows)
    assert all(torch.isfinite(out[n].float()).all() for n in out)


def test_gate_proj_feeds_the_chunked_forward():
    """x -> projection -> forward on the GPU against x -> oracle projection
    (gates quantised as the kernels store them) -> oracle recurrence."""
    B, T, H = 1, 200, 4
    d = 128 * H
    inp = synth.gate_proj_inputs(B * T, d, seed=9)
    tok = synth.generate(synth.GdnShape(B=B, T=T, H=H, dk=128, dv=128, dtype="bf16", hot_channels=6, seed=9))
    out = _run(inp)
    shp = (B, T, H, 128)
    gates = {n: out[n].view(shp) for n in ("b", "g", "w", "z")}
    la = out["log_alpha"].view(shp)
    q, k, v = tok["q"].cuda(), tok["k"].cuda(), tok["v"].cuda()
    gamma = tok["gamma_stat"].cuda()
    o = torch.empty(B, T, H, 128, device="cuda")
    y, S = gdelta_fwd_chunked(q, k, v, gates["b"], gates["w"], gates["z"], gates["g"], la, gamma_stat=gamma, o_raw=o)
    torch.cuda.synchronize()
    assert gdelta_get_last_device_error() == 0
    ref_g = ogp.project(inp["x"], inp["w_down"], inp["w_up"], inp["bias"])
    ref_in = {"q": tok["q"], "k": tok["k"], "v": tok["v"], "gamma_stat": tok["gamma_stat"],
              "log_alpha": torch.from_numpy(ref_g["log_alpha"]).float().view(shp)}
    for n in ("b", "g", "w", "z"):
        ref_in[n] = torch.from_numpy(ref_g[n]).to(torch.bfloat16).view(shp)
    heads = oracle.all_heads(B, H)
    ref = oracle.forward(ref_in, heads=heads)
    assert err_stored(sel_heads(y.cpu(), heads), ref["y"], "bf16") <= TOL_BF16
    assert err(sel_heads(o.cpu(), heads), ref["o_raw"]) <= TOL_BF16
    assert err(torch.stack([S.cpu()[b, h] for b, h in heads]), ref["S"]) <= TOL_BF16
