"""GPU path vs the float64 oracle, element by element on the same seeded
inputs, through the C ABI.  Tolerances are max|diff| / rms(reference):
1e-4 for fp32 inputs, 2e-2 for bf16 inputs / fp32 accumulation."""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests.gpu_util import TOL_BF16, TOL_F32, err, err_stored, gpu_fwd, sel_heads, to_dev

pytestmark = pytest.mark.gpu


def _ref(inputs, heads=None, S0=None):
    return oracle.forward(inputs, heads=heads, S0=S0)


def _storage(t):
    return {torch.bfloat16: "bf16", torch.float16: "f16"}.get(t.dtype, "f32")


def _check(y, S, o, ref, heads, tol, S_heads=None):
    """y is compared allowing its 16-bit storage rounding; o_raw and S (fp32)
    with the plain max|diff|/rms bound."""
    ys = sel_heads(y, heads)
    os_ = sel_heads(o, heads) if o is not None else None
    e_y = err_stored(ys, ref["y"], _storage(y))
    e_o = err(os_, ref["o_raw"]) if os_ is not None else 0.0
    e_s = err(torch.stack([S[b, h] for (b, h) in heads]), ref["S"]) if S is not None else 0.0
    assert e_y <= tol and e_o <= tol and e_s <= tol, (e_y, e_o, e_s)
    return e_y, e_o, e_s


def test_tiny_f32_config_all_heads():
    inp = synth.generate_config("tiny_f32")
    y, S, o = gpu_fwd(inp)
    heads = oracle.all_heads(1, 2)
    _check(y, S, o, _ref(inp, heads), heads, TOL_F32)


@pytest.mark.parametrize("dk,dv", [(64, 64), (64, 128), (128, 64), (128, 128)])
@pytest.mark.parametrize("chunk", [16, 32, 64])
def test_f32_shapes_and_chunks_ragged(dk, dv, chunk):
    shape = synth.GdnShape(B=2, T=157, H=2, dk=dk, dv=dv, chunk=chunk, dtype="f32",
                           u_low=-5, u_high=-1, seed=dk + dv + chunk)
    inp = synth.generate(shape)
    y, S, o = gpu_fwd(inp, chunk=chunk, path="simt")
    heads = oracle.all_heads(2, 2)
    _check(y, S, o, _ref(inp, heads), heads, TOL_F32)


@pytest.mark.parametrize("path", ["auto", "simt"])
def test_bf16_several_chunks_ragged_tail(path):
    shape = synth.GdnShape(B=2, T=64 * 5 + 23, H=3, dk=128, dv=128, dtype="bf16",
                           hot_channels=6, seed=11)
    inp = synth.generate(shape)
    y, S, o = gpu_fwd(inp, path=path)
    heads = oracle.all_heads(2, 3)
    _check(y, S, o, _ref(inp, heads), heads, TOL_BF16)


def test_state_in_and_in_place_out():
    shape = synth.GdnShape(B=1, T=130, H=2, dk=64, dv=64, dtype="f32", u_low=-5, u_high=-1, seed=3)
    inp = synth.generate(shape)
    S0 = torch.randn(1, 2, 64, 64, generator=torch.Generator().manual_seed(1)) * 0.5
    d = to_dev(inp)
    S = S0.cuda()
    import channel_gated_delta_b200 as gd
    y, S_out = gd.gdelta_fwd_chunked(d["q"], d["k"], d["v"], d["b"], d["w"], d["z"], d["g"],
                                     d["log_alpha"], gamma_stat=d["gamma_stat"], S_in=S, S_out=S)
    torch.cuda.synchronize()
    heads = oracle.all_heads(1, 2)
    ref = _ref(inp, heads, S0=S0.reshape(2, 64, 64))
    assert S_out.data_ptr() == S.data_ptr()
    _check(y.cpu(), S.cpu(), None, ref, heads, TOL_F32)


def test_empty_and_single_token():
    import channel_gated_delta_b200 as gd
    shape = synth.GdnShape(B=2, T=1, H=2, dk=128, dv=128, dtype="f32", seed=4)
    inp = synth.generate(shape)
    S0 = torch.randn(2, 2, 128, 128, generator=torch.Generator().manual_seed(2))
    y, S, o = gpu_fwd(inp, S_in=S0.cuda())
    heads = oracle.all_heads(2, 2)
    _check(y, S, o, _ref(inp, heads, S0=S0.reshape(4, 128, 128)), heads, TOL_F32)
    # T = 0: the state passes through unchanged
    d = to_dev({k: v[:, :0] if v.dim() == 4 else v for k, v in inp.items()})
    y0, S_out = gd.gdelta_fwd_chunked(d["q"], d["k"], d["v"], d["b"], d["w"], d["z"], d["g"],
                                      d["log_alpha"], S_in=S0.cuda())
    torch.cuda.synchronize()
    assert y0.numel() == 0 and torch.equal(S_out.cpu(), S0)


def test_split_run_carries_state():
    shape = synth.GdnShape(B=1, T=300, H=2, dk=128, dv=128, dtype="bf16", seed=5)
    inp = synth.generate(shape)
    first = {k: (v[:, :131] if v.dim() == 4 else v) for k, v in inp.items()}
    second = {k: (v[:, 131:] if v.dim() == 4 else v) for k, v in inp.items()}
    y1, S1, _ = gpu_fwd(first)
    y2, S2, _ = gpu_fwd(second, S_in=S1.cuda())
    heads = oracle.all_heads(1, 2)
    ref = _ref(inp, heads)
    assert err_stored(sel_heads(torch.cat([y1, y2], 1), heads), ref["y"], "bf16") <= TOL_BF16
    assert err(torch.stack([S2[b, h] for b, h in heads]), ref["S"]) <= TOL_BF16


@pytest.mark.parametrize("name,heads", [
    ("layer350m_bf16", [(0, 0), (3, 5), (7, 7)]),
    ("muir1b3_bf16", [(0, 0), (1, 9), (3, 15)]),
    ("long32k_bf16", [(0, 0), (0, 11), (0, 15)]),
])
def test_full_size_configs_sampled_heads(name, heads):
    """Full workload in the benchmark's launch configuration; the oracle
    recomputes the sampled heads (heads are independent)."""
    inp = synth.generate_config(name)
    y, S, o = gpu_fwd(inp)
    assert torch.isfinite(y.float()).all()
    _check(y, S, o, _ref(inp, heads), heads, TOL_BF16)


def test_decode_after_forward_continues_the_sequence():
    """Decode steps after a chunked forward equal the forward over the
    concatenated tokens."""
    import channel_gated_delta_b200 as gd
    shape = synth.GdnShape(B=2, T=100, H=2, dk=128, dv=128, dtype="bf16", seed=6)
    inp = synth.generate(shape)
    pre = {k: (v[:, :96] if v.dim() == 4 else v) for k, v in inp.items()}
    _, S, _ = gpu_fwd(pre)
    S = S.cuda()
    d = to_dev(inp)
    ys = []
    for t in range(96, 100):
        tok = {k: d[k][:, t].contiguous() for k in ("q", "k", "v", "b", "w", "z", "g", "log_alpha")}
        ys.append(gd.gdelta_decode_step(tok["q"], tok["k"], tok["v"], tok["b"], tok["w"], tok["z"],
                                        tok["g"], tok["log_alpha"], S,
                                        gamma_stat=d["gamma_stat"]).cpu())
    torch.cuda.synchronize()
    heads = oracle.all_heads(2, 2)
    ref = _ref(inp, heads)
    y_dec = torch.stack(ys, 1)                          # [B,4,H,dv]
    assert err_stored(sel_heads(y_dec, heads), ref["y"][:, 96:], "bf16") <= TOL_BF16
    assert err(torch.stack([S.cpu()[b, h] for b, h in heads]), ref["S"]) <= TOL_BF16


@pytest.mark.parametrize("dk,dv,dtype", [(128, 128, "f32"), (64, 128, "f32"), (128, 64, "bf16"),
                                         (64, 64, "bf16")])
def test_decode_shapes(dk, dv, dtype):
    import channel_gated_delta_b200 as gd
    B, H, steps = 3, 2, 5
    gen = torch.Generator().manual_seed(dk + dv)
    S0 = torch.randn(B, H, dk, dv, generator=gen) * 0.3
    gamma = torch.exp(0.1 * torch.randn(H, dk, generator=gen))
    S = S0.cuda()
    heads = oracle.all_heads(B, H)
    Sref = S0.reshape(B * H, dk, dv).double().numpy()
    tol = TOL_F32 if dtype == "f32" else TOL_BF16
    for s in range(steps):
        inp = synth.decode_step_inputs(s, seed=99, B=B, H=H, dk=dk, dv=dv)
        if dtype == "f32":
            inp = {k: v.float() for k, v in inp.items()}
        d = to_dev(inp)
        o_raw = torch.empty(B, H, dv, device="cuda")
        y = gd.gdelta_decode_step(d["q"], d["k"], d["v"], d["b"], d["w"], d["z"], d["g"],
                                  d["log_alpha"], S, gamma_stat=gamma.cuda(), o_raw=o_raw)
        ref = oracle.decode_steps([inp], Sref, gamma_stat=gamma, heads=heads)
        Sref = ref["S"]
        assert err_stored(y.cpu().reshape(B * H, dv), ref["y"][0], dtype) <= tol
        assert err(o_raw.cpu().reshape(B * H, dv), ref["o_raw"][0]) <= tol
    assert err(S.cpu().reshape(B * H, dk, dv), Sref) <= tol


def test_decode_full_workload_sampled_heads():
    """Batch 64 x 16 heads, d 128: state from 2048 tokens of the 350M-layer
    distributions (oracle, sampled heads; other heads start at zero), then
    1024 consecutive steps on the GPU; the oracle follows the sampled heads."""
    import channel_gated_delta_b200 as gd
    D = synth.DECODE
    B, H, dk, dv = D["B"], D["H"], D["dk"], D["dv"]
    heads = [(0, 0), (5, 3), (17, 15), (40, 8), (63, 1), (63, 14)]
    gamma = synth.decode_gamma()
    S_init = torch.zeros(B, H, dk, dv)
    Sref = np.zeros((len(heads), dk, dv))
    by_b = {}
    for n, (b, h) in enumerate(heads):
        by_b.setdefault(b, []).append((n, h))
    for b, lst in by_b.items():
        tok = synth.decode_init_tokens(b)
        r = oracle.forward(tok, heads=[(0, h) for _, h in lst])      # S_0 = 0, gamma = 1
        for (n, h), S_h in zip(lst, r["S"]):
            Sref[n] = S_h
            S_init[b, h] = torch.from_numpy(S_h).float()
    Sref = S_init.double().numpy()[[b for b, _ in heads], [h for _, h in heads]]
    S = S_init.cuda()
    gam = gamma.cuda()
    worst_y = 0.0
    for s in range(D["steps"]):
        inp = synth.decode_step_inputs(s)
        d = to_dev(inp)
        y = gd.gdelta_decode_step(d["q"], d["k"], d["v"], d["b"], d["w"], d["z"], d["g"],
                                  d["log_alpha"], S, gamma_stat=gam)
        ref = oracle.decode_steps([inp], Sref, gamma_stat=gamma, heads=heads)
        Sref = ref["S"]
        yh = torch.stack([y[b, h] for b, h in heads]).cpu()
        worst_y = max(worst_y, err_stored(yh, ref["y"][0], "bf16"))
    torch.cuda.synchronize()
    assert worst_y <= TOL_BF16
    assert err(torch.stack([S.cpu()[b, h] for b, h in heads]), Sref) <= TOL_BF16


# --------------------------------------------------------------------------
# Tensor-core path (tcgen05, fp16 operands, fp32 accumulation)
# --------------------------------------------------------------------------

@pytest.mark.parametrize("T", [1, 5, 64, 65, 200, 64 * 7 + 9])
def test_tc_ragged_lengths(T):
    shape = synth.GdnShape(B=2, T=T, H=2, dk=128, dv=128, dtype="bf16", hot_channels=6, seed=40 + T)
    inp = synth.generate(shape)
    y, S, o = gpu_fwd(inp, path="tc")
    heads = oracle.all_heads(2, 2)
    _check(y, S, o, _ref(inp, heads), heads, TOL_BF16)


@pytest.mark.parametrize("u", [(-3.0, 0.0), (0.0, 2.0), (2.0, 3.5)])
def test_tc_fast_decay_shortens_chunks(u):
    """Decays fast enough that a 64-token chunk's log-decay span exceeds the
    fp16 operand budget: the kernel shortens chunks (down to one token)."""
    shape = synth.GdnShape(B=1, T=300, H=2, dk=128, dv=128, dtype="bf16", u_low=u[0], u_high=u[1], seed=7)
    inp = synth.generate(shape)
    y, S, o = gpu_fwd(inp, path="tc")
    heads = oracle.all_heads(1, 2)
    _check(y, S, o, _ref(inp, heads), heads, TOL_BF16)


def test_tc_mixed_fast_and_shortened_windows():
    """Windows whose decay span fits one 64-token chunk interleave with windows
    that must be shortened (two in a row, a single one, and the ragged tail):
    the chain switches between precomputed window tiles and its own shorter
    chunks, and a shortened window borrows the other window buffer as scratch."""
    shape = synth.GdnShape(B=2, T=64 * 7 + 17, H=2, dk=128, dv=128, dtype="bf16", hot_channels=6, seed=11)
    inp = synth.generate(shape)
    la = inp["log_alpha"].clone()
    for w in (1, 2, 4, 7):
        la[:, 64 * w: 64 * (w + 1)] *= 40.0
    inp["log_alpha"] = la
    y, S, o = gpu_fwd(inp, path="tc")
    heads = oracle.all_heads(2, 2)
    _check(y, S, o, _ref(inp, heads), heads, TOL_BF16)


def test_tc_state_in_and_in_place():
    import channel_gated_delta_b200 as gd
    shape = synth.GdnShape(B=2, T=150, H=3, dk=128, dv=128, dtype="bf16", seed=8)
    inp = synth.generate(shape)
    S0 = torch.randn(2, 3, 128, 128, generator=torch.Generator().manual_seed(3)) * 0.3
    d = to_dev(inp)
    S = S0.cuda()
    y, _ = gd.gdelta_fwd_chunked(d["q"], d["k"], d["v"], d["b"], d["w"], d["z"], d["g"], d["log_alpha"],
                                 gamma_stat=d["gamma_stat"], S_in=S, S_out=S, path="tc")
    torch.cuda.synchronize()
    assert gd.gdelta_get_last_device_error() == 0
    heads = oracle.all_heads(2, 3)
    ref = _ref(inp, heads, S0=S0.reshape(6, 128, 128))
    _check(y.cpu(), S.cpu(), None, ref, heads, TOL_BF16)


def test_tc_matches_simt_path():
    shape = synth.GdnShape(B=1, T=256, H=4, dk=128, dv=128, dtype="bf16", hot_channels=6, seed=9)
    inp = synth.generate(shape)
    y1, S1, o1 = gpu_fwd(inp, path="tc")
    y2, S2, o2 = gpu_fwd(inp, path="simt")
    assert err(o1, o2.double().numpy()) <= TOL_BF16
    assert err(S1, S2.double().numpy()) <= TOL_BF16


def test_tc_rejects_unsupported_shapes():
    import channel_gated_delta_b200 as gd
    shape = synth.GdnShape(B=1, T=64, H=1, dk=64, dv=64, dtype="bf16", seed=1)
    d = to_dev(synth.generate(shape))
    with pytest.raises(gd.GdeltaError):
        gd.gdelta_fwd_chunked(d["q"], d["k"], d["v"], d["b"], d["w"], d["z"], d["g"], d["log_alpha"], path="tc")
    assert gd.gdelta_fwd_selected_path(d["q"], d["k"], d["v"], d["b"], d["w"], d["z"], d["g"],
                                       d["log_alpha"]) == "simt"


# --------------------------------------------------------------------------
# Reduced gate forms: no z, one beta for b and w (KDA), and a per-token decay
# on top (Gated DeltaNet).  The kernels read the reduced tensors; the oracle
# gets the same values broadcast over the channels, with z = 0.
# --------------------------------------------------------------------------

FORMS = {
    "no_z": dict(drop_z=True, beta=False, decay_tok=False),
    "kda": dict(drop_z=False, beta=True, decay_tok=False),
    "gdn": dict(drop_z=True, beta=True, decay_tok=True),
}


def _reduce(inp, form):
    """(kernel inputs, oracle inputs) for one gate form.  beta is channel 0 of
    w (a sigmoid, as a write strength is); the per-token log-decay is channel 0
    of log_alpha."""
    f = FORMS[form]
    ker, ref = dict(inp), dict(inp)
    dk, dv = inp["k"].shape[-1], inp["v"].shape[-1]
    if f["drop_z"]:
        ker["z"] = None
        ref["z"] = torch.zeros_like(inp["z"])
    if f["beta"]:
        beta = inp["w"][..., 0].contiguous()
        ker["beta"], ker["b"], ker["w"] = beta, None, None
        ref["b"] = beta[..., None].expand(*beta.shape, dk).contiguous()
        ref["w"] = beta[..., None].expand(*beta.shape, dv).contiguous()
    if f["decay_tok"]:
        la = inp["log_alpha"][..., 0].contiguous()
        ker["log_alpha"] = la
        ref["log_alpha"] = la[..., None].expand(*la.shape, dk).contiguous()
    return ker, ref, f["decay_tok"]


def _fwd_reduced(ker, decay_tok, **kw):
    import channel_gated_delta_b200 as gd
    d = to_dev(ker)
    B, T, H, dk = d["q"].shape
    o_raw = torch.empty((B, T, H, d["v"].shape[-1]), dtype=torch.float32, device="cuda")
    y, S = gd.gdelta_fwd_chunked(d["q"], d["k"], d["v"], d.get("b"), d.get("w"), d.get("z"), d["g"],
                                 d["log_alpha"], gamma_stat=d["gamma_stat"], o_raw=o_raw,
                                 beta=d.get("beta"), decay_per_token=decay_tok, **kw)
    torch.cuda.synchronize()
    assert gd.gdelta_get_last_device_error() == 0
    return y.cpu(), S.cpu(), o_raw.cpu()


@pytest.mark.parametrize("form", sorted(FORMS))
@pytest.mark.parametrize("path", ["tc", "simt"])
def test_reduced_gate_forms_bf16(form, path):
    shape = synth.GdnShape(B=2, T=64 * 3 + 29, H=2, dk=128, dv=128, dtype="bf16", hot_channels=6,
                           seed=61)
    ker, ref_in, tok = _reduce(synth.generate(shape), form)
    y, S, o = _fwd_reduced(ker, tok, path=path)
    heads = oracle.all_heads(2, 2)
    _check(y, S, o, _ref(ref_in, heads), heads, TOL_BF16)


@pytest.mark.parametrize("form", sorted(FORMS))
def test_reduced_gate_forms_f32(form):
    shape = synth.GdnShape(B=1, T=101, H=2, dk=64, dv=128, dtype="f32", seed=62)
    ker, ref_in, tok = _reduce(synth.generate(shape), form)
    y, S, o = _fwd_reduced(ker, tok, path="simt", chunk=32)
    heads = oracle.all_heads(1, 2)
    _check(y, S, o, _ref(ref_in, heads), heads, TOL_F32)


def test_tc_per_token_decay_with_shortened_windows():
    """A scalar decay fast enough that some 64-token windows exceed the fp16
    span budget: the chain's own shortened chunks read the per-token decay
    and the single beta too."""
    shape = synth.GdnShape(B=1, T=64 * 5 + 3, H=2, dk=128, dv=128, dtype="bf16", seed=63)
    ker, ref_in, tok = _reduce(synth.generate(shape), "gdn")
    for side in (ker, ref_in):
        la = side["log_alpha"].clone()
        la[:, 64:128] *= 40.0
        la[:, 256:] *= 40.0
        side["log_alpha"] = la
    y, S, o = _fwd_reduced(ker, tok, path="tc")
    heads = oracle.all_heads(1, 2)
    _check(y, S, o, _ref(ref_in, heads), heads, TOL_BF16)


@pytest.mark.parametrize("form", sorted(FORMS))
def test_decode_reduced_gate_forms(form):
    import channel_gated_delta_b200 as gd
    B, H, dk, dv, steps = 3, 2, 128, 128, 4
    S0 = torch.randn(B, H, dk, dv, generator=torch.Generator().manual_seed(5)) * 0.3
    S = S0.cuda()
    heads = oracle.all_heads(B, H)
    Sref = S0.reshape(B * H, dk, dv).double().numpy()
    for s in range(steps):
        ker, ref_in, tok = _reduce(synth.decode_step_inputs(s, seed=71, B=B, H=H, dk=dk, dv=dv), form)
        d = to_dev(ker)
        y = gd.gdelta_decode_step(d["q"], d["k"], d["v"], d.get("b"), d.get("w"), d.get("z"), d["g"],
                                  d["log_alpha"], S, beta=d.get("beta"), decay_per_token=tok)
        ref = oracle.decode_steps([ref_in], Sref, heads=heads)
        Sref = ref["S"]
        assert err_stored(y.cpu().reshape(B * H, dv), ref["y"][0], "bf16") <= TOL_BF16
    assert err(S.cpu().reshape(B * H, dk, dv), Sref) <= TOL_BF16


# --------------------------------------------------------------------------
# Long streams: prefill in consecutive calls carrying the state, then decode
# (Muir review §4.3: one continuous token stream far beyond the training
# length, served with a fixed-size fp32 state).
# --------------------------------------------------------------------------

def test_long_stream_prefill_calls_then_decode():
    """131072 tokens of one sequence (B1, two heads) in 8 forward calls of
    16384 tokens on the tensor-core path, the state updated in place between
    calls, then 16 decode steps.  Every output of every call and the final
    state are compared with the oracle run over the same stream, so error
    that accumulated across 2048 windows of state carries would show."""
    import channel_gated_delta_b200 as gd
    seg, n_seg, H = 16384, 8, 2
    S = torch.zeros(1, H, 128, 128, device="cuda")
    heads = oracle.all_heads(1, H)
    Sref = np.zeros((H, 128, 128))
    gamma = None
    worst = 0.0
    for i in range(n_seg):
        shape = synth.GdnShape(B=1, T=seg, H=H, dk=128, dv=128, dtype="bf16", hot_channels=6, seed=200 + i)
        inp = synth.generate(shape)
        if gamma is None:
            gamma = inp["gamma_stat"]
        inp["gamma_stat"] = gamma                       # one layer: the same static profile throughout
        d = to_dev(inp)
        y, _ = gd.gdelta_fwd_chunked(d["q"], d["k"], d["v"], d["b"], d["w"], d["z"], d["g"], d["log_alpha"],
                                     gamma_stat=d["gamma_stat"], S_in=S, S_out=S, path="tc")
        torch.cuda.synchronize()
        assert gd.gdelta_get_last_device_error() == 0
        ref = _ref(inp, heads, S0=Sref)
        Sref = ref["S"]
        worst = max(worst, err_stored(sel_heads(y.cpu(), heads), ref["y"], "bf16"))
    assert worst <= TOL_BF16, worst
    assert err(S.cpu().reshape(H, 128, 128), Sref) <= TOL_BF16
    gam = gamma.cuda()
    for s in range(16):
        inp = synth.decode_step_inputs(s, seed=81, B=1, H=H, dk=128, dv=128)
        d = to_dev(inp)
        y = gd.gdelta_decode_step(d["q"], d["k"], d["v"], d["b"], d["w"], d["z"], d["g"],
                                  d["log_alpha"], S, gamma_stat=gam)
        ref = oracle.decode_steps([inp], Sref, gamma_stat=gamma, heads=heads)
        Sref = ref["S"]
        assert err_stored(y.cpu().reshape(H, 128), ref["y"][0], "bf16") <= TOL_BF16
    assert err(S.cpu().reshape(H, 128, 128), Sref) <= TOL_BF16


# --------------------------------------------------------------------------
# Sequence sharding: segment maps, their composition, and the forward from
# the composed state, with the segments run one after another on this GPU
# exactly as separate ranks would run them.
# --------------------------------------------------------------------------

@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 128), (128, 64), (64, 64)])
def test_state_affine_matches_float64(dk, dv):
    import channel_gated_delta_b200 as gd
    gen = torch.Generator().manual_seed(dk + dv)
    B, H = 2, 3
    A = torch.randn(B, H, dk, dk, generator=gen) / dk ** 0.5
    S = torch.randn(B, H, dk, dv, generator=gen)
    D = torch.randn(B, H, dk, dv, generator=gen)
    ref = (A.double() @ S.double() + D.double()).numpy()
    Ad, Sd, Dd = A.cuda(), S.cuda(), D.cuda()
    assert err(gd.gdelta_state_affine(Ad, S_in=Sd, D=Dd), ref) <= TOL_F32
    assert err(gd.gdelta_state_affine(Ad, S_in=Sd), (A.double() @ S.double()).numpy()) <= TOL_F32
    assert torch.equal(gd.gdelta_state_affine(Ad, D=Dd).cpu(), D)          # zero state: D itself
    gd.gdelta_state_affine(Ad, S_in=Sd, D=Dd, S_out=Dd)                     # in place on D
    torch.cuda.synchronize()
    assert err(Dd, ref) <= TOL_F32
    with pytest.raises(gd.GdeltaError):
        gd.gdelta_state_affine(Ad, S_in=Sd, S_out=Sd)                        # output over the input


@pytest.mark.parametrize("dtype,path,dk,dv", [("bf16", "tc", 128, 128), ("f32", "simt", 64, 128)])
def test_seqshard_segments_compose_to_the_whole_sequence(dtype, path, dk, dv):
    import channel_gated_delta_b200 as gd
    from channel_gated_delta_b200.seqshard import compose_affine, compose_range
    n_seg, H = 4, 2
    bounds = [0, 150, 301, 470, 637]                   # ragged: windows cross segment ends
    inp = synth.generate(synth.GdnShape(B=1, T=bounds[-1], H=H, dk=dk, dv=dv, dtype=dtype,
                                        hot_channels=6 if dtype == "bf16" else 0, seed=93))
    d = to_dev(inp)
    segs = [{k: (v[:, bounds[r]:bounds[r + 1]] if v.dim() == 4 else v) for k, v in d.items()}
            for r in range(n_seg)]
    maps = [gd.gdelta_segment_map(s["q"], s["k"], s["v"], s["b"], s["w"], s["z"], s["g"], s["log_alpha"],
                                  path=path) for s in segs]
    As, Ds = [m[0] for m in maps], [m[1] for m in maps]
    ys, finals = [], []
    for r, s in enumerate(segs):
        S0 = compose_range(As, Ds, 0, r, None, compose_affine)
        y, S_end = gd.gdelta_fwd_chunked(s["q"], s["k"], s["v"], s["b"], s["w"], s["z"], s["g"], s["log_alpha"],
                                         gamma_stat=d["gamma_stat"], S_in=S0, path=path)
        ys.append(y)
        finals.append(compose_range(As, Ds, r + 1, n_seg, S_end, compose_affine))
    torch.cuda.synchronize()
    assert gd.gdelta_get_last_device_error() == 0
    heads = oracle.all_heads(1, H)
    ref = _ref(inp, heads)
    tol = TOL_BF16 if dtype == "bf16" else TOL_F32
    assert err_stored(sel_heads(torch.cat(ys, 1).cpu(), heads), ref["y"], dtype) <= tol
    for S_fin in finals:                              # every rank ends with the sequence's final state
        assert err(S_fin.cpu().reshape(H, dk, dv), ref["S"]) <= tol


# --------------------------------------------------------------------------
# Raw q and k (qk_raw): the kernels apply SiLU and the per-head l2
# normalisation as they load them; the oracle applies its own preprocessing.
# --------------------------------------------------------------------------

def _raw_qk(inp, seed):
    """Pre-activation q and k: seeded normal draws in the token dtype."""
    gen = torch.Generator().manual_seed(seed)
    out = dict(inp)
    for key in ("q", "k"):
        out[key] = (torch.randn(inp[key].shape, generator=gen) * 1.5).to(inp[key].dtype)
    return out


@pytest.mark.parametrize("path", ["tc", "simt"])
def test_raw_qk_prologue_bf16(path):
    shape = synth.GdnShape(B=2, T=64 * 3 + 29, H=2, dk=128, dv=128, dtype="bf16", hot_channels=6, seed=101)
    inp = _raw_qk(synth.generate(shape), 5)
    y, S, o = gpu_fwd(inp, path=path, qk_raw=True)
    heads = oracle.all_heads(2, 2)
    _check(y, S, o, oracle.forward(inp, heads=heads, qk_raw=True), heads, TOL_BF16)


def test_raw_qk_prologue_f32():
    shape = synth.GdnShape(B=1, T=101, H=2, dk=64, dv=128, dtype="f32", seed=102)
    inp = _raw_qk(synth.generate(shape), 6)
    y, S, o = gpu_fwd(inp, path="simt", chunk=32, qk_raw=True)
    heads = oracle.all_heads(1, 2)
    _check(y, S, o, oracle.forward(inp, heads=heads, qk_raw=True), heads, TOL_F32)


def test_tc_raw_qk_with_shortened_windows_and_reduced_gates():
    """The chain's own shorter chunks preprocess q and k too; with the Gated
    DeltaNet gate form on top (every intra switch on)."""
    shape = synth.GdnShape(B=1, T=64 * 5 + 3, H=2, dk=128, dv=128, dtype="bf16", seed=103)
    ker, ref_in, tok = _reduce(_raw_qk(synth.generate(shape), 7), "gdn")
    for side in (ker, ref_in):
        la = side["log_alpha"].clone()
        la[:, 64:128] *= 40.0
        side["log_alpha"] = la
    y, S, o = _fwd_reduced(ker, tok, path="tc", qk_raw=True)
    heads = oracle.all_heads(1, 2)
    _check(y, S, o, oracle.forward(ref_in, heads=heads, qk_raw=True), heads, TOL_BF16)


def test_decode_raw_qk():
    import channel_gated_delta_b200 as gd
    B, H, dk, dv = 3, 2, 128, 128
    S0 = torch.randn(B, H, dk, dv, generator=torch.Generator().manual_seed(8)) * 0.3
    S = S0.cuda()
    heads = oracle.all_heads(B, H)
    Sref = S0.reshape(B * H, dk, dv).double().numpy()
    for s in range(4):
        inp = _raw_qk(synth.decode_step_inputs(s, seed=104, B=B, H=H, dk=dk, dv=dv), 20 + s)
        d = to_dev(inp)
        y = gd.gdelta_decode_step(d["q"], d["k"], d["v"], d["b"], d["w"], d["z"], d["g"], d["log_alpha"], S,
                                  qk_raw=True)
        ref = oracle.decode_steps([inp], Sref, heads=heads, qk_raw=True)
        Sref = ref["S"]
        assert err_stored(y.cpu().reshape(B * H, dv), ref["y"][0], "bf16") <= TOL_BF16
    assert err(S.cpu().reshape(B * H, dk, dv), Sref) <= TOL_BF16


def test_segment_map_with_raw_qk_composes():
    """The segment maps read raw q and k the same way as the forward."""
    import channel_gated_delta_b200 as gd
    from channel_gated_delta_b200.seqshard import compose_affine, compose_range
    bounds, H = [0, 131, 300], 2
    inp = _raw_qk(synth.generate(synth.GdnShape(B=1, T=300, H=H, dk=128, dv=128, dtype="bf16", seed=105)), 9)
    d = to_dev(inp)
    segs = [{k: (v[:, bounds[r]:bounds[r + 1]] if v.dim() == 4 else v) for k, v in d.items()} for r in range(2)]
    maps = [gd.gdelta_segment_map(s["q"], s["k"], s["v"], s["b"], s["w"], s["z"], s["g"], s["log_alpha"],
                                  qk_raw=True, path="tc") for s in segs]
    As, Ds = [m[0] for m in maps], [m[1] for m in maps]
    S0 = compose_range(As, Ds, 0, 1, None, compose_affine)
    s = segs[1]
    y, S_end = gd.gdelta_fwd_chunked(s["q"], s["k"], s["v"], s["b"], s["w"], s["z"], s["g"], s["log_alpha"],
                                     gamma_stat=d["gamma_stat"], S_in=S0, path="tc", qk_raw=True)
    torch.cuda.synchronize()
    heads = oracle.all_heads(1, H)
    ref = oracle.forward(inp, heads=heads, qk_raw=True)
    assert err_stored(sel_heads(y.cpu(), heads), ref["y"][:, 131:], "bf16") <= TOL_BF16
    assert err(S_end.cpu().reshape(H, 128, 128), ref["S"]) <= TOL_BF16


# --------------------------------------------------------------------------
# Backward pass against the float64 autograd oracle
# --------------------------------------------------------------------------

TOL_BWD = 1e-4      # max |diff| / rms per gradient: fp32 recurrence against float64


def _bwd_case(B, T, H, dtype, seed):
    inp = synth.generate(synth.GdnShape(B=B, T=T, H=H, dk=128, dv=128, dtype=dtype, hot_channels=6, seed=seed))
    gen = torch.Generator().manual_seed(seed)
    dy = torch.randn(B, T, H, 128, generator=gen)
    dS = torch.randn(B, H, 128, 128, generator=gen) * 0.1
    S0 = torch.randn(B, H, 128, 128, generator=gen) * 0.3
    return inp, dy, dS, S0


def bwd_errors(inp, dy, dS, S0):
    """Per-gradient max|diff|/rms of gdelta_bwd against the autograd oracle."""
    import channel_gated_delta_b200 as gd
    from oracle import backward as ob
    B, T, H, _ = inp["q"].shape
    d = to_dev(inp)
    g = gd.gdelta_bwd(d["q"], d["k"], d["v"], d["b"], d["w"], d["z"], d["g"], d["log_alpha"], dy.cuda(),
                      gamma_stat=d["gamma_stat"], S_in=S0.cuda(), grad_S_out=dS.cuda())
    torch.cuda.synchronize()
    assert gd.gdelta_get_last_device_error() == 0
    heads = oracle.all_heads(B, H)
    ref = ob.backward(inp, dy.numpy(), dS_out=dS.reshape(B * H, 128, 128).numpy(),
                      S0=S0.reshape(B * H, 128, 128).numpy(), heads=heads)
    out = {}
    if T > 0:
        for key in ("q", "k", "v", "b", "w", "z", "g", "log_alpha"):
            out[key] = err(sel_heads(g[key].cpu(), heads), ref["d" + key])
        out["gamma_stat"] = err(g["gamma_stat"].cpu(), ref["dgamma_stat"])
    out["S_in"] = err(g["S_in"].cpu().reshape(B * H, 128, 128), ref["dS_in"])
    return out


@pytest.mark.parametrize("B,T,H,dtype", [(2, 77, 2, "f32"), (1, 64, 3, "bf16"), (1, 5, 1, "f32")])
def test_backward_matches_autograd_oracle(B, T, H, dtype):
    """Ragged against the 32-token checkpoints (77), exactly two chunks (64),
    shorter than one chunk (5); fp32 and bf16 token storage."""
    e = bwd_errors(*_bwd_case(B, T, H, dtype, 200 + T))
    assert max(e.values()) <= TOL_BWD, e


@pytest.mark.parametrize("T", [33, 34, 35])
def test_backward_short_last_chunk(T):
    """A last checkpoint chunk of 1, 2 or 3 tokens: its states stay in the two
    shared-memory tiles (1 and 2), one is bulk-loaded back from the checkpoint
    (2), the first state goes through the chunk buffer (3)."""
    e = bwd_errors(*_bwd_case(1, T, 2, "f32", 300 + T))
    assert max(e.values()) <= TOL_BWD, e


def test_backward_long_sequence_matches_autograd_oracle():
    """1024 tokens (32 checkpoint chunks) on every head of B2 H4 (the last
    batch row's last head included), bf16 tokens, a non-zero initial state and
    state gradient: gradient errors do not grow along the sequence."""
    e = bwd_errors(*_bwd_case(2, 1024, 4, "bf16", 1024))
    assert max(e.values()) <= TOL_BWD, e


def test_backward_full_size_sampled_heads():
    """The benchmark workload (B4 T4096 H16 bf16, the call `bench.py` times):
    every token gradient of the first and the last head against the float64
    autograd oracle (about 18 s of CPU a head); the other heads run in the
    same launch."""
    import channel_gated_delta_b200 as gd
    from oracle import backward as ob
    shape = synth.CONFIGS["muir1b3_bf16"]
    inp = synth.generate(shape)
    d = to_dev(inp)
    dy = torch.randn(shape.B, shape.T, shape.H, 128, generator=torch.Generator().manual_seed(13))
    g = gd.gdelta_bwd(d["q"], d["k"], d["v"], d["b"], d["w"], d["z"], d["g"], d["log_alpha"], dy.cuda(),
                      gamma_stat=d["gamma_stat"])
    torch.cuda.synchronize()
    assert gd.gdelta_get_last_device_error() == 0
    heads = [(0, 0), (shape.B - 1, shape.H - 1)]
    ref = ob.backward(inp, dy.numpy(), heads=heads)
    e = {key: err(sel_heads(g[key].cpu(), heads), ref["d" + key])
         for key in ("q", "k", "v", "b", "w", "z", "g", "log_alpha")}
    assert max(e.values()) <= TOL_BWD, e


def test_backward_without_tokens_passes_the_state_gradient_through():
    import channel_gated_delta_b200 as gd
    B, H = 1, 2
    inp, dy, dS, S0 = _bwd_case(B, 3, H, "f32", 9)
    d = {k: (v[:, :0] if v.dim() == 4 else v) for k, v in to_dev(inp).items()}
    g = gd.gdelta_bwd(d["q"], d["k"], d["v"], d["b"], d["w"], d["z"], d["g"], d["log_alpha"],
                      dy[:, :0].cuda(), S_in=S0.cuda(), grad_S_out=dS.cuda())
    torch.cuda.synchronize()
    assert torch.equal(g["S_in"].cpu(), dS)
