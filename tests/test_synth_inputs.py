"""The seeded input generators produce the stated distributions and layouts."""
import numpy as np
import torch

import synth


def test_tiny_config_shapes_dtypes_and_determinism():
    a = synth.generate_config("tiny_f32")
    b = synth.generate_config("tiny_f32")
    for key in ("q", "k", "v", "b", "w", "z", "g", "log_alpha"):
        assert torch.equal(a[key], b[key])
    assert a["q"].shape == (1, 256, 2, 64) and a["q"].dtype == torch.float32
    assert a["gamma_stat"].shape == (2, 64)
    qn = a["q"].double().norm(dim=-1)
    assert torch.allclose(qn, torch.ones_like(qn), atol=1e-6)
    la = a["log_alpha"].double()
    assert float(la.max()) < 0 and float(la.min()) > -np.exp(-1) - 1e-6
    assert float(a["b"].min()) > 0 and float(a["b"].max()) < 2
    assert float(a["w"].min()) > 0 and float(a["w"].max()) < 1


def test_hot_key_channels_hold_stated_energy():
    shape = synth.GdnShape(B=2, T=64, H=3, dk=128, dv=128, dtype="f32", hot_channels=6, seed=5)
    d = synth.generate(shape)
    k = d["k"].double()
    e = k * k                                           # [B,T,H,dk]
    for h in range(3):
        # the hot set is fixed per head: the 6 channels with the largest mean energy
        hot = torch.topk(e[:, :, h].mean((0, 1)), 6).indices
        share = e[:, :, h][..., hot].sum(-1)
        assert torch.allclose(share, torch.full_like(share, 0.8), atol=1e-5)


def test_bf16_rounding_is_storage_only():
    shape = synth.GdnShape(B=1, T=8, H=1, dk=16, dv=16, dtype="bf16", seed=1)
    d = synth.generate(shape)
    assert d["q"].dtype == torch.bfloat16 and d["log_alpha"].dtype == torch.float32


def test_decode_inputs_are_seeded_per_step():
    a = synth.decode_step_inputs(3, B=2, H=2, dk=8, dv=8)
    b = synth.decode_step_inputs(3, B=2, H=2, dk=8, dv=8)
    c = synth.decode_step_inputs(4, B=2, H=2, dk=8, dv=8)
    assert torch.equal(a["k"], b["k"]) and not torch.equal(a["k"], c["k"])
    assert a["k"].shape == (2, 2, 8)
