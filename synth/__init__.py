"""Seeded synthetic inputs for the channel-wise gated delta-rule token mixer.

This module is shared by the oracle-side tests and by the GPU-side tests and
bench.  It holds only random-number draws and the input distributions; none of
the mixer's arithmetic lives here.

Distributions (all drawn in float64 from ``numpy.random.PCG64``, then quantised
once; the oracle and the GPU read exactly the quantised values):

* q, k  = SiLU(N(0,1)) then l2-normalised over d_k, per head and token
  ("Muir review" §2.1: keys and queries pass SiLU then l2 normalisation,
  values are not normalised);
* v     ~ N(0,1);
* log_alpha = -exp(u), u ~ U(u_low, u_high), one value per key channel
  (so alpha = exp(-exp(u)) is in (0,1)); kept in fp32;
* b     = 2*sigmoid(N(0,1)) in (0,2)^{d_k}   (erase gate);
* w     = sigmoid(N(0,1))   in (0,1)^{d_v}   (write gate);
* z     ~ N(0,1) over d_k                      (raw dynamic readout logit);
* g     = sigmoid(N(0,1))   over d_v           (output gate);
* gamma_stat = exp(0.1*N(0,1)), shape [H, d_k], fp32 (static readout profile).

Draw order: q, k, v, u, b, w, z, g, gamma_stat, then (only when requested) the
per-head hot key channels.  With ``hot_channels > 0`` a fixed random set of
channels per head is rescaled, before l2 normalisation, so that it holds
exactly ``hot_energy`` of each key's squared norm (the low effective key
participation the Muir review reports in §2.2: about 6 of 128 channels).

Layout: token tensors are ``[B, T, H, d]`` with d innermost.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, Optional

import numpy as np
import torch

__all__ = [
    "GdnShape",
    "CONFIGS",
    "generate",
    "generate_config",
    "decode_init_tokens",
    "decode_step_inputs",
    "decode_gamma",
    "quantise",
    "GATE_RANKS",
    "gate_proj_inputs",
]

TOKEN_KEYS = ("q", "k", "v", "b", "w", "z", "g")


@dataclasses.dataclass(frozen=True)
class GdnShape:
    B: int
    T: int
    H: int
    dk: int
    dv: int
    chunk: int = 64
    dtype: str = "bf16"          # dtype of q,k,v,b,w,z,g,y ("bf16" or "f32")
    u_low: float = -7.0
    u_high: float = -2.0
    hot_channels: int = 0
    hot_energy: float = 0.8
    seed: int = 0


# The five workloads.  Names say what they are; sizes follow the Muir review
# (d_k = d_v = 128, T = 4096 training length, H = 16 for the 1.34B model whose
# 24 layers hold 25 MB of fp32 state) and the ETH study's 32768-token timing.
CONFIGS: Dict[str, GdnShape] = {
    "tiny_f32": GdnShape(B=1, T=256, H=2, dk=64, dv=64, chunk=64, dtype="f32",
                         u_low=-5.0, u_high=-1.0, seed=0),
    "layer350m_bf16": GdnShape(B=8, T=4096, H=8, dk=128, dv=128, chunk=64,
                               dtype="bf16", seed=1),
    "muir1b3_bf16": GdnShape(B=4, T=4096, H=16, dk=128, dv=128, chunk=64,
                             dtype="bf16", hot_channels=6, seed=2),
    "long32k_bf16": GdnShape(B=1, T=32768, H=16, dk=128, dv=128, chunk=64,
                             dtype="bf16", hot_channels=6, seed=3),
}

# Decode workload: batch 64, H 16, d 128; state built from 2048 tokens of the
# 350M-layer distributions, then 1024 single-token steps.
DECODE = dict(B=64, H=16, dk=128, dv=128, init_tokens=2048, steps=1024, seed=4,
              u_low=-7.0, u_high=-2.0)


def _silu(x: np.ndarray) -> np.ndarray:
    return x / (1.0 + np.exp(-x))


def _sigmoid(x: np.ndarray) -> np.ndarray:
    return 1.0 / (1.0 + np.exp(-x))


def _l2n(x: np.ndarray) -> np.ndarray:
    n = np.sqrt(np.sum(x * x, axis=-1, keepdims=True))
    return x / np.maximum(n, 1e-300)


def quantise(x: np.ndarray, dtype: str) -> torch.Tensor:
    """float64 -> the storage dtype (round to nearest even)."""
    t = torch.from_numpy(np.ascontiguousarray(x))
    if dtype == "bf16":
        return t.to(torch.bfloat16)
    if dtype == "f32":
        return t.to(torch.float32)
    raise ValueError(dtype)


def _concentrate(k: np.ndarray, hot: np.ndarray, energy: float) -> np.ndarray:
    """Rescale so channels ``hot[h]`` hold ``energy`` of each row's squared norm.

    k: [B,T,H,dk] (non-negative-ish SiLU outputs); hot: [H, n_hot] indices.
    The result has unit norm up to rounding.
    """
    B, T, H, dk = k.shape
    mask = np.zeros((H, dk), dtype=bool)
    for h in range(H):
        mask[h, hot[h]] = True
    m = mask[None, None, :, :]
    e_hot = np.sum(np.where(m, k * k, 0.0), axis=-1, keepdims=True)
    e_cold = np.sum(np.where(m, 0.0, k * k), axis=-1, keepdims=True)
    s_hot = np.sqrt(energy / np.maximum(e_hot, 1e-300))
    s_cold = np.sqrt((1.0 - energy) / np.maximum(e_cold, 1e-300))
    return np.where(m, k * s_hot, k * s_cold)


def _draw_tokens(rng: np.random.Generator, B: int, T: int, H: int, dk: int,
                 dv: int, u_low: float, u_high: float, hot: Optional[np.ndarray],
                 hot_energy: float):
    q = _l2n(_silu(rng.standard_normal((B, T, H, dk))))
    k = _silu(rng.standard_normal((B, T, H, dk)))
    if hot is not None:
        k = _concentrate(k, hot, hot_energy)
    k = _l2n(k)
    v = rng.standard_normal((B, T, H, dv))
    u = rng.uniform(u_low, u_high, (B, T, H, dk))
    log_alpha = -np.exp(u)
    b = 2.0 * _sigmoid(rng.standard_normal((B, T, H, dk)))
    w = _sigmoid(rng.standard_normal((B, T, H, dv)))
    z = rng.standard_normal((B, T, H, dk))
    g = _sigmoid(rng.standard_normal((B, T, H, dv)))
    return dict(q=q, k=k, v=v, log_alpha=log_alpha, b=b, w=w, z=z, g=g)


def _pack(raw: dict, dtype: str, gamma: np.ndarray) -> Dict[str, torch.Tensor]:
    out = {key: quantise(raw[key], dtype) for key in TOKEN_KEYS}
    out["log_alpha"] = torch.from_numpy(raw["log_alpha"]).to(torch.float32)
    out["gamma_stat"] = torch.from_numpy(gamma).to(torch.float32)
    return out


def generate(shape: GdnShape, seed: Optional[int] = None) -> Dict[str, torch.Tensor]:
    """All inputs of one chunked-forward workload, as CPU tensors.

    Returns q,k,v,b,w,z,g in ``shape.dtype`` ([B,T,H,d]), log_alpha fp32
    [B,T,H,dk] and gamma_stat fp32 [H,dk].  The initial state is zero.
    """
    seed = shape.seed if seed is None else seed
    rng = np.random.Generator(np.random.PCG64(seed))
    B, T, H, dk, dv = shape.B, shape.T, shape.H, shape.dk, shape.dv
    # Hot channels are drawn from a separate stream so that the main draw order
    # (q, k, v, u, b, w, z, g, gamma) is the same with and without them.
    hot = None
    if shape.hot_channels > 0:
        hrng = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, 7])))
        hot = np.stack([hrng.choice(dk, size=shape.hot_channels, replace=False)
                        for _ in range(H)])
    raw = _draw_tokens(rng, B, T, H, dk, dv, shape.u_low, shape.u_high, hot,
                       shape.hot_energy)
    gamma = np.exp(0.1 * rng.standard_normal((H, dk)))
    return _pack(raw, shape.dtype, gamma)


def generate_config(name: str) -> Dict[str, torch.Tensor]:
    return generate(CONFIGS[name])


def decode_gamma(seed: int = DECODE["seed"], H: int = DECODE["H"],
                 dk: int = DECODE["dk"]) -> torch.Tensor:
    rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, 2])))
    return torch.from_numpy(np.exp(0.1 * rng.standard_normal((H, dk)))).to(torch.float32)


def decode_init_tokens(b_index: int, seed: int = DECODE["seed"], T: int = DECODE["init_tokens"],
                       H: int = DECODE["H"], dk: int = DECODE["dk"],
                       dv: int = DECODE["dv"]) -> Dict[str, torch.Tensor]:
    """Tokens that build batch row ``b_index``'s initial decode state: [1,T,H,d]."""
    rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, 0, b_index])))
    raw = _draw_tokens(rng, 1, T, H, dk, dv, DECODE["u_low"], DECODE["u_high"], None, 0.8)
    out = _pack(raw, "bf16", np.ones((H, dk)))
    del out["gamma_stat"]
    return out


def decode_step_inputs(step: int, seed: int = DECODE["seed"], B: int = DECODE["B"],
                       H: int = DECODE["H"], dk: int = DECODE["dk"],
                       dv: int = DECODE["dv"]) -> Dict[str, torch.Tensor]:
    """Fresh single-token inputs for decode step ``step``: [B,H,d] each."""
    rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, 1, step])))
    raw = _draw_tokens(rng, B, 1, H, dk, dv, DECODE["u_low"], DECODE["u_high"], None, 0.8)
    out = _pack(raw, "bf16", np.ones((H, dk)))
    del out["gamma_stat"]
    return {key: val[:, 0] for key, val in out.items()}


# Ranks of the five-gate projection in gate order f, b, g, w, q (the Muir
# review's main model: 64, 64, 128, 128, 128; 512 in all).
GATE_RANKS = (64, 64, 128, 128, 128)


def gate_proj_inputs(N: int, d: int, ranks=GATE_RANKS, seed: int = 0) -> Dict[str, torch.Tensor]:
    """Synthetic layer input and projection weights (no trained weights exist
    here): x [N, d] ~ N(0, 1); w_down [d, R] ~ N(0, 1/d) so the codes have unit
    variance; w_up [R, d] with each gate's rows ~ N(0, 1/r_gate) so every
    logit has unit variance before its bias; all three in bf16.  Biases [5, d]
    fp32: the decay gate's ~ U(2, 7), the decay logits of the workloads'
    log-decays -exp(u), u ~ U(-7, -2); the other gates' 0."""
    R = int(sum(ranks))
    rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, 7])))
    x = rng.standard_normal((N, d))
    w_down = rng.standard_normal((d, R)) / np.sqrt(d)
    w_up = np.concatenate([rng.standard_normal((r, d)) / np.sqrt(r) for r in ranks])
    bias = np.zeros((len(ranks), d))
    bias[0] = rng.uniform(2.0, 7.0, d)
    return {"x": quantise(x, "bf16"), "w_down": quantise(w_down, "bf16"), "w_up": quantise(w_up, "bf16"),
            "bias": torch.from_numpy(bias).to(torch.float32)}
