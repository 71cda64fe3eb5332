"""Gradients of the token mixer: float64 PyTorch autograd over the plain
token-by-token recurrence.

TEST INFRASTRUCTURE, like the rest of ``oracle``: only the tests may use it.

``forward_torch`` restates, with torch ops so that autograd can differentiate
it, the same per-token definition the C recurrence computes (Muir review
§2.1: S_hat = Diag(alpha) S; S = S_hat - (b*k)^T (k S_hat) + k^T (w*v);
o = (q * gamma * 2 sigmoid(z)) S; y = g * o / sqrt(mean(o^2) + eps)).  A pin
ties its outputs to the C oracle's and central finite differences pin the
gradients, so neither rests on this file alone.  ``backward`` returns the
gradients of L = sum(dy * y) + sum(dS_out * S_T) with respect to every input,
the initial state and the static readout profile.
"""
from __future__ import annotations

from typing import Dict, Optional, Sequence, Tuple

import numpy as np
import torch

TOKEN_KEYS = ("q", "k", "v", "b", "w", "z", "g", "log_alpha")


def forward_torch(q, k, v, b, w, z, g, log_alpha, gamma, S0, eps: float):
    """q, k, z, b, log_alpha [n, T, dk]; v, w, g [n, T, dv]; gamma [n, dk];
    S0 [n, dk, dv] (all float64).  Returns y [n, T, dv] and S_T."""
    S = S0
    ys = []
    for t in range(q.shape[1]):
        alpha = torch.exp(log_alpha[:, t])
        S_hat = alpha[:, :, None] * S
        kt = k[:, t]
        r = torch.einsum("ni,nij->nj", kt, S_hat)
        kh = b[:, t] * kt
        vh = w[:, t] * v[:, t]
        S = S_hat - kh[:, :, None] * r[:, None, :] + kt[:, :, None] * vh[:, None, :]
        qt = q[:, t] * gamma * 2.0 * torch.sigmoid(z[:, t])
        o = torch.einsum("ni,nij->nj", qt, S)
        ys.append(g[:, t] * o / torch.sqrt((o * o).mean(-1, keepdim=True) + eps))
    if ys:
        return torch.stack(ys, 1), S
    return torch.zeros(q.shape[0], 0, v.shape[-1], dtype=q.dtype), S


def _heads_tensor(x, heads) -> torch.Tensor:
    """[B, T, H, d] (torch or numpy, any float dtype) -> float64 [n, T, d]."""
    x = torch.as_tensor(np.asarray(x.detach().cpu().double() if isinstance(x, torch.Tensor) else x,
                                   dtype=np.float64))
    return torch.stack([x[b_, :, h_, :] for (b_, h_) in heads]).contiguous()


def backward(inputs: Dict, dy, dS_out=None, S0=None, heads: Optional[Sequence[Tuple[int, int]]] = None,
             eps: float = 1e-6) -> Dict[str, np.ndarray]:
    """Gradients of sum(dy * y) + sum(dS_out * S_T).

    inputs: q, k, v, b, w, z, g, log_alpha [B, T, H, d] and optionally
    gamma_stat [H, dk]; dy [B, T, H, dv]; dS_out, S0 [n_heads, dk, dv] or None
    (zero).  heads: (b, h) pairs, default all.  Returns float64 arrays: the
    token gradients [n_heads, T, d] under the input names prefixed with "d",
    dgamma_stat [H, dk] (summed over the listed heads) and dS_in
    [n_heads, dk, dv]; also y and S_T.
    """
    B, T, H, dk = tuple(inputs["q"].shape)
    dv = int(inputs["v"].shape[-1])
    heads = [(b_, h_) for b_ in range(B) for h_ in range(H)] if heads is None else list(heads)
    n = len(heads)
    leaves = {key: _heads_tensor(inputs[key], heads).requires_grad_(True) for key in TOKEN_KEYS}
    gs = inputs.get("gamma_stat")
    gamma_all = (torch.ones(H, dk, dtype=torch.float64) if gs is None
                 else torch.as_tensor(np.asarray(gs, dtype=np.float64)).clone())
    gamma_all.requires_grad_(True)
    gamma = torch.stack([gamma_all[h_] for (_, h_) in heads])
    S_init = (torch.zeros(n, dk, dv, dtype=torch.float64) if S0 is None
              else torch.as_tensor(np.asarray(S0, dtype=np.float64)).clone())
    S_init.requires_grad_(True)
    y, S_T = forward_torch(*(leaves[key] for key in TOKEN_KEYS), gamma, S_init, eps)
    loss = (y * _heads_tensor(dy, heads)).sum()
    if dS_out is not None:
        loss = loss + (S_T * torch.as_tensor(np.asarray(dS_out, dtype=np.float64))).sum()
    wrt = [leaves[key] for key in TOKEN_KEYS] + [gamma_all, S_init]
    grads = torch.autograd.grad(loss, wrt, allow_unused=True)
    out = {}
    for key, gr, leaf in zip(list(TOKEN_KEYS) + ["gamma_stat", "S_in"], grads, wrt):
        out["d" + key] = (torch.zeros_like(leaf) if gr is None else gr).detach().numpy()
    out["y"] = y.detach().numpy()
    out["S"] = S_T.detach().numpy()
    return out
