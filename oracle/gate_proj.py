"""Five-gate low-rank projection -- float64 oracle.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module.  It shares no code
with the CUDA product path.

Muir review §2.3 ("五门融合投影与参数再分配"): the decay f, erase b, output g,
write w and query-gain q gates share one down-projection of the layer input
whose width is the sum of their ranks, (r_f, r_b, r_g, r_w, r_q) = (64, 64,
128, 128, 128), 512 in all; each gate then has its own up-projection back to
the model width and a per-channel bias, which give its logits.  The
projection has 2 d R_tot parameters (d x R_tot down, R_tot x d up).

Readings where the page is silent (each stated in the design notes):

* Layout: x is [N, d] (tokens by model width, the heads' channels
  contiguous, h-major, as the mixer's [B, T, H, 128] inputs are), w_down is
  [d, R_tot] with its columns grouped f | b | g | w | q, w_up is [R_tot, d]
  with its rows grouped the same way, bias is [5, d] in the same gate order.
* Activations: the review fixes the gates' ranges (§2.1: alpha in (0, 1),
  b in (0, 2), w in (0, 1); g is a sigmoid gate; the query gain enters the
  readout as 2 sigmoid(z)).  The plainest activations with those ranges are
  alpha = sigmoid(f) (kept as log alpha = log sigmoid(f), in fp32 as the
  review's setup keeps the log-decay), b = 2 sigmoid(.), g = sigmoid(.),
  w = sigmoid(.), and z = the q logit itself (the mixer applies 2 sigmoid).
"""
from __future__ import annotations

from typing import Dict, Sequence

import numpy as np

GATES = ("f", "b", "g", "w", "q")
RANKS = (64, 64, 128, 128, 128)


def _f64(x) -> np.ndarray:
    try:
        import torch
        if isinstance(x, torch.Tensor):
            return x.detach().to("cpu", torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(x, dtype=np.float64)


def logits(x, w_down, w_up, bias, ranks: Sequence[int] = RANKS) -> Dict[str, np.ndarray]:
    """The five gates' logits: codes c = x w_down, then for gate i the slice of
    c (and the rows of w_up) that belong to it, up-projected, plus its bias."""
    x, w_down, w_up, bias = _f64(x), _f64(w_down), _f64(w_up), _f64(bias)
    codes = x @ w_down
    out = {}
    off = 0
    for i, (name, r) in enumerate(zip(GATES, ranks)):
        out[name] = codes[:, off:off + r] @ w_up[off:off + r, :] + bias[i]
        off += r
    assert off == w_down.shape[1] == w_up.shape[0]
    return out


def activate(lg: Dict[str, np.ndarray]) -> Dict[str, np.ndarray]:
    """Gate values in the form the mixer takes them: log_alpha = log sigmoid(f)
    (computed as -log(1 + e^-f) without overflow), b = 2 sigmoid, g and w =
    sigmoid, z = the q logit."""
    def sig(v):
        return 0.5 * (1.0 + np.tanh(0.5 * v))
    return {
        "log_alpha": -np.logaddexp(0.0, -lg["f"]),
        "b": 2.0 * sig(lg["b"]),
        "g": sig(lg["g"]),
        "w": sig(lg["w"]),
        "z": lg["q"].copy(),
    }


def project(x, w_down, w_up, bias, ranks: Sequence[int] = RANKS) -> Dict[str, np.ndarray]:
    """Activated gates [N, d] (float64): log_alpha, b, g, w, z."""
    return activate(logits(x, w_down, w_up, bias, ranks))


def parameter_count(d: int, ranks: Sequence[int] = RANKS) -> int:
    """Weights of the projection: d x R_tot down plus R_tot x d up."""
    return 2 * d * int(sum(ranks))
