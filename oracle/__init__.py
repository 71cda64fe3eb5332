"""Oracle for the channel-wise gated delta-rule token mixer.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  It shares no code
with the CUDA product path, and the product path never calls it.

* ``forward``  -- the float64 token-by-token recurrence (C, ``gdn2_oracle.c``),
  threaded over heads and value-column blocks.  It is the definition the GPU
  path is compared against.
* ``chunked``  -- a float64 numpy restatement of the chunked algorithm the
  Muir review describes in §2.4 (boundary-pivoted decay products, divide-and-
  conquer inverse of the unit lower-triangular chunk matrix with Neumann-series
  leaves, inter-chunk state scan).  It is pinned against ``forward``.

Every input is first upcast to float64 from whatever storage dtype it has
(bf16 or fp32), so both sides read the same quantised values.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Dict, Iterable, List, Optional, Sequence, Tuple

import numpy as np

from . import chunked  # noqa: F401  (re-exported)

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdn2_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle_gdn2.so")
_lib = None

TOKEN_KEYS = ("q", "k", "v", "b", "w", "z", "g", "log_alpha")


def build(force: bool = False) -> str:
    """Compile the C oracle (plain -O2, no fast-math) next to its source."""
    stale = (not os.path.exists(_LIB_PATH)
             or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC))
    if force or stale:
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        dp = ctypes.POINTER(ctypes.c_double)
        lib.oracle_gdn2_forward.restype = ctypes.c_int
        lib.oracle_gdn2_forward.argtypes = ([ctypes.c_int] * 4 + [dp] * 9 + [dp, dp, dp]
                                            + [ctypes.c_double, ctypes.c_int])
        lib.oracle_num_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def _f64(x) -> np.ndarray:
    """Any torch tensor / numpy array -> float64 numpy (exact upcast)."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            return x.detach().to("cpu", torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(x, dtype=np.float64)


def _gather(x, heads: Sequence[Tuple[int, int]]) -> np.ndarray:
    """[B,T,H,d] -> contiguous float64 [n_heads, T, d] for the listed (b,h)."""
    return np.ascontiguousarray(np.stack([_f64(x[b_, :, h_, :]) for (b_, h_) in heads]))


def _ptr(a: np.ndarray):
    assert a.dtype == np.float64 and a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def all_heads(B: int, H: int) -> List[Tuple[int, int]]:
    return [(b_, h_) for b_ in range(B) for h_ in range(H)]


def preprocess_qk(x) -> np.ndarray:
    """Key and query preprocessing (Muir review §2.1: SiLU, then l2
    normalisation per head; values are left alone): x sigmoid(x), divided by
    its l2 norm over the last axis (the head's channels), the norm floored at
    1e-12 so that a zero row stays zero.  [..., d] in, float64 out."""
    x = _f64(x)
    s = x / (1.0 + np.exp(-x))
    n = np.sqrt(np.sum(s * s, axis=-1, keepdims=True))
    return s / np.maximum(n, 1e-12)


def _with_raw_qk(inputs: Dict) -> Dict:
    out = dict(inputs)
    out["q"] = preprocess_qk(inputs["q"])
    out["k"] = preprocess_qk(inputs["k"])
    return out


def forward(inputs: Dict, heads: Optional[Iterable[Tuple[int, int]]] = None,
            S0=None, eps: float = 1e-6, n_threads: int = 0, qk_raw: bool = False) -> Dict[str, np.ndarray]:
    """Token-by-token float64 recurrence over the listed heads.

    inputs: q,k,v,b,w,z,g,log_alpha as [B,T,H,d] (torch or numpy, any float
    dtype) and optionally gamma_stat [H,dk] (absent or None = ones).
    heads:  list of (b, h); None = all heads in (b, h) order.
    S0:     None (zeros) or [n_heads, dk, dv].
    qk_raw: q and k are given before ``preprocess_qk``, which is applied first.
    Returns float64 arrays y, o_raw [n_heads, T, dv], S [n_heads, dk, dv] and
    the thread count used under "threads".
    """
    if qk_raw:
        inputs = _with_raw_qk(inputs)
    B, T, H, dk = tuple(inputs["q"].shape)
    dv = int(inputs["v"].shape[-1])
    heads = all_heads(B, H) if heads is None else list(heads)
    n = len(heads)
    arrs = {key: _gather(inputs[key], heads) for key in TOKEN_KEYS}
    gs = inputs.get("gamma_stat")
    gsf = np.ones((H, dk)) if gs is None else _f64(gs)
    gamma = np.ascontiguousarray(np.stack([gsf[h_] for (_, h_) in heads]))
    S = np.zeros((n, dk, dv)) if S0 is None else np.array(_f64(S0), dtype=np.float64, order="C", copy=True)
    assert S.shape == (n, dk, dv)
    o_raw = np.zeros((n, T, dv))
    y = np.zeros((n, T, dv))
    lib = _load()
    used = lib.oracle_gdn2_forward(n, T, dk, dv, *[_ptr(arrs[key]) for key in TOKEN_KEYS],
                                   _ptr(gamma), _ptr(S), _ptr(o_raw), _ptr(y), float(eps),
                                   int(n_threads))
    if used < 0:
        raise ValueError("oracle_gdn2_forward rejected its arguments")
    return {"y": y, "o_raw": o_raw, "S": S, "threads": used}


def forward_full(inputs: Dict, S0=None, eps: float = 1e-6, n_threads: int = 0) -> Dict[str, np.ndarray]:
    """``forward`` over every head, reshaped to [B,T,H,dv] / [B,H,dk,dv]."""
    B, T, H, dk = tuple(inputs["q"].shape)
    dv = int(inputs["v"].shape[-1])
    S0h = None if S0 is None else _f64(S0).reshape(B * H, dk, dv)
    r = forward(inputs, None, S0h, eps, n_threads)
    return {
        "y": r["y"].reshape(B, H, T, dv).transpose(0, 2, 1, 3),
        "o_raw": r["o_raw"].reshape(B, H, T, dv).transpose(0, 2, 1, 3),
        "S": r["S"].reshape(B, H, dk, dv),
        "threads": r["threads"],
    }


def decode_steps(step_inputs: Sequence[Dict], S0, gamma_stat=None,
                 heads: Optional[Sequence[Tuple[int, int]]] = None, eps: float = 1e-6,
                 n_threads: int = 0, qk_raw: bool = False) -> Dict[str, np.ndarray]:
    """Consecutive single-token updates.

    step_inputs: one dict per step with [B,H,d] tensors; S0: [n_heads,dk,dv]
    for the listed heads (default all, (b,h) order).  Returns the last step's
    y/o_raw [n_heads, dv], every step's y stacked [steps, n_heads, dv] and the
    final S.
    """
    S = S0
    ys, os_ = [], []
    for inp in step_inputs:
        tok = {key: inp[key][:, None] for key in TOKEN_KEYS}
        tok["gamma_stat"] = gamma_stat
        r = forward(tok, heads, S, eps, n_threads, qk_raw=qk_raw)
        S = r["S"]
        ys.append(r["y"][:, 0])
        os_.append(r["o_raw"][:, 0])
    return {"y": np.stack(ys), "o_raw": np.stack(os_), "S": S}
