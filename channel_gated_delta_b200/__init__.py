"""B200 (sm_100a) channel-wise gated delta-rule token mixer.

Thin Python binding over the C ABI in ``include/gdelta.h`` (library
``libgdelta.so`` built in-tree by ``channel_gated_delta_b200.build``).  The
functions carry the C names and do argument marshalling only; PyTorch supplies
device memory and streams.  Every step of the mixer runs in the library's CUDA
kernels and a missing library raises -- there is no CPU fallback.

The operation (Muir review §2.1, GDN-2 update with the Muir readout), per head
and token, row-vector convention::

    S_hat = Diag(exp(log_alpha_t)) S
    S     = S_hat - (b_t*k_t)^T (k_t S_hat) + k_t^T (w_t*v_t)
    o_t   = (q_t * gamma_stat * 2 sigmoid(z_t)) S
    y_t   = g_t * o_t / sqrt(mean(o_t^2) + eps)
"""
from __future__ import annotations

import ctypes
from typing import Optional, Tuple

import torch

from . import _native

__all__ = [
    "GdeltaError",
    "gdelta_abi_version",
    "gdelta_status_string",
    "gdelta_fwd_workspace_bytes",
    "gdelta_fwd_selected_path",
    "gdelta_state_init",
    "gdelta_state_affine",
    "gdelta_segment_map",
    "gdelta_fwd_chunked",
    "gdelta_decode_step",
    "gdelta_bwd",
    "gdelta_gate_proj",
    "gdelta_set_wait_limit",
    "gdelta_set_wait_timeout_test",
    "gdelta_get_last_device_error",
]


class GdeltaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        name = _native.STATUS_NAMES.get(status, str(status))
        super().__init__(f"{where}: {name} ({gdelta_status_string(status)})")


def _lib():
    return _native.load()


def _check(status: int, where: str) -> None:
    if status != _native.GDELTA_OK:
        raise GdeltaError(status, where)


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _dev_ptr(t: Optional[torch.Tensor], name: str, dtype=None, shape=None, required=True):
    if t is None:
        if required:
            raise ValueError(f"{name} is required")
        return None
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    return t.data_ptr()


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return _native.GDELTA_BF16
    if t.dtype == torch.float32:
        return _native.GDELTA_F32
    raise ValueError(f"token tensors must be bf16 or fp32, got {t.dtype}")


def gdelta_abi_version() -> int:
    return int(_lib().gdelta_abi_version())


def gdelta_status_string(status: int) -> str:
    return _lib().gdelta_status_string(int(status)).decode()


def _fwd_struct(q, k, v, b, w, z, g, log_alpha, gamma_stat, S_in, S_out, y, o_raw, chunk, eps,
                path, workspace, beta=None, decay_per_token=False, qk_raw=False) -> _native.FwdArgs:
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dt = q.dtype
    a = _native.FwdArgs()
    a.B, a.T, a.H, a.dk, a.dv = int(B), int(T), int(H), int(dk), int(dv)
    a.chunk = int(chunk)
    a.dtype = _dtype_code(q)
    a.path = _native.PATHS[path]
    ks, vs = (B, T, H, dk), (B, T, H, dv)
    a.q = _dev_ptr(q, "q", dt, ks)
    a.k = _dev_ptr(k, "k", dt, ks)
    a.z = _dev_ptr(z, "z", dt, ks, required=False)
    a.b = _dev_ptr(b, "b", dt, ks, required=beta is None)
    a.v = _dev_ptr(v, "v", dt, vs)
    a.w = _dev_ptr(w, "w", dt, vs, required=beta is None)
    a.g = _dev_ptr(g, "g", dt, vs)
    a.beta = _dev_ptr(beta, "beta", dt, (B, T, H), required=False)
    a.decay_per_token = int(bool(decay_per_token))
    a.qk_raw = int(bool(qk_raw))
    a.log_alpha = _dev_ptr(log_alpha, "log_alpha", torch.float32, (B, T, H) if decay_per_token else ks)
    a.gamma_stat = _dev_ptr(gamma_stat, "gamma_stat", torch.float32, (H, dk), required=False)
    a.S_in = _dev_ptr(S_in, "S_in", torch.float32, (B, H, dk, dv), required=False)
    a.S_out = _dev_ptr(S_out, "S_out", torch.float32, (B, H, dk, dv), required=False)
    a.y = _dev_ptr(y, "y", dt, vs, required=False)
    a.o_raw = _dev_ptr(o_raw, "o_raw", torch.float32, vs, required=False)
    a.eps = float(eps)
    if workspace is not None:
        a.workspace = _dev_ptr(workspace, "workspace")
        a.workspace_bytes = workspace.numel() * workspace.element_size()
    return a


def gdelta_fwd_workspace_bytes(q, k, v, b, w, z, g, log_alpha, *, chunk: int = 64,
                               path: str = "auto", beta=None, decay_per_token: bool = False,
                               qk_raw: bool = False) -> int:
    a = _fwd_struct(q, k, v, b, w, z, g, log_alpha, None, None, None, None, None, chunk, 1e-6,
                    path, None, beta, decay_per_token, qk_raw)
    return int(_lib().gdelta_fwd_workspace_bytes(ctypes.byref(a)))


def gdelta_fwd_selected_path(q, k, v, b, w, z, g, log_alpha, *, chunk: int = 64,
                             path: str = "auto", beta=None, decay_per_token: bool = False,
                             qk_raw: bool = False) -> str:
    a = _fwd_struct(q, k, v, b, w, z, g, log_alpha, None, None, None, None, None, chunk, 1e-6,
                    path, None, beta, decay_per_token, qk_raw)
    code = int(_lib().gdelta_fwd_selected_path(ctypes.byref(a)))
    if code < 0:
        raise GdeltaError(2, "gdelta_fwd_selected_path")
    return _native.PATH_NAMES[code]


def gdelta_state_init(S: torch.Tensor, S_src: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """S <- 0 (S_src None) or S <- S_src.  S: [B,H,dk,dv] fp32 on the GPU."""
    if S.dim() != 4:
        raise ValueError("S must be [B, H, dk, dv]")
    B, H, dk, dv = S.shape
    p = _dev_ptr(S, "S", torch.float32)
    ps = _dev_ptr(S_src, "S_src", torch.float32, tuple(S.shape), required=False)
    _check(_lib().gdelta_state_init(p, B, H, dk, dv, ps, _stream(stream)), "gdelta_state_init")
    return S


def gdelta_state_affine(A: torch.Tensor, S_in: Optional[torch.Tensor] = None, D: Optional[torch.Tensor] = None,
                        S_out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """S_out = A S_in + D per (batch, head).  A [B,H,dk,dk], S_in / D / S_out
    [B,H,dk,dv] fp32 on the GPU; S_in or D None reads as zero; S_out may be D.
    Returns S_out (allocated when not given)."""
    if A.dim() != 4 or A.shape[-1] != A.shape[-2]:
        raise ValueError("A must be [B, H, dk, dk]")
    B, H, dk, _ = A.shape
    ref = S_in if S_in is not None else D if D is not None else S_out
    if ref is None:
        raise ValueError("one of S_in, D, S_out is needed for d_v")
    dv = ref.shape[-1]
    shp = (B, H, dk, dv)
    if S_out is None:
        S_out = torch.empty(shp, dtype=torch.float32, device=A.device)
    _check(_lib().gdelta_state_affine(_dev_ptr(S_out, "S_out", torch.float32, shp),
                                      _dev_ptr(A, "A", torch.float32, (B, H, dk, dk)),
                                      _dev_ptr(S_in, "S_in", torch.float32, shp, required=False),
                                      _dev_ptr(D, "D", torch.float32, shp, required=False),
                                      B, H, dk, dv, _stream(stream)), "gdelta_state_affine")
    return S_out


def gdelta_segment_map(q, k, v, b, w, z, g, log_alpha, *, beta=None, decay_per_token: bool = False,
                       qk_raw: bool = False, chunk: int = 64, path: str = "auto", stream=None
                       ) -> Tuple[torch.Tensor, torch.Tensor]:
    """(A, D) with S_end = A S_start + D for this segment of tokens, every
    (batch, head): A [B,H,dk,dk] is the forward's final state from S_in = I
    with zero values (d_v = d_k), D its final state from S_in = 0.  Two
    forward calls; their y is scratch.  z does not reach the state and is not
    read (g is read only for the scratch y)."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dev = q.device
    zeros = torch.zeros((B, T, H, dk), dtype=q.dtype, device=dev)     # v, w and g of the A pass
    eye = torch.eye(dk, dtype=torch.float32, device=dev).expand(B, H, dk, dk).contiguous()
    A = torch.empty((B, H, dk, dk), dtype=torch.float32, device=dev)
    D = torch.empty((B, H, dk, dv), dtype=torch.float32, device=dev)
    y_a = torch.empty((B, T, H, dk), dtype=q.dtype, device=dev)
    y_d = y_a if dv == dk else torch.empty((B, T, H, dv), dtype=q.dtype, device=dev)
    gdelta_fwd_chunked(q, k, zeros, b, None if beta is not None else zeros, None, zeros, log_alpha,
                       S_in=eye, S_out=A, y=y_a, chunk=chunk, path=path, stream=stream, beta=beta,
                       decay_per_token=decay_per_token, qk_raw=qk_raw)
    gdelta_fwd_chunked(q, k, v, b, w, None, g, log_alpha, S_out=D, y=y_d, chunk=chunk, path=path,
                       stream=stream, beta=beta, decay_per_token=decay_per_token, qk_raw=qk_raw)
    return A, D


def gdelta_fwd_chunked(q, k, v, b, w, z, g, log_alpha, *, gamma_stat=None, S_in=None, S_out=None,
                       y=None, o_raw=None, chunk: int = 64, eps: float = 1e-6, path: str = "auto",
                       workspace=None, return_state: bool = True, stream=None, beta=None,
                       decay_per_token: bool = False, qk_raw: bool = False
                       ) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """Chunked forward over [B,T,H,d] tokens.  Returns (y, S_out).

    Reduced gate forms: ``z`` may be None (no dynamic readout gain);
    ``beta`` [B,T,H] replaces ``b`` and ``w`` (pass them as None) with one
    gate per token and head; ``decay_per_token`` takes ``log_alpha`` as
    [B,T,H].  Together these give the KDA and Gated DeltaNet special cases.
    ``qk_raw``: q and k are pre-activation; the kernels apply SiLU and the
    per-head l2 normalisation as they load them.

    Outputs not passed in are allocated with torch on q's device; S_out is
    only allocated when ``return_state``.  ``workspace`` (uint8 CUDA tensor) is
    allocated when the selected kernel needs one and none is given.
    """
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if y is None:
        y = torch.empty((B, T, H, dv), dtype=q.dtype, device=q.device)
    if S_out is None and return_state:
        S_out = torch.empty((B, H, dk, dv), dtype=torch.float32, device=q.device)
    if workspace is None:
        need = gdelta_fwd_workspace_bytes(q, k, v, b, w, z, g, log_alpha, chunk=chunk, path=path,
                                          beta=beta, decay_per_token=decay_per_token, qk_raw=qk_raw)
        if need:
            workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    a = _fwd_struct(q, k, v, b, w, z, g, log_alpha, gamma_stat, S_in, S_out, y, o_raw, chunk, eps,
                    path, workspace, beta, decay_per_token, qk_raw)
    _check(_lib().gdelta_fwd_chunked(ctypes.byref(a), _stream(stream)), "gdelta_fwd_chunked")
    return y, S_out


def gdelta_decode_step(q, k, v, b, w, z, g, log_alpha, S, *, gamma_stat=None, y=None, o_raw=None,
                       eps: float = 1e-6, stream=None, beta=None,
                       decay_per_token: bool = False, qk_raw: bool = False) -> torch.Tensor:
    """One token per (batch, head): S [B,H,dk,dv] fp32 updated in place; returns y [B,H,dv].

    ``z``, ``beta``, ``decay_per_token`` and ``qk_raw`` as in gdelta_fwd_chunked, with
    beta [B,H] and a per-token log_alpha [B,H].
    """
    B, H, dk = q.shape
    dv = v.shape[-1]
    dt = q.dtype
    if y is None:
        y = torch.empty((B, H, dv), dtype=dt, device=q.device)
    a = _native.DecodeArgs()
    a.B, a.H, a.dk, a.dv = int(B), int(H), int(dk), int(dv)
    a.dtype = _dtype_code(q)
    a.reserved = 0
    ks, vs = (B, H, dk), (B, H, dv)
    a.q = _dev_ptr(q, "q", dt, ks)
    a.k = _dev_ptr(k, "k", dt, ks)
    a.z = _dev_ptr(z, "z", dt, ks, required=False)
    a.b = _dev_ptr(b, "b", dt, ks, required=beta is None)
    a.v = _dev_ptr(v, "v", dt, vs)
    a.w = _dev_ptr(w, "w", dt, vs, required=beta is None)
    a.g = _dev_ptr(g, "g", dt, vs)
    a.beta = _dev_ptr(beta, "beta", dt, (B, H), required=False)
    a.decay_per_token = int(bool(decay_per_token))
    a.qk_raw = int(bool(qk_raw))
    a.log_alpha = _dev_ptr(log_alpha, "log_alpha", torch.float32, (B, H) if decay_per_token else ks)
    a.gamma_stat = _dev_ptr(gamma_stat, "gamma_stat", torch.float32, (H, dk), required=False)
    a.S = _dev_ptr(S, "S", torch.float32, (B, H, dk, dv))
    a.y = _dev_ptr(y, "y", dt, vs)
    a.o_raw = _dev_ptr(o_raw, "o_raw", torch.float32, vs, required=False)
    a.eps = float(eps)
    _check(_lib().gdelta_decode_step(ctypes.byref(a), _stream(stream)), "gdelta_decode_step")
    return y


def gdelta_bwd(q, k, v, b, w, z, g, log_alpha, grad_y, *, gamma_stat=None, S_in=None, grad_S_out=None,
               eps: float = 1e-6, workspace=None, stream=None) -> dict:
    """Gradients of a loss L given dL/dy (grad_y [B,T,H,dv] fp32) and
    optionally dL/dS_T (grad_S_out [B,H,dk,dv] fp32), for the forward
    gdelta_fwd_chunked(q, k, v, b, w, z, g, log_alpha, gamma_stat=..., S_in=...)
    computes (d_k = d_v = 128).  Returns fp32 tensors under the keys q, k, v,
    b, w, z, g, log_alpha, gamma_stat ([H,dk]) and S_in ([B,H,dk,dv])."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dt = q.dtype
    dev = q.device
    ks, vs = (B, T, H, dk), (B, T, H, dv)
    f32 = dict(dtype=torch.float32, device=dev)
    out = {n: torch.empty(ks, **f32) for n in ("q", "k", "z", "b", "log_alpha")}
    out.update({n: torch.empty(vs, **f32) for n in ("v", "w", "g")})
    out["gamma_stat"] = torch.empty((H, dk), **f32)
    out["S_in"] = torch.empty((B, H, dk, dv), **f32)
    a = _native.BwdArgs()
    a.B, a.T, a.H, a.dk, a.dv = int(B), int(T), int(H), int(dk), int(dv)
    a.dtype = _dtype_code(q)
    for n, t, shp in (("q", q, ks), ("k", k, ks), ("z", z, ks), ("b", b, ks), ("v", v, vs), ("w", w, vs),
                      ("g", g, vs)):
        setattr(a, n, _dev_ptr(t, n, dt, shp))
    a.log_alpha = _dev_ptr(log_alpha, "log_alpha", torch.float32, ks)
    a.gamma_stat = _dev_ptr(gamma_stat, "gamma_stat", torch.float32, (H, dk), required=False)
    a.S_in = _dev_ptr(S_in, "S_in", torch.float32, (B, H, dk, dv), required=False)
    a.grad_y = _dev_ptr(grad_y, "grad_y", torch.float32, vs)
    a.grad_S_out = _dev_ptr(grad_S_out, "grad_S_out", torch.float32, (B, H, dk, dv), required=False)
    a.eps = float(eps)
    for n in ("q", "k", "z", "b", "log_alpha", "v", "w", "g", "gamma_stat", "S_in"):
        setattr(a, "grad_" + n, out[n].data_ptr())
    need = int(_lib().gdelta_bwd_workspace_bytes(ctypes.byref(a)))
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    a.workspace = _dev_ptr(workspace, "workspace")
    a.workspace_bytes = workspace.numel() * workspace.element_size()
    _check(_lib().gdelta_bwd(ctypes.byref(a), _stream(stream)), "gdelta_bwd")
    return out


GATE_RANKS = (64, 64, 128, 128, 128)


def _gate_proj_struct(x, w_down, w_up, bias, ranks, out, workspace) -> _native.GateProjArgs:
    if x.dim() != 2:
        raise ValueError("x must be [N, d]")
    N, d = x.shape
    R = int(sum(ranks))
    a = _native.GateProjArgs()
    a.N, a.d = int(N), int(d)
    for i, r in enumerate(ranks):
        a.ranks[i] = int(r)
    bf = torch.bfloat16
    a.x = _dev_ptr(x, "x", bf, (N, d))
    a.w_down = _dev_ptr(w_down, "w_down", bf, (d, R))
    a.w_up = _dev_ptr(w_up, "w_up", bf, (R, d))
    a.bias = _dev_ptr(bias, "bias", torch.float32, (5, d))
    if out is not None:
        a.log_alpha = _dev_ptr(out["log_alpha"], "log_alpha", torch.float32, (N, d))
        for n in ("b", "g", "w", "z"):
            setattr(a, n, _dev_ptr(out[n], n, bf, (N, d)))
    if workspace is not None:
        a.workspace = _dev_ptr(workspace, "workspace")
        a.workspace_bytes = workspace.numel() * workspace.element_size()
    return a


def gdelta_gate_proj(x, w_down, w_up, bias, *, ranks=GATE_RANKS, out=None, workspace=None, stream=None) -> dict:
    """Five-gate low-rank projection (Muir review §2.3): x [N, d] bf16,
    w_down [d, R], w_up [R, d] bf16 (gate blocks in the order f, b, g, w, q),
    bias [5, d] fp32.  Returns the mixer's gate inputs as [N, d] tensors:
    log_alpha (fp32) = log sigmoid(f), b = 2 sigmoid, g, w = sigmoid, z = the
    q logit (bf16).  ``out`` (a dict with those keys) and ``workspace`` are
    allocated when not given."""
    N, d = x.shape
    if out is None:
        out = {"log_alpha": torch.empty((N, d), dtype=torch.float32, device=x.device)}
        out.update({n: torch.empty((N, d), dtype=torch.bfloat16, device=x.device) for n in ("b", "g", "w", "z")})
    if workspace is None:
        need = int(_lib().gdelta_gate_proj_workspace_bytes(
            ctypes.byref(_gate_proj_struct(x, w_down, w_up, bias, ranks, None, None))))
        if need == 0:
            raise GdeltaError(2, "gdelta_gate_proj_workspace_bytes")
        workspace = torch.empty(need, dtype=torch.uint8, device=x.device)
    a = _gate_proj_struct(x, w_down, w_up, bias, ranks, out, workspace)
    _check(_lib().gdelta_gate_proj(ctypes.byref(a), _stream(stream)), "gdelta_gate_proj")
    return out


def gdelta_set_wait_limit(polls: int) -> None:
    """Polls before a tensor-core kernel's bounded wait gives up (0 = default 2^20)."""
    _check(_lib().gdelta_set_wait_limit(int(polls)), "gdelta_set_wait_limit")


def gdelta_set_wait_timeout_test(on: bool) -> None:
    """Failure-path test switch: tensor-core forward calls queued while it is on
    first wait on a barrier nothing completes and report GDELTA_ERR_TIMEOUT."""
    _check(_lib().gdelta_set_wait_timeout_test(int(bool(on))), "gdelta_set_wait_timeout_test")


def gdelta_get_last_device_error(stream=None) -> int:
    """Synchronises the stream; returns (and clears) the device status code."""
    return int(_lib().gdelta_get_last_device_error(_stream(stream)))
