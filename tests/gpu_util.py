"""Helpers shared by the GPU tests: device copies and the error metric."""
import numpy as np
import torch

TOKEN_KEYS = ("q", "k", "v", "b", "w", "z", "g", "log_alpha")

# Spec tolerances: max |diff| / rms(reference).
TOL_F32 = 1e-4
TOL_BF16 = 2e-2


def to_dev(inputs, device="cuda"):
    return {k: (v.to(device) if isinstance(v, torch.Tensor) else v) for k, v in inputs.items()}


def err(x, ref) -> float:
    """max |x - ref| / rms(ref), in float64."""
    x = x.detach().cpu().double().numpy() if isinstance(x, torch.Tensor) else np.asarray(x, np.float64)
    ref = np.asarray(ref, np.float64)
    rms = np.sqrt(np.mean(ref * ref))
    return float(np.max(np.abs(x - ref)) / max(rms, 1e-300))


def err_stored(x, ref, storage) -> float:
    """``err`` for an output stored in a 16-bit float: each element may also
    carry its storage rounding (half an ulp of the reference value in that
    format) on top of the computation error.  fp32 outputs use ``err``."""
    if storage == "f32":
        return err(x, ref)
    x = x.detach().cpu().double().numpy() if isinstance(x, torch.Tensor) else np.asarray(x, np.float64)
    ref = np.asarray(ref, np.float64)
    mant = {"bf16": 8, "f16": 11}[storage]          # significand bits incl. the implicit one
    e = np.floor(np.log2(np.maximum(np.abs(ref), 1e-300)))
    half_ulp = np.ldexp(1.0, (e - mant).astype(np.int64))
    rms = np.sqrt(np.mean(ref * ref))
    excess = np.maximum(np.abs(x - ref) - half_ulp, 0.0)
    return float(np.max(excess) / max(rms, 1e-300))


def gpu_fwd(inputs, **kw):
    """Runs the chunked forward through the C ABI; returns CPU tensors."""
    import channel_gated_delta_b200 as gd
    d = to_dev(inputs)
    B, T, H, dk = d["q"].shape
    dv = d["v"].shape[-1]
    o_raw = torch.empty((B, T, H, dv), dtype=torch.float32, device="cuda") if kw.pop("want_o", True) else None
    y, S = gd.gdelta_fwd_chunked(d["q"], d["k"], d["v"], d["b"], d["w"], d["z"], d["g"], d["log_alpha"],
                                 gamma_stat=d.get("gamma_stat"), o_raw=o_raw, **kw)
    torch.cuda.synchronize()
    assert gd.gdelta_get_last_device_error() == 0
    return y.cpu(), (S.cpu() if S is not None else None), (o_raw.cpu() if o_raw is not None else None)


def sel_heads(x, heads):
    """[B,T,H,d] tensor -> [n,T,d] for the listed (b,h)."""
    return torch.stack([x[b, :, h] for (b, h) in heads])
