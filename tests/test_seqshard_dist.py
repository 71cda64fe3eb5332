"""Sequence sharding's host logic on CPU (gloo, world sizes 2 and 3): each rank
holds one segment of a sequence, gets its segment's affine state map from two
runs of the float64 oracle (state I with zero values -> A; state 0 -> D), and
the product's all-gather and composition helpers give it its starting state.
The per-rank oracle run from that state must equal the oracle over the whole
sequence, so the affine decomposition and the exchange order are both checked
without a GPU."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _segment(inp, lo, hi):
    return {k: (v[:, lo:hi] if v.dim() == 4 else v) for k, v in inp.items()}


def _worker(rank, world, port, out, T, dk, dv):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    import oracle
    import synth
    from channel_gated_delta_b200.seqshard import compose_range, gather_maps
    dist.init_process_group("gloo", rank=rank, world_size=world)
    H = 2
    inp = synth.generate(synth.GdnShape(B=1, T=T, H=H, dk=dk, dv=dv, dtype="f32", u_low=-4, u_high=0, seed=17))
    bounds = np.linspace(0, T, world + 1).astype(int)
    seg = _segment(inp, bounds[rank], bounds[rank + 1])
    heads = oracle.all_heads(1, H)
    # the segment's map from two runs: S_in = I with v = 0 (d_v = d_k) -> A; S_in = 0 -> D
    amap = dict(seg)
    z0 = torch.zeros(seg["k"].shape, dtype=seg["k"].dtype)
    amap["v"], amap["w"], amap["g"] = z0, z0, z0
    A = oracle.forward(amap, heads=heads, S0=np.stack([np.eye(dk)] * H))["S"]
    D = oracle.forward(seg, heads=heads)["S"]
    As, Ds = gather_maps(torch.from_numpy(A), torch.from_numpy(D))

    def compose(Am, S, Dm):
        return Dm.clone() if S is None else Am @ S + Dm

    S0 = compose_range(As, Ds, 0, rank, None, compose)
    r = oracle.forward(seg, heads=heads, S0=None if S0 is None else S0.numpy())
    S_final = compose_range(As, Ds, rank + 1, world, torch.from_numpy(r["S"]), compose)
    full = oracle.forward(inp, heads=heads)
    y_ref = full["y"][:, bounds[rank]:bounds[rank + 1]]
    out[rank] = (float(np.max(np.abs(r["y"] - y_ref)) / np.sqrt(np.mean(y_ref ** 2))),
                 float(np.max(np.abs(S_final.numpy() - full["S"])) / np.sqrt(np.mean(full["S"] ** 2))))
    dist.destroy_process_group()


@pytest.mark.parametrize("world,T,dk,dv", [(2, 150, 64, 64), (3, 97, 32, 64)])
def test_segment_maps_compose_across_ranks(world, T, dk, dv):
    port = _free_port()
    out = mp.Manager().dict()
    mp.spawn(_worker, args=(world, port, out, T, dk, dv), nprocs=world, join=True)
    for r in range(world):
        e_y, e_s = out[r]
        assert e_y < 1e-9 and e_s < 1e-9, (r, e_y, e_s)


def _worker_orchestration(rank, world, port, out):
    """gdelta_fwd_seqshard itself, with its three GPU calls replaced inside this
    test by float64 oracle stand-ins of the same contract."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    import oracle
    import synth
    from channel_gated_delta_b200 import seqshard
    dist.init_process_group("gloo", rank=rank, world_size=world)
    B, H, dk, dv, T = 2, 2, 16, 8, 120
    inp = synth.generate(synth.GdnShape(B=B, T=T, H=H, dk=dk, dv=dv, dtype="f32", u_low=-4, u_high=0, seed=23))
    S_in = torch.from_numpy(np.random.Generator(np.random.PCG64(4)).standard_normal((B, H, dk, dv)) * 0.3)
    bounds = np.linspace(0, T, world + 1).astype(int)
    seg = _segment(inp, bounds[rank], bounds[rank + 1])

    def fake_fwd(q, k, v, b, w, z, g, log_alpha, gamma_stat=None, S_in=None, y=None, **kw):
        t = {"q": q, "k": k, "v": v, "b": b, "w": w, "z": z, "g": g, "log_alpha": log_alpha,
             "gamma_stat": gamma_stat}
        if t["z"] is None:
            t["z"] = torch.zeros_like(q)
        r = oracle.forward_full(t, S0=None if S_in is None else S_in.numpy())
        return torch.from_numpy(r["y"]), torch.from_numpy(r["S"])

    def fake_map(q, k, v, b, w, z, g, log_alpha, **kw):
        zero = torch.zeros(q.shape, dtype=q.dtype)
        eye = torch.eye(dk, dtype=torch.float64).expand(B, H, dk, dk).contiguous()
        _, A = fake_fwd(q, k, zero, b, zero, None, zero, log_alpha, S_in=eye)
        _, D = fake_fwd(q, k, v, b, w, None, g, log_alpha)
        return A, D

    seqshard.gdelta_fwd_chunked = fake_fwd
    seqshard.gdelta_segment_map = fake_map
    seqshard.compose_affine = lambda A, S, D: D.clone() if S is None else A @ S + D
    y, S_final = seqshard.gdelta_fwd_seqshard(seg["q"], seg["k"], seg["v"], seg["b"], seg["w"], seg["z"],
                                              seg["g"], seg["log_alpha"], gamma_stat=seg["gamma_stat"],
                                              S_in=S_in)
    full = oracle.forward_full(inp, S0=S_in.numpy())
    y_ref = full["y"][:, bounds[rank]:bounds[rank + 1]]
    out[rank] = (float(np.max(np.abs(y.numpy() - y_ref))), float(np.max(np.abs(S_final.numpy() - full["S"]))))
    dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_seqshard_forward_orchestration(world):
    """Every rank's y is its slice of the whole-sequence output and every rank
    ends with the whole sequence's final state (S_in given, B = H = 2)."""
    port = _free_port()
    out = mp.Manager().dict()
    mp.spawn(_worker_orchestration, args=(world, port, out), nprocs=world, join=True)
    for r in range(world):
        e_y, e_s = out[r]
        assert e_y < 1e-9 and e_s < 1e-9, (r, e_y, e_s)
