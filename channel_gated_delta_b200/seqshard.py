"""One long sequence split over ranks (one process per GPU).

Each token's update moves the state by an affine map whose linear part acts
on the key rows only, so a segment of tokens moves it by S_end = A S_start + D
("Kimi3 = GPT2 x 22580" §4: a chunk's transition is the product of its
tokens' generalised Householder factors plus an accumulated write).  Rank r
holds segment r of every (batch, head):

1. (A_r, D_r) = gdelta_segment_map(segment r)         two forward calls
2. all-gather of (A_j, D_j) over the group             one collective
3. S_start(r) = map_{r-1} o ... o map_0 (S_in)          gdelta_state_affine
4. y_r = gdelta_fwd_chunked(segment r, S_in = S_start(r))
5. S_final = map_{N-1} o ... o map_{r+1} (S_end(r))     the same on every rank

Each rank runs three forwards over T/N tokens instead of one over T, so the
split pays from N > 3 on; the exchange is 4 B (d_k + d_v) d_k bytes per
(batch, head) and rank.
"""
from __future__ import annotations

from typing import Callable, List, Optional, Sequence, Tuple

import torch

from . import gdelta_fwd_chunked, gdelta_segment_map, gdelta_state_affine

Compose = Callable[[torch.Tensor, Optional[torch.Tensor], torch.Tensor], torch.Tensor]


def gather_maps(A: torch.Tensor, D: torch.Tensor, group=None) -> Tuple[List[torch.Tensor], List[torch.Tensor]]:
    """Every rank's (A, D), in rank order, on every rank."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    As = [torch.empty_like(A) for _ in range(world)]
    Ds = [torch.empty_like(D) for _ in range(world)]
    dist.all_gather(As, A.contiguous(), group=group)
    dist.all_gather(Ds, D.contiguous(), group=group)
    return As, Ds


def compose_range(As: Sequence[torch.Tensor], Ds: Sequence[torch.Tensor], lo: int, hi: int,
                  S: Optional[torch.Tensor], compose: Compose) -> Optional[torch.Tensor]:
    """Applies the maps of segments lo .. hi-1, in order, to S (None = zero)."""
    for j in range(lo, hi):
        S = compose(As[j], S, Ds[j])
    return S


def compose_affine(A, S, D):
    """S -> A S + D on the GPU (gdelta_state_affine); S None reads as zero."""
    return gdelta_state_affine(A, S_in=S, D=D)


def gdelta_fwd_seqshard(q, k, v, b, w, z, g, log_alpha, *, group=None, S_in=None, gamma_stat=None,
                        y=None, chunk: int = 64, eps: float = 1e-6, path: str = "auto", beta=None,
                        decay_per_token: bool = False, qk_raw: bool = False, stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Forward over this rank's segment of one sequence split in rank order.

    Tensors are this rank's segment ([B, T_r, H, d]); S_in is the state before
    the first segment (the same on every rank, or None for zero).  Returns
    this segment's y and the state after the whole sequence (every rank)."""
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        rank, world = dist.get_rank(group), dist.get_world_size(group)
    else:
        rank, world = 0, 1
    if world == 1:                                    # one segment: the plain forward
        return gdelta_fwd_chunked(q, k, v, b, w, z, g, log_alpha, gamma_stat=gamma_stat, S_in=S_in, y=y,
                                  chunk=chunk, eps=eps, path=path, stream=stream, beta=beta,
                                  decay_per_token=decay_per_token, qk_raw=qk_raw)
    A, D = gdelta_segment_map(q, k, v, b, w, z, g, log_alpha, beta=beta, decay_per_token=decay_per_token,
                              qk_raw=qk_raw, chunk=chunk, path=path, stream=stream)
    As, Ds = gather_maps(A, D, group)
    S0 = compose_range(As, Ds, 0, rank, S_in, compose_affine)
    y, S_end = gdelta_fwd_chunked(q, k, v, b, w, z, g, log_alpha, gamma_stat=gamma_stat, S_in=S0, y=y,
                                  chunk=chunk, eps=eps, path=path, stream=stream, beta=beta,
                                  decay_per_token=decay_per_token, qk_raw=qk_raw)
    S_final = compose_range(As, Ds, rank + 1, world, S_end, compose_affine)
    return y, S_final
