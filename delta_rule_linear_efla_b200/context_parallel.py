"""Context-parallel EFLA forward: one sequence sharded over the ranks of a process group.

Rank r holds tokens [r*Ls, (r+1)*Ls) of every head (any shard lengths work; shards are in rank
order).  A stretch of tokens maps the state affinely, S_out = P S_in + H: by the update rule
("Exact Flow Linear Attention", technical summary, Methodology 3) each token applies
S <- (I - a k k^T) S + a k v^T, so over the stretch P is the product of the (I - a k k^T) and H
is the stretch's state from zero.  So:

1. every rank computes its shard's map: H from S0 = 0, and P from S0 = I with v = 0 (rank 0,
   which knows its starting state, runs its shard for real instead: P = 0, H = its final state);
2. the maps are all-gathered (2 x [B,H,dk,dv or dk] fp32 per rank: NCCL over NVLink on GPUs);
3. rank r chains S_in(r) = P_{r-1}( ... (P_1 H_0 + H_1) ... ) + H_{r-1} with efla_state_affine;
4. rank r > 0 reruns its shard from S_in(r), which gives its outputs and its final state.

Ranks other than 0 do three passes over their shard; the pass in step 1 and the one in step 4
are the chunk forward of this library.  The collective is the one all_gather in step 2; every
rank makes it, in the same order.  The last rank's final state is the sequence's S_final.
"""
from __future__ import annotations

import torch

from . import efla


def _gpu_fwd(q, k, v, beta, S0, rule, chunk):
    return efla.chunk_fwd(q, k, v, beta, S0, chunk=chunk, rule=rule)


def _gpu_affine(P, S_in, H):
    return efla.state_affine(P, S_in, H)


def shard_map(q, k, v, beta, rule: str = "exact", chunk: int = 64, fwd=None):
    """(P, H) of this shard: S_out = P S_in + H.  P is [B,H,dk,dk], H is [B,H,dk,dv]."""
    fwd = fwd or _gpu_fwd
    B, Hh, L, dk = q.shape
    _, Hm = fwd(q, k, v, beta, None, rule, chunk)
    v0 = torch.zeros((B, Hh, L, dk), dtype=v.dtype, device=v.device)
    eye = torch.eye(dk, dtype=torch.float32, device=q.device).expand(B, Hh, dk, dk).contiguous()
    _, P = fwd(q, k, v0, beta, eye, rule, chunk)
    return P, Hm


def chain_start(maps, affine=None):
    """Starting state of the shard after `maps` = [(P_0, H_0), (P_1, H_1), ...] (in order):
    S = P_j S + H_j from S = 0.  Returns None for an empty list (the sequence's own S0)."""
    affine = affine or _gpu_affine
    S = None
    for P, Hm in maps:
        S = affine(P, S, Hm)
    return S


def cp_chunk_fwd(q, k, v, beta, S0=None, group=None, rule: str = "exact", chunk: int = 64,
                 fwd=None, affine=None):
    """Forward over this rank's shard of a sequence sharded across `group` (rank order = token
    order).  Returns (o for this shard, the state after this shard); the last rank's state is
    the sequence's S_final.  S0 is the sequence's initial state, used by rank 0 only."""
    import torch.distributed as dist

    fwd = fwd or _gpu_fwd
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    if world == 1:
        return fwd(q, k, v, beta, S0, rule, chunk)
    B, Hh, _, dk = q.shape
    dv = v.shape[-1]
    if rank == 0:
        o, S_out = fwd(q, k, v, beta, S0, rule, chunk)
        P = torch.zeros((B, Hh, dk, dk), dtype=S_out.dtype, device=q.device)
        Hm = S_out.contiguous()
    else:
        P, Hm = shard_map(q, k, v, beta, rule, chunk, fwd)
    Ps = [torch.empty_like(P) for _ in range(world)]
    Hs = [torch.empty_like(Hm) for _ in range(world)]
    dist.all_gather(Ps, P.contiguous(), group=group)
    dist.all_gather(Hs, Hm.contiguous(), group=group)
    if rank == 0:
        return o, S_out
    S_in = chain_start(list(zip(Ps[:rank], Hs[:rank])), affine)
    assert S_in is not None and S_in.shape == (B, Hh, dk, dv)
    return fwd(q, k, v, beta, S_in, rule, chunk)
