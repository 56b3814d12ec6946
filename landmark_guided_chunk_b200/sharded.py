"""Multi-device HSA: the (batch, kv head) split of prefill and the
context-sharded decode.

Prefill split (``prefill_shard_range``, ``sharded_prefill``).  Each kv head's
landmarks, selection, chunk attention and fusion read only that kv head's K, V
and its G query heads (HSA summary page, Implementation: one selection per
query, attention inside the kept chunks; the GQA group shares it), and each
sequence is independent.  So the (b, kv head) units split over devices with no
exchange at all: a rank holds the Q, K, V of its units -- the layout a
head-parallel model already has -- and computes their O.  With Hkv divisible
by the world size the ranks take contiguous blocks of Hkv / world kv heads
(this shortens one long sequence's prefill); otherwise, with B divisible, they
take contiguous blocks of sequences.  The only collective is optional: an
all-gather that assembles the whole O on every rank.

Context-sharded decode (HSA summary page, Implementation: the retrieval
scores rank the chunks and weight their outputs).

A long context's chunks are split into contiguous ranges, one per device: each
rank holds K, V and the landmarks of its range only.  A decode step then runs
in three parts:

1. local (``shard_partials``): every rank selects its own top kmax chunks with
   the router off -- kmax = 2k when the router is on, so no rank's list is cut
   before the global decision -- turns their indices into global chunk
   indices, and computes each kept chunk's attention output without a fusion
   weight (``hsa_attend_partials``);
2. exchange (``gather_shards``): one all-gather over the process group leaves
   every rank the shard-major concatenation of all ranks' (score, idx, keff,
   o) -- per kv head, kmax * (G*d*4 + 8) bytes;
3. merge (``hsa_merge_partials``): the top kmax of the union in the
   single-device order, the gap router on the merged list, and the
   score-weighted sum of the kept chunks' outputs.

The global top kmax is always inside the union of the local top kmax lists,
so the result is the selection and output of one device holding the whole
context (up to the summation order of fp32 scores).  The ranks compute their
own chunks only; the only cross-device traffic is step 2.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import attend_partials, forward, kmax_of, merge_partials, select

__all__ = ["local_q_pos", "shard_partials", "gather_shards", "sharded_decode", "prefill_shard_range",
           "shard_inputs", "sharded_prefill"]


def _world_rank(group):
    if group is None and not dist.is_initialized():
        return 1, 0
    return dist.get_world_size(group), dist.get_rank(group)


def prefill_shard_range(B: int, Hkv: int, world: int, rank: int):
    """This rank's units of the (b, kv head) split: ("heads", j0, j1) -- kv
    heads j0..j1-1 of every sequence -- when world divides Hkv, else
    ("batch", b0, b1) -- sequences b0..b1-1 -- when it divides B."""
    if Hkv % world == 0:
        n = Hkv // world
        return "heads", rank * n, (rank + 1) * n
    if B % world == 0:
        n = B // world
        return "batch", rank * n, (rank + 1) * n
    raise ValueError(f"neither Hkv={Hkv} nor B={B} is divisible by the world size {world}")


def shard_inputs(Q, K, V, world: int, rank: int):
    """This rank's part of Q [B,T,H,d], K and V [B,T,Hkv,d] under the (b, kv
    head) split, as contiguous copies (a head-parallel model holds them this way
    already).  Returns (kind, Q, K, V) with kind "heads" or "batch"."""
    B, Hkv = K.shape[0], K.shape[2]
    G = Q.shape[2] // Hkv
    kind, a, b = prefill_shard_range(B, Hkv, world, rank)
    if kind == "heads":
        return kind, Q[:, :, a * G:b * G].contiguous(), K[:, :, a:b].contiguous(), V[:, :, a:b].contiguous()
    return kind, Q[a:b].contiguous(), K[a:b].contiguous(), V[a:b].contiguous()


def sharded_prefill(Q, K, V, W_L, S, k, tau=0.0, kind="heads", group=None, gather=False, forward_fn=forward):
    """The (b, kv head) split of a prefill on this rank.  Q, K, V are this
    rank's shard and kind its split (``shard_inputs``); W_L is shared.  Returns
    this rank's O, or with gather=True the whole O [B, T, H, d] on every rank,
    assembled by one all-gather (ranks concatenated along the heads or the
    batch).  forward_fn computes one shard (the CUDA path by default)."""
    O = forward_fn(Q, K, V, W_L, S, k, tau)
    world, _ = _world_rank(group)
    if not gather or world == 1:
        return O
    parts = [torch.empty_like(O) for _ in range(world)]
    dist.all_gather(parts, O.contiguous(), group=group)
    return torch.cat(parts, dim=2 if kind == "heads" else 0)


def local_q_pos(q_pos0: int, chunk0: int, S: int) -> int:
    """Position of the query relative to a shard whose first chunk is global
    chunk chunk0: the shard's candidates are then its chunks c < (q_pos0 / S - chunk0)."""
    return max(0, q_pos0 - chunk0 * S)


def shard_partials(Q, K, V, L, S, k, tau, q_pos0, chunk0, kv_len=None, ws=None):
    """Part 1 on one rank.  K, V [B, Tcap, Hkv, d] hold the shard's tokens (the
    first kv_len of them, default all); L [B, Hkv, Tcap // S, d] their landmarks;
    chunk0 is the global index of the shard's first chunk.  Returns (score, idx,
    keff, o) with global chunk indices in idx."""
    km = kmax_of(k, tau)
    qp = local_q_pos(q_pos0, chunk0, S)
    n = K.shape[1] if kv_len is None else kv_len
    idx, score, keff = select(Q, L, S, km, 0.0, qp, Tkv=n, ws=ws)
    o = attend_partials(Q, K, V, idx, keff, S, km, 0.0, qp, kv_len=n, ws=ws)
    gidx = torch.where(idx >= 0, idx + chunk0, idx)
    return score, gidx, keff, o


def gather_shards(tensors, group=None):
    """Part 2: all-gather each tensor over the group and stack the ranks'
    copies shard-major (rank order).  With no group (or one rank) the tensors
    are just given a leading axis of 1."""
    world = 1 if group is None and not dist.is_initialized() else dist.get_world_size(group)
    out = []
    for t in tensors:
        if world == 1:
            out.append(t.unsqueeze(0))
            continue
        parts = [torch.empty_like(t) for _ in range(world)]
        dist.all_gather(parts, t.contiguous(), group=group)
        out.append(torch.stack(parts))
    return out


def sharded_decode(Q, K, V, L, S, k, tau, q_pos0, chunk0, group=None, kv_len=None, ws=None,
                   return_selection=False):
    """A whole decode step on this rank's shard; every rank returns the same O
    (and, with return_selection, the merged (idx, score, keff))."""
    score, gidx, keff, o = shard_partials(Q, K, V, L, S, k, tau, q_pos0, chunk0, kv_len, ws)
    sc_all, idx_all, ke_all, o_all = gather_shards((score, gidx, keff, o), group)
    return merge_partials(sc_all, idx_all, ke_all, o_all, S, k, tau, dtype=Q.dtype,
                          return_selection=return_selection)
