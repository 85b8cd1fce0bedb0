"""Head-parallel split of one attention layer over ranks (one process per GPU).

Every step of the S2O path works per head: a query head's orderings, block scores, early-stop
lists and attention read only its own queries and its KV head's keys and values ("S2O: Early
Stopping for Sparse Attention via Online Permutation", Summary ¶2: the orderings are built for
each head). So one layer splits by KV head with no exchange at all: rank r of R takes the KV heads
{g : g mod R = r} and the G query heads of each, and K and V are never replicated. The output
stays sharded, or one all-gather over the process group assembles it in head order. The pages
themselves run on a single GPU (Key points); this is the natural split of their per-head work.

Only tensor bookkeeping lives here (which heads, slicing, the final gather): the prefill itself
is the library's C ABI on each rank's shard.
"""
from __future__ import annotations

import dataclasses

import torch

__all__ = ["kv_heads", "query_heads", "shard_config", "shard_inputs", "gather_output"]


def kv_heads(n_kv_heads: int, rank: int, world: int) -> list[int]:
    """KV heads of `rank`: g = rank, rank + world, ... (round robin)."""
    if not 0 <= rank < world:
        raise ValueError("rank out of range")
    return list(range(rank, n_kv_heads, world))


def query_heads(n_q_heads: int, n_kv_heads: int, rank: int, world: int) -> list[int]:
    """Query heads of `rank`: the G = n_q_heads / n_kv_heads heads of each of its KV heads."""
    G = n_q_heads // n_kv_heads
    return [g * G + i for g in kv_heads(n_kv_heads, rank, world) for i in range(G)]


def shard_config(cfg, rank: int, world: int):
    """The layer configuration of `rank`'s shard (same fields, fewer heads). `cfg` is any frozen
    dataclass with n_q_heads / n_kv_heads fields (the binding's Config, gen.Workload)."""
    n_kv = len(kv_heads(cfg.n_kv_heads, rank, world))
    if n_kv == 0:
        raise ValueError("more ranks than KV heads: this rank would have no work")
    G = cfg.n_q_heads // cfg.n_kv_heads
    return dataclasses.replace(cfg, n_q_heads=G * n_kv, n_kv_heads=n_kv)


def shard_inputs(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, rank: int, world: int):
    """Contiguous shards of Q [batch, Hq, N, d] and K, V [batch, Hkv, N, d] for `rank`."""
    n_q, n_kv = q.shape[1], k.shape[1]
    qi = torch.tensor(query_heads(n_q, n_kv, rank, world), device=q.device)
    ki = torch.tensor(kv_heads(n_kv, rank, world), device=k.device)
    return (q.index_select(1, qi).contiguous(), k.index_select(1, ki).contiguous(),
            v.index_select(1, ki).contiguous())


def gather_output(o_shard: torch.Tensor, n_q_heads: int, n_kv_heads: int, rank: int, world: int,
                  dist) -> torch.Tensor:
    """The full O [batch, Hq, N, d] in head order from every rank's shard, with one all-gather
    (shards are padded to the largest rank's head count when R does not divide Hkv)."""
    heads = [query_heads(n_q_heads, n_kv_heads, r, world) for r in range(world)]
    most = max(len(h) for h in heads)
    b, h_r, n, d = o_shard.shape
    if h_r != len(heads[rank]):
        raise ValueError("shard does not match this rank's heads")
    send = o_shard
    if h_r < most:
        send = torch.cat([o_shard, o_shard.new_zeros((b, most - h_r, n, d))], dim=1)
    parts = [torch.empty_like(send) for _ in range(world)]
    dist.all_gather(parts, send.contiguous())
    out = o_shard.new_empty((b, n_q_heads, n, d))
    for r in range(world):
        idx = torch.tensor(heads[r], device=out.device)
        out.index_copy_(1, idx, parts[r][:, :len(heads[r])])
    return out
