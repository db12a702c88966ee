"""Splitting one prefill workload over ranks by KV group: tensor parallelism
of the attention heads.

"Llama 3.1 Architecture: Dense Scaling to 405B and 128K Context", "The 4D
Parallelism Execution Strategy", tensor-parallel bullet: the linear weights
are partitioned over the 8 GPUs of an NVLink node. With the QKV projection
split by output columns, rank r produces the query, key and value heads of
its own columns; under GQA ("How Meta's Llama 3.1 405B Architecture Actually
Works", GQA paragraph: each KV head serves a group of G = Hq / Hkv query
heads) a rank that owns KV heads [g0, g1) and their query heads
[g0 G, g1 G) has everything its heads' attention reads. The step needs no
collective: each rank runs the prefill on its contiguous [B, S, Hq/N, D] and
[B, S, Hkv/N, D] tensors, and the row-parallel output projection that follows
consumes its heads in place.

N must divide Hkv (N <= 8 for the pages' 8 KV heads). gather_heads (an
all-gather along the head axis) is only needed to assemble a whole output,
e.g. to compare it with an unsharded run.
"""
from __future__ import annotations


def kv_group_heads(Hq: int, Hkv: int, world_size: int, rank: int):
    """(hq0, hq1, hkv0, hkv1): the query-head and KV-head ranges of `rank`."""
    if world_size <= 0 or not (0 <= rank < world_size):
        raise ValueError("bad world_size / rank")
    if Hkv <= 0 or Hq % Hkv != 0:
        raise ValueError("Hq must be a positive multiple of Hkv")
    if Hkv % world_size != 0:
        raise ValueError(f"world_size {world_size} must divide the {Hkv} KV heads")
    G = Hq // Hkv
    per = Hkv // world_size
    return rank * per * G, (rank + 1) * per * G, rank * per, (rank + 1) * per


def shard_heads(x, h0: int, h1: int):
    """Heads [h0, h1) of a [B, S, H, D] tensor, as a contiguous tensor (the
    layout a column-parallel QKV projection writes on its rank)."""
    return x[:, :, h0:h1].contiguous()


def shard_qkv(q, k, v, world_size: int, rank: int):
    """The rank's (q, k, v) heads of one workload."""
    hq0, hq1, hk0, hk1 = kv_group_heads(q.shape[2], k.shape[2], world_size, rank)
    return shard_heads(q, hq0, hq1), shard_heads(k, hk0, hk1), shard_heads(v, hk0, hk1)


def gather_heads(x_local, world_size: int, group=None):
    """All-gather of every rank's [B, S, H/N, D] heads into [B, S, H, D]."""
    import torch
    import torch.distributed as dist
    if world_size == 1:
        return x_local
    parts = [torch.empty_like(x_local) for _ in range(world_size)]
    dist.all_gather(parts, x_local.contiguous(), group=group)
    return torch.cat(parts, dim=2)


def tp_prefill(q_local, k_local, v_local, doc_offsets=None, rope_theta: float = 500000.0, attn=None, out=None):
    """One rank's share of a KV-group-split prefill: attention of its own
    heads (no exchange). attn(q, k, v, doc_offsets, rope_theta, out) computes
    it; it defaults to the library's llama_attn_prefill."""
    if attn is None:
        from . import llama_attn_prefill
        return llama_attn_prefill(q_local, k_local, v_local, out=out, doc_offsets=doc_offsets,
                                  rope_theta=rope_theta)
    return attn(q_local, k_local, v_local, doc_offsets, rope_theta, out)
