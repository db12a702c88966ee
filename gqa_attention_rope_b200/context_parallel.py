"""Context parallelism for long-sequence prefill: the sequence is split along
tokens over the ranks and the keys and values are exchanged ("Llama 3.1
Architecture: Dense Scaling to 405B and 128K Context", "The 4D Parallelism
Execution Strategy", context-parallel bullet: the 128K sequence is partitioned
along the token dimension across 8 groups of GPUs, with the KV states
communicated).

Split (zigzag): the S tokens are cut into 2N equal chunks; rank r owns chunks
r and 2N-1-r. Under the causal mask chunk c costs about c + 1/2 chunk-sized key
blocks, so every rank gets the same work, (r + 1/2) + (2N-1-r + 1/2) = 2N.

Exchange: each rank holds the queries, keys and values of its own two chunks.
One all-gather of K and one of V per chunk slot (torch.distributed; NCCL over
NVLink on GPUs) place every chunk at its sequence position in a local
[B, S, Hkv, D] buffer, so the attention kernel reads only this GPU's memory.
With GQA the exchanged bytes are small: 2 * S * Hkv * D * 2 bytes per batch
row (0.5 GiB at S = 128K, Hkv = 8, D = 128).

Compute: llama_attn_prefill_cp over the rank's 2L query rows against the whole
sequence (causal at global positions, queries rotated at their global
positions). The result rows are final: every key a query sees is local after
the exchange, so no log-sum-exp merge across ranks is needed.
"""
from __future__ import annotations

TILE = 128  # the prefill kernel's query tile: chunk lengths and positions are multiples of it


def zigzag_chunks(S: int, world_size: int, rank: int):
    """(pos_a, pos_b, L): global start of rank's first and second chunk and
    the chunk length. S must be a multiple of 2 * world_size * 128."""
    if world_size <= 0 or not (0 <= rank < world_size):
        raise ValueError("bad world_size / rank")
    n = 2 * world_size
    if S <= 0 or S % (n * TILE) != 0:
        raise ValueError(f"S={S} must be a positive multiple of 2 * world_size * {TILE} = {n * TILE}")
    L = S // n
    return rank * L, (n - 1 - rank) * L, L


def shard_rows(x, world_size: int, rank: int):
    """The rank's rows of a [B, S, ...] tensor: chunk r followed by chunk
    2N-1-r, as one contiguous [B, 2L, ...] tensor."""
    import torch
    pos_a, pos_b, L = zigzag_chunks(x.shape[1], world_size, rank)
    return torch.cat([x[:, pos_a:pos_a + L], x[:, pos_b:pos_b + L]], dim=1).contiguous()


def unshard_rows(parts, world_size: int):
    """Inverse of shard_rows: parts[r] is rank r's [B, 2L, ...] tensor."""
    import torch
    L = parts[0].shape[1] // 2
    S = 2 * world_size * L
    full = torch.empty((parts[0].shape[0], S) + tuple(parts[0].shape[2:]), dtype=parts[0].dtype,
                       device=parts[0].device)
    for r, part in enumerate(parts):
        pos_a, pos_b, _ = zigzag_chunks(S, world_size, r)
        full[:, pos_a:pos_a + L] = part[:, :L]
        full[:, pos_b:pos_b + L] = part[:, L:]
    return full


def gather_sequence(x_local, world_size: int, group=None):
    """All-gather of every rank's [B, 2L, H, D] shard into the whole sequence
    [B, S, H, D] in token order, in this rank's memory.

    With B == 1 each chunk of the output is a contiguous slice, and the two
    all-gathers write the chunks straight into place. With B > 1 the chunks
    are gathered into a staging buffer and then placed."""
    import torch
    import torch.distributed as dist
    B, L2 = x_local.shape[0], x_local.shape[1]
    L = L2 // 2
    S = 2 * world_size * L
    tail = tuple(x_local.shape[2:])
    if world_size == 1:
        return unshard_rows([x_local], 1)
    full = torch.empty((B, S) + tail, dtype=x_local.dtype, device=x_local.device)
    first = x_local[:, :L].contiguous()
    second = x_local[:, L:].contiguous()
    if B == 1:
        outs_a = [full[:, r * L:(r + 1) * L] for r in range(world_size)]
        outs_b = [full[:, (2 * world_size - 1 - r) * L:(2 * world_size - r) * L] for r in range(world_size)]
        dist.all_gather(outs_a, first, group=group)
        dist.all_gather(outs_b, second, group=group)
        return full
    outs_a = [torch.empty_like(first) for _ in range(world_size)]
    outs_b = [torch.empty_like(second) for _ in range(world_size)]
    dist.all_gather(outs_a, first, group=group)
    dist.all_gather(outs_b, second, group=group)
    return unshard_rows([torch.cat([a, b], dim=1) for a, b in zip(outs_a, outs_b)], world_size)


def cp_prefill(q_local, k_local, v_local, world_size: int, rank: int, group=None, lse=None,
               rope_theta: float = 500000.0, attn=None):
    """One rank's context-parallel prefill. q_local [B, 2L, Hq, D] and
    k_local / v_local [B, 2L, Hkv, D] are the rank's zigzag shards (see
    shard_rows). Returns (out_local [B, 2L, Hq, D], lse_local or None).

    attn(q, k_full, v_full, pos_a, split, pos_b, lse, rope_theta) computes the
    local rows; it defaults to the library's llama_attn_prefill_cp."""
    L = q_local.shape[1] // 2
    S = 2 * world_size * L
    pos_a, pos_b, _ = zigzag_chunks(S, world_size, rank)
    k_full = gather_sequence(k_local, world_size, group)
    v_full = gather_sequence(v_local, world_size, group)
    if attn is None:
        from . import llama_attn_prefill_cp
        return llama_attn_prefill_cp(q_local, k_full, v_full, pos_a, L, pos_b, lse=lse, rope_theta=rope_theta)
    return attn(q_local, k_full, v_full, pos_a, L, pos_b, lse, rope_theta)
