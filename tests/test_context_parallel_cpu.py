"""Host logic of context-parallel prefill, on CPU.

The zigzag split is pinned by hand-worked chunk positions and by its purpose
(equal causal work on every rank); the shard / unshard pair is checked as a
permutation; and two gloo ranks run cp_prefill with the float64 oracle as the
attention step, so that the all-gather assembly and the chunk positions are
checked against the oracle's result for the same rows of the whole sequence.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from gqa_attention_rope_b200 import context_parallel as CP


def test_zigzag_hand_worked():
    # S = 1024 over 2 ranks: 4 chunks of 256; rank 0 gets chunks 0 and 3, rank 1 chunks 1 and 2
    assert CP.zigzag_chunks(1024, 2, 0) == (0, 768, 256)
    assert CP.zigzag_chunks(1024, 2, 1) == (256, 512, 256)
    # one rank: the two halves in order
    assert CP.zigzag_chunks(256, 1, 0) == (0, 128, 128)
    # 128K over 8 ranks: 16 chunks of 8192
    assert CP.zigzag_chunks(131072, 8, 3) == (3 * 8192, 12 * 8192, 8192)


@pytest.mark.parametrize("S,N", [(1000, 2), (1024, 3), (0, 1), (256, 0)])
def test_zigzag_rejects(S, N):
    with pytest.raises(ValueError):
        CP.zigzag_chunks(S, N, 0)


@pytest.mark.parametrize("N", [1, 2, 4, 8])
def test_zigzag_balances_causal_work(N):
    S = 2 * N * 128 * 3
    work = []
    covered = np.zeros(S, dtype=np.int64)
    for r in range(N):
        pos_a, pos_b, L = CP.zigzag_chunks(S, N, r)
        rows = np.r_[pos_a:pos_a + L, pos_b:pos_b + L]
        covered[rows] += 1
        work.append(int(np.sum(rows + 1)))  # query at position P sees P + 1 keys
    assert np.all(covered == 1), "chunks must tile the sequence exactly once"
    assert len(set(work)) == 1, f"unequal causal work {work}"


def test_shard_unshard_roundtrip():
    x = torch.arange(2 * 1024 * 3, dtype=torch.float32).reshape(2, 1024, 3)
    parts = [CP.shard_rows(x, 2, r) for r in range(2)]
    assert parts[0].shape == (2, 512, 3)
    assert torch.equal(parts[0][:, :256], x[:, :256]) and torch.equal(parts[0][:, 256:], x[:, 768:])
    assert torch.equal(CP.unshard_rows(parts, 2), x)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _oracle_attn(O):
    def attn(q_local, k_full, v_full, pos_a, split, pos_b, lse, rope_theta):
        B, Sq, Hq, D = q_local.shape
        S = k_full.shape[1]
        q_full = torch.zeros(B, S, Hq, D, dtype=q_local.dtype)
        pos = np.r_[pos_a:pos_a + split, pos_b:pos_b + (Sq - split)]
        q_full[:, torch.from_numpy(pos)] = q_local
        rows = (np.arange(B)[:, None] * S + pos[None, :]).reshape(-1)
        out = O.prefill(q_full, k_full, v_full, None, rope_theta, rows=rows)
        return out.reshape(B, Sq, Hq, D), None
    return attn


def _worker(rank, world, port, result_dir, B):
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    from gqa_attention_rope_b200 import context_parallel as CPw
    from gqa_attention_rope_b200 import workloads as W
    from oracle import oracle as O

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = W.custom_prefill(41 + B, B, 2 * world * 128, 4, 2, 16, "f32", None)
        inp = W.make_prefill_inputs(w)
        q_l, k_l, v_l = (CPw.shard_rows(inp[n], world, rank) for n in ("q", "k", "v"))
        out_l, _ = CPw.cp_prefill(q_l, k_l, v_l, world, rank, attn=_oracle_attn(O), rope_theta=w.rope_theta)
        parts = [torch.zeros_like(torch.from_numpy(out_l)) for _ in range(world)]
        dist.all_gather(parts, torch.from_numpy(np.ascontiguousarray(out_l)))
        if rank == 0:
            got = CPw.unshard_rows(parts, world).numpy()
            ref = O.prefill(inp["q"], inp["k"], inp["v"], None, w.rope_theta)
            np.save(os.path.join(result_dir, f"cp_{B}.npy"), np.array([float(np.abs(got - ref).max())]))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("B", [1, 2])
def test_cp_prefill_two_gloo_ranks(tmp_path, B):
    world = 2
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path), B), nprocs=world, join=True,
                       start_method="spawn")
    err = np.load(os.path.join(tmp_path, f"cp_{B}.npy"))[0]
    # same float64 arithmetic on the same rows: the assembly must be exact
    assert err == 0.0, f"context-parallel assembly differs from the whole-sequence oracle by {err}"
