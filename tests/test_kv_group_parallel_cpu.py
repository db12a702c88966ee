"""Host logic of the KV-group (tensor-parallel head) split, on CPU.

The head ranges are pinned by hand-worked values and by their purpose (every
query head lands on the rank of the KV head it reads, every head exactly
once); two gloo ranks then shard one workload with the product helpers, run
their heads' attention with the float64 oracle as the attention step, and
all-gather the heads; the assembly must equal the oracle's unsharded result
exactly (each head's arithmetic does not depend on the others).
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from gqa_attention_rope_b200 import kv_group_parallel as KG


def test_head_ranges_hand_worked():
    # 405B head layout (128 query heads, 8 KV heads) over 8 ranks: one KV head and 16 query heads each
    assert KG.kv_group_heads(128, 8, 8, 0) == (0, 16, 0, 1)
    assert KG.kv_group_heads(128, 8, 8, 7) == (112, 128, 7, 8)
    # 8B layout (32 / 8) over 2 ranks
    assert KG.kv_group_heads(32, 8, 2, 1) == (16, 32, 4, 8)
    assert KG.kv_group_heads(32, 8, 1, 0) == (0, 32, 0, 8)


@pytest.mark.parametrize("Hq,Hkv,N,r", [(32, 8, 3, 0), (32, 8, 16, 0), (32, 6, 2, 0), (32, 8, 2, 2), (32, 8, 0, 0)])
def test_head_ranges_reject(Hq, Hkv, N, r):
    with pytest.raises(ValueError):
        KG.kv_group_heads(Hq, Hkv, N, r)


@pytest.mark.parametrize("Hq,Hkv,N", [(32, 8, 1), (32, 8, 2), (32, 8, 4), (32, 8, 8), (128, 8, 8), (64, 8, 4)])
def test_every_query_head_sits_with_its_kv_head(Hq, Hkv, N):
    G = Hq // Hkv
    seen_q, seen_kv = [], []
    for r in range(N):
        hq0, hq1, hk0, hk1 = KG.kv_group_heads(Hq, Hkv, N, r)
        seen_q += list(range(hq0, hq1))
        seen_kv += list(range(hk0, hk1))
        for h in range(hq0, hq1):
            assert hk0 <= h // G < hk1, "a query head was placed away from its KV head"
    assert seen_q == list(range(Hq)) and seen_kv == list(range(Hkv))


def test_shard_qkv_slices_heads():
    q = torch.arange(2 * 3 * 8 * 4, dtype=torch.float32).reshape(2, 3, 8, 4)
    k = torch.arange(2 * 3 * 2 * 4, dtype=torch.float32).reshape(2, 3, 2, 4)
    ql, kl, vl = KG.shard_qkv(q, k, k, 2, 1)
    assert torch.equal(ql, q[:, :, 4:8]) and ql.is_contiguous()
    assert torch.equal(kl, k[:, :, 1:2]) and torch.equal(vl, k[:, :, 1:2])


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, result_dir):
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    from gqa_attention_rope_b200 import kv_group_parallel as KG
    from gqa_attention_rope_b200 import workloads as W
    from oracle import oracle as O

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = W.custom_prefill(37, 2, 80, 8, 4, 16, "f32", (5, 40))
        inp = W.make_prefill_inputs(w)
        ql, kl, vl = KG.shard_qkv(inp["q"], inp["k"], inp["v"], world, rank)

        def oracle_attn(q, k, v, offs, theta, out):
            return torch.from_numpy(O.prefill(q, k, v, offs, theta))

        out_local = KG.tp_prefill(ql, kl, vl, inp["doc_offsets"], w.rope_theta, attn=oracle_attn)
        full = KG.gather_heads(out_local, world)
        if rank == 0:
            ref = O.prefill(inp["q"], inp["k"], inp["v"], inp["doc_offsets"], w.rope_theta)
            np.save(os.path.join(result_dir, "err.npy"),
                    np.array([float(np.abs(full.numpy() - ref).max()), float(full.shape[2])]))
    finally:
        dist.destroy_process_group()


def test_two_rank_kv_group_split_assembles_unsharded_result(tmp_path):
    port = _free_port()
    mp.start_processes(_worker, args=(2, port, str(tmp_path)), nprocs=2, join=True, start_method="spawn")
    err, heads = np.load(tmp_path / "err.npy")
    assert heads == 8
    assert err == 0.0
