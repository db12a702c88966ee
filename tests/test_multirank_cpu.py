"""World-size-2 tests of the multi-rank host logic on CPU (gloo).

The prefill shards into independent (batch row, KV group) units and the decode
into independent sequences; no data-path collective is needed. These tests run
two gloo ranks that each compute their shard with the float64 oracle, gather
the shards and check the assembly against the unsharded result, and check the
max-over-ranks timing reduction the bench uses.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, result_dir):
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    from gqa_attention_rope_b200 import shard_units
    from gqa_attention_rope_b200 import workloads as W
    from oracle import oracle as O

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # prefill: units are (b, g) pairs; each rank computes the query heads of its units
        w = W.custom_prefill(31, 2, 96, 8, 2, 16, "f32", (10, 50))
        inp = W.make_prefill_inputs(w)
        G = w.Hq // w.Hkv
        units = list(shard_units(w.B * w.Hkv, world, rank))
        part = torch.zeros(w.B, w.S, w.Hq, w.D, dtype=torch.float64)
        for u in units:
            b, g = divmod(u, w.Hkv)
            heads = slice(g * G, (g + 1) * G)
            sub = O.prefill(inp["q"][b:b + 1, :, heads], inp["k"][b:b + 1, :, g:g + 1],
                            inp["v"][b:b + 1, :, g:g + 1],
                            None if inp["doc_offsets"] is None else
                            _row_offsets(inp["doc_offsets"], b, w.S))
            part[b, :, heads] = torch.from_numpy(sub[0])
        dist.all_reduce(part)  # disjoint shards: the sum assembles them
        # decode: units are sequences
        wd = W.custom_decode(32, 5, 8, 2, 16, 40, (1, 40))
        dinp = W.make_decode_inputs(wd, poison=False)
        dpart = torch.zeros(wd.B, wd.Hq, wd.D, dtype=torch.float64)
        seqs = list(shard_units(wd.B, world, rank))
        if seqs:
            sl = slice(seqs[0], seqs[-1] + 1)
            dpart[sl] = torch.from_numpy(O.decode(dinp["q"][sl], dinp["kcache"][sl], dinp["vcache"][sl],
                                                  dinp["cache_lens"][sl]))
        dist.all_reduce(dpart)
        # timing reduction: max over ranks
        t = torch.tensor([10.0 + rank], dtype=torch.float64)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        if rank == 0:
            full = O.prefill(inp["q"], inp["k"], inp["v"], inp["doc_offsets"])
            dfull = O.decode(dinp["q"], dinp["kcache"], dinp["vcache"], dinp["cache_lens"])
            np.save(os.path.join(result_dir, "ok.npy"), np.array([
                float(np.abs(part.numpy() - full).max()),
                float(np.abs(dpart.numpy() - dfull).max()),
                float(t.item())]))
    finally:
        dist.destroy_process_group()


def _row_offsets(offs, b, S):
    o = offs.to(torch.int64)
    sel = o[(o >= b * S) & (o <= (b + 1) * S)] - b * S
    return sel.to(torch.int32)


def test_two_rank_sharding_assembles_unsharded_result(tmp_path):
    port = _free_port()
    mp.start_processes(_worker, args=(2, port, str(tmp_path)), nprocs=2, join=True, start_method="spawn")
    perr, derr, tmax = np.load(tmp_path / "ok.npy")
    assert perr <= 1e-12 and derr <= 1e-12
    assert tmax == 11.0
