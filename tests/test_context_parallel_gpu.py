"""GPU parity of llama_attn_prefill_cp, the per-rank step of context-parallel
prefill, through the C ABI.

This machine has one GPU, so the ranks of a zigzag split run one after another
on it; each gets the whole sequence's K and V (what the all-gather delivers).
Two checks: against the float64 oracle (bf16 tolerance 1.5e-2, as for the
prefill), and bit for bit against llama_attn_prefill over the whole sequence,
since a query tile at a given global position goes through the same
arithmetic in both calls.
"""
import numpy as np
import pytest
import torch

import gqa_attention_rope_b200 as la
from gqa_attention_rope_b200 import build as labuild
from gqa_attention_rope_b200 import context_parallel as CP
from gqa_attention_rope_b200 import workloads as W
from guards import check_guard, guarded
from oracle import oracle as O

pytestmark = pytest.mark.gpu

TOL_BF16 = 1.5e-2


@pytest.fixture(scope="module", autouse=True)
def _lib():
    labuild.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    la.lib()
    la.llama_attn_get_device_error()
    yield
    assert la.llama_attn_get_device_error() == 0


def _inputs(seed, B, S, Hq, Hkv):
    w = W.custom_prefill(seed, B, S, Hq, Hkv, 128, "bf16", None)
    inp = W.make_prefill_inputs(w)
    return w, inp, tuple(inp[n].cuda() for n in ("q", "k", "v"))


@pytest.mark.parametrize("N,B,S,Hq,Hkv", [(2, 1, 1024, 8, 2), (4, 2, 1024, 4, 1), (3, 1, 768, 6, 2)])
def test_zigzag_ranks_match_whole_prefill(N, B, S, Hq, Hkv):
    w, inp, (q, k, v) = _inputs(200 + N, B, S, Hq, Hkv)
    ref_out, ref_lse = la.llama_attn_prefill_ex(q, k, v, lse=torch.empty(B, S, Hq, device="cuda"))
    outs, lses = [], []
    for r in range(N):
        pos_a, pos_b, L = CP.zigzag_chunks(S, N, r)
        q_l = CP.shard_rows(q, N, r)
        lse_buf, lse_l = guarded((B, 2 * L, Hq), torch.float32)
        lse_l.fill_(float("nan"))
        out_buf, out_l = guarded(q_l.shape)
        la.llama_attn_prefill_cp(q_l, k, v, pos_a, L, pos_b, out=out_l, lse=lse_l)
        outs.append(out_l)
        lses.append(lse_l)
        bufs = (out_buf, lse_buf)
        torch.cuda.synchronize()
        check_guard(bufs[0])
        check_guard(bufs[1], what="lse")
    got = CP.unshard_rows(outs, N)
    assert torch.equal(got, ref_out), "context-parallel rows differ from the whole-sequence prefill"
    assert torch.equal(CP.unshard_rows(lses, N), ref_lse)
    ref = O.prefill(inp["q"], inp["k"], inp["v"], None, w.rope_theta)
    err = np.abs(got.float().cpu().numpy() - ref).max()
    assert err <= TOL_BF16, f"max abs err {err}"


@pytest.mark.parametrize("Skv,pos_a,split,pos_b,Sq", [
    (1000, 0, 256, 768, 488),    # ragged second chunk ending at the sequence end
    (1000, 384, 384, 0, 384),    # one chunk only (q_split = Sq), not at the start
    (1000, 0, 0, 640, 360),      # second chunk only (q_split = 0)
    (640, 512, 128, 0, 256),     # chunks out of order
])
def test_chunks_match_rows_of_whole_prefill(Skv, pos_a, split, pos_b, Sq):
    B, Hq, Hkv = 1, 8, 2
    w, inp, (q, k, v) = _inputs(300 + Skv + pos_a, B, Skv, Hq, Hkv)
    full = la.llama_attn_prefill(q, k, v)
    rows = np.r_[pos_a:pos_a + split, pos_b:pos_b + (Sq - split)]
    idx = torch.from_numpy(rows).cuda()
    q_l = q[:, idx].contiguous()
    buf, out_l = guarded(q_l.shape)
    la.llama_attn_prefill_cp(q_l, k, v, pos_a, split, pos_b, out=out_l)
    torch.cuda.synchronize()
    check_guard(buf)
    assert torch.equal(out_l, full[:, idx])
    ref = O.prefill(inp["q"], inp["k"], inp["v"], None, w.rope_theta, rows=rows)
    err = np.abs(out_l[0].float().cpu().numpy() - ref).max()
    assert err <= TOL_BF16, f"max abs err {err}"


@pytest.mark.parametrize("pos_a,split,pos_b,Sq", [
    (64, 128, 512, 256),     # position not a multiple of 128
    (0, 100, 512, 256),      # split not a multiple of 128
    (0, 128, 900, 256),      # second chunk runs past Skv
    (640, 128, 0, 128),      # first chunk runs past Skv
    (0, 384, 0, 256),        # split > Sq
])
def test_rejects_bad_chunks(pos_a, split, pos_b, Sq):
    _, _, (q, k, v) = _inputs(5, 1, 640, 4, 1)
    q_l = q[:, :Sq].contiguous()
    with pytest.raises(la.LlamaAttnError):
        la.llama_attn_prefill_cp(q_l, k, v, pos_a, split, pos_b)


def test_128k_rank_matches_whole_prefill_rows():
    """The 128K single-document workload (Hq 32, Hkv 8), rank 3 of 8: its
    16384 query rows equal the whole-sequence prefill's rows bit for bit."""
    w = W.LONG_128K
    inp = W.make_prefill_inputs(w)
    q, k, v = (inp[n].cuda() for n in ("q", "k", "v"))
    full = la.llama_attn_prefill(q, k, v)
    N, r = 8, 3
    pos_a, pos_b, L = CP.zigzag_chunks(w.S, N, r)
    out_l, _ = la.llama_attn_prefill_cp(CP.shard_rows(q, N, r), k, v, pos_a, L, pos_b)
    torch.cuda.synchronize()
    assert torch.equal(out_l, CP.shard_rows(full, N, r))
