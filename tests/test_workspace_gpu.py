"""GPU tests of the caller-memory prefill entry points, the caller-owned RoPE
table, and the KV-group (tensor-parallel head) split.

* llama_attn_prefill_ws / llama_attn_prefill_cp_ws run the same kernels as the
  convenience calls on caller memory: their outputs, LSE and cache rows must be
  bit-identical, and a call must allocate no device memory (free memory is
  read before and after a call on a shape larger than any before it).
* llama_attn_rope_table_build against the closed form cos / sin of
  p * base^(-2k/D) evaluated in float64 (the table is float32: one rounding).
* Per-rank head slices of one workload (kv_group_parallel) run through the
  library reassemble the whole prefill bit for bit: each query head's
  arithmetic is the same whichever rank runs it.
"""
import numpy as np
import pytest
import torch

import gqa_attention_rope_b200 as la
from gqa_attention_rope_b200 import build as labuild
from gqa_attention_rope_b200 import kv_group_parallel as KG
from gqa_attention_rope_b200 import workloads as W
from oracle import oracle as O

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    labuild.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    la.lib()
    la.llama_attn_get_device_error()
    yield
    assert la.llama_attn_get_device_error() == 0


def _inputs(seed, B, S, Hq, Hkv, docs):
    w = W.custom_prefill(seed, B, S, Hq, Hkv, 128, "bf16", docs)
    inp = W.make_prefill_inputs(w)
    dev = {n: inp[n].cuda() for n in ("q", "k", "v")}
    dev["doc_offsets"] = inp["doc_offsets"].cuda() if inp["doc_offsets"] is not None else None
    return w, inp, dev


def _workspace(B, S, Hkv):
    n = la.llama_attn_prefill_workspace_size(B, S, Hkv)
    assert n > 0
    return torch.empty(n, dtype=torch.uint8, device="cuda")


def test_rope_table_matches_closed_form():
    maxpos, D, base = 5000, 128, 500000.0
    tab = la.llama_attn_rope_table_build(maxpos, D, base)
    torch.cuda.synchronize()
    got = tab.cpu().numpy().astype(np.float64)
    freqs = O.rope_freqs(D, base)  # theta_k = base^(-2k/D), float64
    ang = np.arange(maxpos, dtype=np.float64)[:, None] * freqs[None, :]
    err_c = np.abs(got[:, :, 0] - np.cos(ang)).max()
    err_s = np.abs(got[:, :, 1] - np.sin(ang)).max()
    assert max(err_c, err_s) <= 2.0 ** -24, (err_c, err_s)  # one float32 rounding of a value in [-1, 1]


@pytest.mark.parametrize("B,S,Hq,Hkv,docs", [
    (2, 700, 8, 2, (60, 300)),
    (1, 333, 6, 2, None),
    (1, 5, 4, 1, None),
])
def test_prefill_ws_equals_convenience_call(B, S, Hq, Hkv, docs):
    w, inp, d = _inputs(91 + S, B, S, Hq, Hkv, docs)
    tab = la.llama_attn_rope_table_build(S, 128, w.rope_theta)
    ws = _workspace(B, S, Hkv)
    ws.fill_(0xAB)  # contents need no initialisation
    lse_a = torch.empty(B, S, Hq, dtype=torch.float32, device="cuda")
    lse_b = torch.empty_like(lse_a)
    kc_a = torch.zeros(B, Hkv, S + 3, 128, dtype=torch.bfloat16, device="cuda")
    vc_a, kc_b, vc_b = torch.zeros_like(kc_a), torch.zeros_like(kc_a), torch.zeros_like(kc_a)
    out_a, _ = la.llama_attn_prefill_ex(d["q"], d["k"], d["v"], lse=lse_a, doc_offsets=d["doc_offsets"],
                                        kcache=kc_a, vcache=vc_a)
    out_b, _ = la.llama_attn_prefill_ws(d["q"], d["k"], d["v"], tab, ws, lse=lse_b, doc_offsets=d["doc_offsets"],
                                        kcache=kc_b, vcache=vc_b)
    torch.cuda.synchronize()
    assert torch.equal(out_a, out_b)
    assert torch.equal(lse_a, lse_b)
    assert torch.equal(kc_a, kc_b) and torch.equal(vc_a, vc_b)


def test_prefill_cp_ws_equals_convenience_call():
    S, L = 1024, 256
    w, inp, d = _inputs(93, 1, S, 8, 2, None)
    q_local = torch.cat([d["q"][:, 0:L], d["q"][:, 768:768 + L]], dim=1).contiguous()
    tab = la.llama_attn_rope_table_build(S, 128, w.rope_theta)
    ws = _workspace(1, S, 2)
    a, _ = la.llama_attn_prefill_cp(q_local, d["k"], d["v"], 0, L, 768)
    b, _ = la.llama_attn_prefill_cp_ws(q_local, d["k"], d["v"], 0, L, 768, tab, ws)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def test_prefill_ws_allocates_nothing():
    # warm up every kernel the call launches (module and function loading may allocate)
    w, inp, d = _inputs(95, 1, 300, 8, 2, (50, 200))
    tab = la.llama_attn_rope_table_build(4096, 128, w.rope_theta)
    la.llama_attn_prefill_ws(d["q"], d["k"], d["v"], tab, _workspace(1, 300, 2), doc_offsets=d["doc_offsets"])
    torch.cuda.synchronize()
    # a larger shape than any call before, every buffer made up front
    w2, inp2, d2 = _inputs(96, 2, 4000, 8, 2, (100, 3000))
    ws2 = _workspace(2, 4000, 2)
    out2 = torch.empty_like(d2["q"])
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    la.llama_attn_prefill_ws(d2["q"], d2["k"], d2["v"], tab, ws2, out=out2, doc_offsets=d2["doc_offsets"])
    torch.cuda.synchronize()
    free1 = torch.cuda.mem_get_info()[0]
    assert free1 == free0, f"device free memory changed by {free0 - free1} bytes"
    ref = la.llama_attn_prefill(d2["q"], d2["k"], d2["v"], doc_offsets=d2["doc_offsets"])
    torch.cuda.synchronize()
    assert torch.equal(out2, ref)


@pytest.mark.parametrize("N", [2, 4, 8])
def test_kv_group_shards_reassemble_whole_prefill(N):
    B, S, Hq, Hkv = 2, 640, 32, 8
    w, inp, d = _inputs(97, B, S, Hq, Hkv, (100, 400))
    whole = la.llama_attn_prefill(d["q"], d["k"], d["v"], doc_offsets=d["doc_offsets"])
    parts = []
    for r in range(N):  # the ranks' steps, one after another on this GPU
        ql, kl, vl = KG.shard_qkv(d["q"], d["k"], d["v"], N, r)
        parts.append(KG.tp_prefill(ql, kl, vl, d["doc_offsets"]))
    torch.cuda.synchronize()
    assert torch.equal(torch.cat(parts, dim=2), whole)
