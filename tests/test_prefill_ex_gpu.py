"""GPU parity of llama_attn_prefill_ex: the log-sum-exp output, the KV-cache
append, and a prefill followed by a decode that continues from the cache it
wrote, all against the float64 oracle.

LSE tolerance: the scores differ from the oracle's by the bf16 rounding of the
rotated q and k (a few 1e-3 at the tails for unit-variance inputs) and the
exponential approximations (relative 7.5e-5 at most); a log-sum-exp moves by
at most the largest score error, so 1e-2 absolute bounds it with margin.
Cache tolerance: the kernel rotates in fp32 and rounds once to bf16, so each
element is within one bf16 ulp of the float64 rotation rounded to bf16.
"""
import numpy as np
import pytest
import torch

import gqa_attention_rope_b200 as la
from gqa_attention_rope_b200 import build as labuild
from gqa_attention_rope_b200 import workloads as W
from guards import check_guard, guarded
from oracle import oracle as O

pytestmark = pytest.mark.gpu

TOL_BF16 = 1.5e-2
TOL_LSE = 1e-2


@pytest.fixture(scope="module", autouse=True)
def _lib():
    labuild.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    la.lib()
    la.llama_attn_get_device_error()
    yield
    assert la.llama_attn_get_device_error() == 0


def bf16_ulp(x: np.ndarray) -> np.ndarray:
    """Spacing of bf16 numbers at |x| (8 significant bits)."""
    e = np.floor(np.log2(np.maximum(np.abs(x), 2.0 ** -126)))
    return 2.0 ** (e - 7)


@pytest.mark.parametrize("B,S,Hq,Hkv,docs", [
    (2, 700, 8, 2, (60, 300)),
    (1, 333, 6, 2, None),
    (1, 260, 4, 1, (1, 3)),
])
def test_prefill_ex_lse_and_output(B, S, Hq, Hkv, docs):
    w = W.custom_prefill(31 + S, B, S, Hq, Hkv, 128, "bf16", docs)
    inp = W.make_prefill_inputs(w)
    q, k, v = (inp[n].cuda() for n in ("q", "k", "v"))
    offs = inp["doc_offsets"].cuda() if inp["doc_offsets"] is not None else None
    lse_buf, lse = guarded((B, S, Hq), torch.float32)
    lse.fill_(float("nan"))
    out_buf, out = guarded(q.shape)
    la.llama_attn_prefill_ex(q, k, v, out=out, lse=lse, doc_offsets=offs)
    plain = la.llama_attn_prefill(q, k, v, doc_offsets=offs)
    torch.cuda.synchronize()
    check_guard(out_buf)
    check_guard(lse_buf, what="lse")
    assert torch.equal(out, plain), "prefill_ex output differs from prefill"
    ref_out, ref_lse = O.prefill_lse(inp["q"], inp["k"], inp["v"], inp["doc_offsets"])
    got_lse = lse.cpu().numpy().astype(np.float64)
    assert np.all(np.isfinite(got_lse))
    err = np.abs(got_lse - ref_lse).max()
    assert err <= TOL_LSE, f"lse max abs err {err}"
    oerr = np.abs(out.float().cpu().numpy() - ref_out).max()
    assert oerr <= TOL_BF16, f"out max abs err {oerr}"


@pytest.mark.parametrize("docs", [None, (50, 200)])
def test_kv_cache_append(docs):
    B, S, Hq, Hkv, Lmax = 2, 450, 8, 2, 512
    w = W.custom_prefill(77, B, S, Hq, Hkv, 128, "bf16", docs)
    inp = W.make_prefill_inputs(w)
    q, k, v = (inp[n].cuda() for n in ("q", "k", "v"))
    offs = inp["doc_offsets"].cuda() if inp["doc_offsets"] is not None else None
    canary = 7.0
    kc_buf, kc = guarded((B, Hkv, Lmax, 128), fill=canary)
    vc_buf, vc = guarded((B, Hkv, Lmax, 128), fill=canary)
    la.llama_attn_prefill_ex(q, k, v, doc_offsets=offs, kcache=kc, vcache=vc)
    torch.cuda.synchronize()
    check_guard(kc_buf, fill=canary, what="kcache")
    check_guard(vc_buf, fill=canary, what="vcache")
    kc_h, vc_h = kc.cpu(), vc.cpu()
    # values: copied bit for bit; rows past S untouched
    assert torch.equal(vc_h[:, :, :S], inp["v"].permute(0, 2, 1, 3))
    assert torch.all(kc_h[:, :, S:] == canary) and torch.all(vc_h[:, :, S:] == canary)
    # keys: the float64 rotation at each token's document position
    _, pos = O.doc_layout(inp["doc_offsets"], B, S)
    krot = O.rope_rotate(inp["k"].reshape(B * S, Hkv, 128), pos.astype(np.float64), w.rope_theta)
    krot = krot.reshape(B, S, Hkv, 128).transpose(0, 2, 1, 3)
    ref = torch.from_numpy(krot).to(torch.bfloat16).double().numpy()
    got = kc_h[:, :, :S].double().numpy()
    assert np.all(np.abs(got - ref) <= bf16_ulp(ref) + 1e-30)


def test_prefill_then_decode_continues_from_the_cache():
    B, S, Hq, Hkv, Lmax = 2, 700, 16, 2, 1024
    w = W.custom_prefill(91, B, S, Hq, Hkv, 128, "bf16", None)
    inp = W.make_prefill_inputs(w)
    q, k, v = (inp[n].cuda() for n in ("q", "k", "v"))
    kc = torch.zeros((B, Hkv, Lmax, 128), dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    la.llama_attn_prefill_ex(q, k, v, kcache=kc, vcache=vc)
    gen = torch.Generator().manual_seed(92)
    q_new = torch.randn(B, Hq, 128, generator=gen).to(torch.bfloat16)
    lens = torch.full((B,), S, dtype=torch.int32)
    out = la.llama_attn_decode(q_new.cuda(), kc, vc, lens.cuda())
    torch.cuda.synchronize()
    # oracle: keys rotated in float64 at positions 0..S-1, the new query at S
    krot = O.rope_rotate(inp["k"].reshape(B * S, Hkv, 128), np.tile(np.arange(S, dtype=np.float64), B),
                         w.rope_theta).reshape(B, S, Hkv, 128).transpose(0, 2, 1, 3)
    ref = O.decode(q_new, torch.from_numpy(np.ascontiguousarray(krot)),
                   inp["v"].permute(0, 2, 1, 3).contiguous(), lens, w.rope_theta)
    err = np.abs(out.float().cpu().numpy() - ref).max()
    assert err <= TOL_BF16, f"decode after prefill max abs err {err}"
