"""GPU parity of llama_attn_decode_paged: a decode whose KV cache lives in
fixed-size pages of a shared pool, addressed through a block table.

The pages of each sequence are scattered over the pool by a random
permutation; pool pages that no sequence uses hold NaN. The paged result must
equal, bit for bit, the regular decode on the same rows laid out contiguously
(the arithmetic is the same, only the addressing differs), and match the
float64 oracle within the bf16 tolerance.
"""
import ctypes

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


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def make_paged(inp, Hkv, page_size, seed):
    """Scatter the contiguous caches [B, Hkv, Lmax, D] into a page pool."""
    kc, vc, lens = inp["kcache"], inp["vcache"], inp["cache_lens"]
    B, _, Lmax, D = kc.shape
    max_blocks = (Lmax + page_size - 1) // page_size
    need = [(int(n) + page_size - 1) // page_size for n in lens]
    n_pages = sum(need) + 3
    gen = torch.Generator().manual_seed(seed)
    perm = torch.randperm(n_pages, generator=gen).tolist()
    kp = torch.full((n_pages, Hkv, page_size, D), float("nan"), dtype=torch.bfloat16)
    vp = torch.full_like(kp, float("nan"))
    table = torch.full((B, max_blocks), -1, dtype=torch.int32)
    it = iter(perm)
    for b in range(B):
        for j in range(need[b]):
            pg = next(it)
            table[b, j] = pg
            lo, hi = j * page_size, min((j + 1) * page_size, Lmax)
            kp[pg, :, :hi - lo] = kc[b, :, lo:hi]
            vp[pg, :, :hi - lo] = vc[b, :, lo:hi]
    return kp, vp, table, n_pages, max_blocks


@pytest.mark.parametrize("page_size,lens", [
    (64, [1, 63, 64, 65, 1000, 2048]),
    (256, [2048, 777, 1, 256]),
])
def test_paged_decode(page_size, lens):
    labuild.build()
    lib = la.lib()
    la.llama_attn_get_device_error()
    B, Hq, Hkv, Lmax = len(lens), 16, 2, 2048
    w = W.custom_decode(55 + page_size, B, Hq, Hkv, 128, Lmax, (1, Lmax))
    inp = W.make_decode_inputs(w, poison=True, lens=lens)
    kp, vp, table, n_pages, max_blocks = make_paged(inp, Hkv, page_size, 7)
    q, lens_d = inp["q"].cuda(), inp["cache_lens"].cuda()
    kp, vp, table = kp.cuda(), vp.cuda(), table.cuda()
    ws_bytes = lib.llama_attn_decode_workspace_size(B, Hq, max_blocks * page_size, 128)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    buf, out = guarded(q.shape)
    st = lib.llama_attn_decode_paged(_p(q), _p(kp), _p(vp), _p(table), _p(lens_d), _p(out), B, Hq, Hkv, 128,
                                     page_size, max_blocks, n_pages, ctypes.c_float(w.rope_theta), _p(ws), ws_bytes,
                                     ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0
    torch.cuda.synchronize()
    check_guard(buf)
    # the Python binding's wrapper makes the same call
    out_py = la.llama_attn_decode_paged(q, kp, vp, table, lens_d, rope_theta=w.rope_theta)
    ref_gpu = la.llama_attn_decode(q, inp["kcache"].cuda(), inp["vcache"].cuda(), lens_d)
    torch.cuda.synchronize()
    assert torch.equal(out, ref_gpu), "paged decode differs from contiguous decode"
    assert torch.equal(out_py, out), "binding wrapper differs from the direct call"
    ref = O.decode(inp["q"], inp["kcache"], inp["vcache"], inp["cache_lens"], w.rope_theta)
    err = np.abs(out.float().cpu().numpy() - ref).max()
    assert err <= TOL_BF16, f"max abs err {err}"
    assert la.llama_attn_get_device_error() == 0


def test_paged_decode_bad_block_id_sets_device_error():
    labuild.build()
    lib = la.lib()
    la.llama_attn_get_device_error()
    B, Hq, Hkv, page_size = 1, 8, 1, 64
    q = torch.zeros(B, Hq, 128, dtype=torch.bfloat16, device="cuda")
    kp = torch.zeros(2, Hkv, page_size, 128, dtype=torch.bfloat16, device="cuda")
    vp = torch.zeros_like(kp)
    table = torch.tensor([[0, 5]], dtype=torch.int32, device="cuda")  # page 5 does not exist
    lens = torch.tensor([100], dtype=torch.int32, device="cuda")
    out = torch.empty_like(q)
    ws_bytes = lib.llama_attn_decode_workspace_size(B, Hq, 2 * page_size, 128)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    st = lib.llama_attn_decode_paged(_p(q), _p(kp), _p(vp), _p(table), _p(lens), _p(out), B, Hq, Hkv, 128, page_size,
                                     2, 2, ctypes.c_float(5e5), _p(ws), ws_bytes,
                                     ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0
    assert la.llama_attn_get_device_error() == la.DEVERR_BLOCK_TABLE
    assert torch.isfinite(out.float()).all()
