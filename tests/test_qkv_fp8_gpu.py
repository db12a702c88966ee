"""GPU parity of the FP8 QKV projection with RoPE and of the prefill on
pre-rotated inputs, through the C ABI, against the float64 oracle
(oracle/fp8.py, oracle/oracle.py).

Quantizer: the E4M3 codes and the scale are integer / exact results of the
same float32 quotient on both sides, so they must match bit for bit.

Projection tolerance, per output element: the kernel accumulates exact E4M3
products in fp32 on the tensor cores, applies the scale and the rotation in
fp32 and rounds once to bf16. So |got - ref| <= 2^-8 |ref| (bf16 rounding,
with margin) + 2^-16 A, where A = s_x s_w sum_k |x_k w_k| bounds the fp32
accumulation error (K <= 4096 additions of relative error 2^-24 each, about
2^-12 A in the worst case; 2^-16 A leaves room for the typical sqrt(K) growth
but catches a wrong product or a dropped K step) -- for a rotated element A is
that of its pair's two columns added.

Attention after the projection: the bf16 attention tolerance (1.5e-2).
"""
import numpy as np
import pytest
import torch

import gqa_attention_rope_b200 as la
from gqa_attention_rope_b200 import build as labuild
from gqa_attention_rope_b200 import workloads as W
from guards import check_guard, guarded
from oracle import fp8 as F
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


def _bf16(gen, shape, std=1.0):
    return (torch.randn(*shape, generator=gen) * std).to(torch.bfloat16)


@pytest.mark.parametrize("n,std,extra", [(8 * 1000, 1.0, None), (4096 * 64, 3.0, 30000.0), (8 * 7, 1e-3, None)])
def test_quantize_bit_exact(n, std, extra):
    gen = torch.Generator().manual_seed(n)
    x = _bf16(gen, (n,), std)
    if extra is not None:
        x[17] = extra           # one large value: most codes fall into the subnormal range
        x[18] = -extra / 3
    x[3] = 0.0
    codes, s = la.llama_attn_quantize_e4m3(x.cuda())
    torch.cuda.synchronize()
    ref_codes, ref_s = F.quantize_per_tensor(x.float().numpy())
    assert s.item() == float(ref_s)
    assert np.array_equal(codes.cpu().numpy(), ref_codes)


def test_quantize_zeros_and_rejects():
    codes, s = la.llama_attn_quantize_e4m3(torch.zeros(64, dtype=torch.bfloat16, device="cuda"))
    torch.cuda.synchronize()
    assert s.item() == 1.0 and int(codes.abs().sum()) == 0
    with pytest.raises(la.LlamaAttnError):
        la.llama_attn_quantize_e4m3(torch.ones(12, dtype=torch.bfloat16, device="cuda"))


def _quantized_problem(seed, M, d_model, Hq, Hkv, w_std=None):
    """Oracle-quantized X [M, d_model] and W [N, d_model] (codes and scales)."""
    gen = torch.Generator().manual_seed(seed)
    N = (Hq + 2 * Hkv) * 128
    x = _bf16(gen, (M, d_model))
    w = _bf16(gen, (N, d_model), w_std if w_std else d_model ** -0.5)
    xc, sx = F.quantize_per_tensor(x.float().numpy())
    wc, sw = F.quantize_per_tensor(w.float().numpy())
    return xc, sx, wc, sw


def _gpu_projection(xc, sx, wc, sw, B, S, Hq, Hkv, offs, theta):
    """The library's projection into q, k, v tensors that sit inside canary
    guard bands; the bands are checked after the call."""
    (bq, q), (bk, k), (bv, v) = (guarded((B, S, H, 128)) for H in (Hq, Hkv, Hkv))
    la.llama_attn_qkv_fp8_rope(
        torch.from_numpy(xc).cuda(), torch.tensor([sx], dtype=torch.float32, device="cuda"),
        torch.from_numpy(wc).cuda(), torch.tensor([sw], dtype=torch.float32, device="cuda"),
        B, S, Hq, Hkv, doc_offsets=None if offs is None else offs.cuda(), rope_theta=theta, q=q, k=k, v=v)
    torch.cuda.synchronize()
    for buf, name in ((bq, "q"), (bk, "k"), (bv, "v")):
        check_guard(buf, what=name)
    return q, k, v


def _abs_sum(xc, sx, wc, sw, Hq, Hkv, rows=None):
    X = np.abs(F.e4m3_decode(xc if rows is None else xc[rows]))
    Wm = np.abs(F.e4m3_decode(wc))
    A = float(sx) * float(sw) * (X @ Wm.T)
    T = A.shape[0]
    aq = A[:, :Hq * 128].reshape(T, Hq, 128)
    ak = A[:, Hq * 128:(Hq + Hkv) * 128].reshape(T, Hkv, 128)
    av = A[:, (Hq + Hkv) * 128:].reshape(T, Hkv, 128)
    pair = lambda a: np.repeat(a[..., 0::2] + a[..., 1::2], 2, axis=-1)  # noqa: E731
    return pair(aq), pair(ak), av


def _check(got, ref, A, what):
    got = got.float().cpu().numpy().reshape(ref.shape)
    bound = 2.0 ** -8 * np.abs(ref) + 2.0 ** -16 * A.reshape(ref.shape) + 1e-30
    ratio = np.abs(got - ref) / bound
    assert np.all(np.isfinite(got)), what
    assert ratio.max() <= 1.0, f"{what}: worst error / bound = {ratio.max():.3f}"


@pytest.mark.parametrize("B,S,d_model,Hq,Hkv,docs", [
    (1, 300, 256, 4, 2, None),        # ragged token tail, two tiles of N
    (2, 200, 384, 3, 1, (20, 90)),    # odd head count: the last N tile is half empty; documents
    (1, 128, 128, 2, 2, None),        # one K step
    (3, 77, 512, 8, 2, (5, 40)),      # many short documents
])
def test_projection_matches_oracle(B, S, d_model, Hq, Hkv, docs):
    w_ = W.custom_prefill(900 + S, B, S, Hq, Hkv, 128, "bf16", docs)
    offs = W.make_prefill_inputs(w_)["doc_offsets"]
    xc, sx, wc, sw = _quantized_problem(S + d_model, B * S, d_model, Hq, Hkv)
    theta = 500000.0
    q, k, v = _gpu_projection(xc, sx, wc, sw, B, S, Hq, Hkv, offs, theta)
    torch.cuda.synchronize()
    rq, rk, rv = F.qkv_projection_rope(xc, sx, wc, sw, Hq, Hkv, 128, B, S, offs, theta)
    aq, ak, av = _abs_sum(xc, sx, wc, sw, Hq, Hkv)
    _check(q, rq, aq, "q")
    _check(k, rk, ak, "k")
    _check(v, rv, av, "v")


def test_projection_8b_shape_sampled_rows():
    """The 8B packed workload's projection (32768 tokens, d_model 4096, 32 query
    and 8 KV heads, its documents), checked on 96 sampled tokens."""
    w_ = W.PACKED_8B
    offs = W.make_prefill_inputs(w_)["doc_offsets"]
    B, S, Hq, Hkv, d_model = w_.B, w_.S, w_.Hq, w_.Hkv, 4096
    # random finite E4M3 codes (the NaN codes 0x7F / 0xFF moved to +-448) and fixed scales
    rng = np.random.default_rng(77)
    xc = rng.integers(0, 256, (B * S, d_model), dtype=np.uint8)
    wc = rng.integers(0, 256, ((Hq + 2 * Hkv) * 128, d_model), dtype=np.uint8)
    for c in (xc, wc):
        c[(c & 0x7F) == 0x7F] -= 1
    sx, sw = np.float32(2.0 ** -7), np.float32(2.0 ** -9)
    q, k, v = _gpu_projection(xc, sx, wc, sw, B, S, Hq, Hkv, offs, w_.rope_theta)
    torch.cuda.synchronize()
    rows = np.sort(np.random.default_rng(5).choice(B * S, 96, replace=False))
    Xr = F.e4m3_decode(xc[rows])
    Y = (float(sx) * float(sw)) * (Xr @ F.e4m3_decode(wc).T)
    _, pos = O.doc_layout(offs, B, S)
    p = pos[rows].astype(np.float64)
    rq = O.rope_rotate(Y[:, :Hq * 128].reshape(-1, Hq, 128), p, w_.rope_theta)
    rk = O.rope_rotate(Y[:, Hq * 128:(Hq + Hkv) * 128].reshape(-1, Hkv, 128), p, w_.rope_theta)
    rv = Y[:, (Hq + Hkv) * 128:].reshape(-1, Hkv, 128)
    aq, ak, av = _abs_sum(xc, sx, wc, sw, Hq, Hkv, rows)
    idx = torch.from_numpy(rows).cuda()
    _check(q.reshape(B * S, Hq, 128)[idx], rq, aq, "q")
    _check(k.reshape(B * S, Hkv, 128)[idx], rk, ak, "k")
    _check(v.reshape(B * S, Hkv, 128)[idx], rv, av, "v")


def test_projection_rejects():
    x = torch.zeros(128, 200, dtype=torch.uint8, device="cuda")
    w = torch.zeros(4 * 128, 200, dtype=torch.uint8, device="cuda")
    s = torch.ones(1, dtype=torch.float32, device="cuda")
    with pytest.raises(la.LlamaAttnError):  # d_model not a multiple of 128
        la.llama_attn_qkv_fp8_rope(x, s, w, s, 1, 128, 2, 1)


@pytest.mark.parametrize("B,S,Hq,Hkv,docs", [(2, 333, 8, 2, (40, 200)), (1, 700, 4, 1, None)])
def test_prefill_rotated_matches_oracle(B, S, Hq, Hkv, docs):
    """q and k rotated by the oracle (float64, rounded to bf16) through the
    pre-rotated prefill, against the oracle's attention of the un-rotated rows."""
    w_ = W.custom_prefill(600 + S, B, S, Hq, Hkv, 128, "bf16", docs)
    inp = W.make_prefill_inputs(w_)
    _, pos = O.doc_layout(inp["doc_offsets"], B, S)
    p = pos.astype(np.float64)
    qr = O.rope_rotate(inp["q"].reshape(B * S, Hq, 128), p, w_.rope_theta).reshape(B, S, Hq, 128)
    kr = O.rope_rotate(inp["k"].reshape(B * S, Hkv, 128), p, w_.rope_theta).reshape(B, S, Hkv, 128)
    qg = torch.from_numpy(qr).to(torch.bfloat16).cuda()
    kg = torch.from_numpy(kr).to(torch.bfloat16).cuda()
    offs = inp["doc_offsets"].cuda() if inp["doc_offsets"] is not None else None
    lse = torch.empty(B, S, Hq, device="cuda")
    out, _ = la.llama_attn_prefill_rotated(qg, kg, inp["v"].cuda(), lse=lse, doc_offsets=offs)
    torch.cuda.synchronize()
    ref, ref_lse = O.prefill_lse(inp["q"], inp["k"], inp["v"], inp["doc_offsets"], w_.rope_theta)
    err = np.abs(out.float().cpu().numpy() - ref).max()
    assert err <= TOL_BF16, f"max abs err {err}"
    assert np.abs(lse.cpu().numpy() - ref_lse).max() <= 1e-2


def test_fp8_projection_then_attention():
    """X -> E4M3 -> QKV projection with RoPE -> pre-rotated prefill, against the
    oracle's float64 projection of the same codes followed by its attention."""
    B, S, Hq, Hkv, d_model = 2, 400, 8, 2, 512
    w_ = W.custom_prefill(55, B, S, Hq, Hkv, 128, "bf16", (60, 250))
    offs = W.make_prefill_inputs(w_)["doc_offsets"]
    xc, sx, wc, sw = _quantized_problem(56, B * S, d_model, Hq, Hkv)
    q, k, v = _gpu_projection(xc, sx, wc, sw, B, S, Hq, Hkv, offs, w_.rope_theta)
    out, _ = la.llama_attn_prefill_rotated(q, k, v, doc_offsets=offs.cuda())
    torch.cuda.synchronize()
    uq, uk, uv = F.qkv_projection(xc, sx, wc, sw, Hq, Hkv, 128)
    ref = O.prefill(uq.reshape(B, S, Hq, 128), uk.reshape(B, S, Hkv, 128), uv.reshape(B, S, Hkv, 128), offs,
                    w_.rope_theta)
    err = np.abs(out.float().cpu().numpy() - ref).max()
    assert err <= TOL_BF16, f"max abs err {err} (std of v {float(np.std(uv)):.3f})"
