"""GPU parity: the CUDA library, called through its C ABI, against the float64
oracle on the same seeded inputs.

Tolerances (max-abs error), as the specification states them: 1e-5 for the
fp32 path, 1.5e-2 for the bf16 paths (fp32 accumulation).
"""
import json
import os

import numpy as np
import pytest
import torch

import gqa_attention_rope_b200 as la
from gqa_attention_rope_b200 import build as labuild
from gqa_attention_rope_b200 import workloads as W
from guards import check_guard, guarded
from oracle import oracle as O

pytestmark = pytest.mark.gpu

TOL_F32 = 1e-5
TOL_BF16 = 1.5e-2


@pytest.fixture(scope="module", autouse=True)
def _lib():
    labuild.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    la.lib()
    la.llama_attn_get_device_error()  # start from a clear error word
    yield
    assert la.llama_attn_get_device_error() == 0


def report(got: np.ndarray, ref: np.ndarray, tol: float, what: str, rows=None):
    """Max-abs error against the oracle; the worst element, its location and
    value are printed and, with LLAMA_ATTN_PARITY_LOG set, appended to that
    file as one JSON line (the margin to the tolerance is then on record)."""
    got64 = got.astype(np.float64)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    err = np.abs(got64 - ref)
    worst = float(err.max())
    loc = np.unravel_index(int(err.argmax()), err.shape)
    log_parity(what, worst, loc, ref, tol, rows)
    assert worst <= tol, f"{what}: max abs err {worst:.3e} at {loc} (ref {ref[loc]:.4f}) > {tol}"
    return worst


def log_parity(what, worst, loc, ref, tol, rows=None):
    loc = tuple(int(x) for x in loc)
    where = {"index": loc, "ref": float(ref[loc]), "abs_ref_max": float(np.abs(ref).max())}
    if rows is not None:
        where["token"] = int(rows[loc[0]])
    rec = {"case": what, "max_abs_err": worst, "tol": tol, "margin": tol - worst, **where}
    print(json.dumps(rec))
    path = os.environ.get("LLAMA_ATTN_PARITY_LOG")
    if path:
        with open(path, "a") as f:
            f.write(json.dumps(rec) + "\n")


def to_dev(x):
    return None if x is None else x.cuda()


# ---------------------------------------------------------------- prefill fp32

def test_prefill_f32_tiny_config():
    w = W.TINY_F32
    inp = W.make_prefill_inputs(w)
    out = la.llama_attn_prefill_f32(*(to_dev(inp[n]) for n in ("q", "k", "v")), rope_theta=w.rope_theta)
    torch.cuda.synchronize()
    ref = O.prefill(inp["q"], inp["k"], inp["v"], None, w.rope_theta)
    report(out.cpu().numpy(), ref, TOL_F32, w.name)


@pytest.mark.parametrize("B,S,Hq,Hkv,D,docs", [
    (2, 200, 4, 1, 64, (1, 90)),
    (1, 130, 6, 6, 32, None),
    (3, 97, 8, 2, 128, (20, 60)),
])
def test_prefill_f32_packed(B, S, Hq, Hkv, D, docs):
    w = W.custom_prefill(7, B, S, Hq, Hkv, D, "f32", docs)
    inp = W.make_prefill_inputs(w)
    out = la.llama_attn_prefill_f32(*(to_dev(inp[n]) for n in ("q", "k", "v")),
                                    doc_offsets=to_dev(inp["doc_offsets"]))
    torch.cuda.synchronize()
    ref = O.prefill(inp["q"], inp["k"], inp["v"], inp["doc_offsets"])
    report(out.cpu().numpy(), ref, TOL_F32, f"f32 {B}x{S}x{Hq}/{Hkv}x{D}")


# ---------------------------------------------------------------- prefill bf16 (tcgen05)

BF16_CASES = [
    # B, S, Hq, Hkv, docs, theta
    (1, 128, 2, 1, None, 5e5),            # one tile, one head pair
    (1, 256, 8, 2, None, 5e5),            # causal, two tiles
    (2, 700, 8, 2, (60, 300), 5e5),       # ragged tail, packed documents, G=4 (two heads per CTA)
    (1, 333, 6, 2, (1, 40), 5e5),         # G=3 (one head per CTA), many short documents
    (1, 513, 4, 4, None, 5e6),            # MHA (G=1), base 5,000,000
    (2, 384, 16, 1, (128, 128), 5e5),     # G=16, documents aligned to tiles
    (1, 260, 2, 1, (1, 1), 5e5),          # every document of length 1
    (1, 1, 2, 1, None, 5e5),              # one query row: a single ragged tile
    (2, 5, 4, 2, None, 5e5),              # five rows
    (1, 127, 8, 2, None, 5e5),            # one row short of a tile
    (3, 129, 8, 1, (1, 129), 5e5),        # one row past a tile, G=8
]


@pytest.mark.parametrize("B,S,Hq,Hkv,docs,theta", BF16_CASES)
def test_prefill_bf16_small(B, S, Hq, Hkv, docs, theta):
    w = W.custom_prefill(11 + S, B, S, Hq, Hkv, 128, "bf16", docs, theta)
    inp = W.make_prefill_inputs(w)
    q, k, v = (to_dev(inp[n]) for n in ("q", "k", "v"))
    buf, out = guarded(q.shape)
    la.llama_attn_prefill(q, k, v, out=out, doc_offsets=to_dev(inp["doc_offsets"]), rope_theta=theta)
    torch.cuda.synchronize()
    check_guard(buf)
    ref = O.prefill(inp["q"], inp["k"], inp["v"], inp["doc_offsets"], theta)
    report(out.float().cpu().numpy(), ref, TOL_BF16, f"bf16 {B}x{S}x{Hq}/{Hkv} docs={docs}")


@pytest.mark.parametrize("B,S,Hq,Hkv,offsets", [
    (1, 384, 4, 2, [0, 127, 384]),            # a document starts on the last row of a tile
    (1, 384, 4, 2, [0, 127, 128, 255, 384]),  # starts on rows 127, 128 and 255: tile edges from both sides
    (2, 256, 8, 2, [0, 1, 127, 256, 383, 512]),  # a length-1 document, then starts at 127 in both rows
])
def test_prefill_bf16_document_at_tile_edge(B, S, Hq, Hkv, offsets):
    w = W.custom_prefill(71 + S + len(offsets), B, S, Hq, Hkv, 128, "bf16", None)
    inp = W.make_prefill_inputs(w)
    offs = torch.tensor(offsets, dtype=torch.int32)
    q, k, v = (to_dev(inp[n]) for n in ("q", "k", "v"))
    buf, out = guarded(q.shape)
    la.llama_attn_prefill(q, k, v, out=out, doc_offsets=offs.cuda())
    torch.cuda.synchronize()
    check_guard(buf)
    ref = O.prefill(inp["q"], inp["k"], inp["v"], offs)
    report(out.float().cpu().numpy(), ref, TOL_BF16, f"bf16 {B}x{S}x{Hq}/{Hkv} offsets={offsets}")


def test_prefill_bf16_repeatable_and_stream():
    w = W.custom_prefill(5, 2, 300, 8, 2, 128, "bf16", (50, 200))
    inp = W.make_prefill_inputs(w)
    q, k, v = (to_dev(inp[n]) for n in ("q", "k", "v"))
    offs = to_dev(inp["doc_offsets"])
    a = la.llama_attn_prefill(q, k, v, doc_offsets=offs)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        b = la.llama_attn_prefill(q, k, v, doc_offsets=offs)
    s.synchronize()
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def test_prefill_bad_doc_offsets_sets_device_error():
    w = W.custom_prefill(3, 1, 256, 2, 1, 128, "bf16", None)
    inp = W.make_prefill_inputs(w)
    q, k, v = (to_dev(inp[n]) for n in ("q", "k", "v"))
    bad = torch.tensor([0, 100, 90, 256], dtype=torch.int32, device="cuda")
    la.llama_attn_prefill(q, k, v, doc_offsets=bad)
    assert la.llama_attn_get_device_error() == la.DEVERR_DOC_OFFSETS
    assert la.llama_attn_get_device_error() == 0


# ---------------------------------------------------------------- decode

DECODE_CASES = [
    # B, Hq, Hkv, Lmax, lens
    (6, 16, 2, 3000, [1, 127, 128, 129, 3000, 1025]),
    (3, 16, 1, 2100, [2048, 2049, 64]),       # G=16
    (2, 4, 4, 700, [700, 513]),               # G=1
    (3, 8, 1, 1024, [0, 1, 1024]),            # empty cache gives 0
]


@pytest.mark.parametrize("B,Hq,Hkv,Lmax,lens", DECODE_CASES)
def test_decode_small(B, Hq, Hkv, Lmax, lens):
    w = W.custom_decode(21 + B, B, Hq, Hkv, 128, Lmax, (1, Lmax))
    inp = W.make_decode_inputs(w, poison=True, lens=lens)
    buf, out = guarded(tuple(inp["q"].shape))
    la.llama_attn_decode(*(to_dev(inp[n]) for n in ("q", "kcache", "vcache", "cache_lens")), out=out)
    torch.cuda.synchronize()
    check_guard(buf)
    ref = O.decode(inp["q"], inp["kcache"], inp["vcache"], inp["cache_lens"])
    got = out.float().cpu().numpy()
    report(got, ref, TOL_BF16, f"decode lens={lens}")
    for b, n in enumerate(lens):
        if n == 0:
            assert np.all(got[b] == 0.0)


def test_decode_bad_length_sets_device_error():
    w = W.custom_decode(4, 2, 8, 1, 128, 256, (1, 256))
    inp = W.make_decode_inputs(w, poison=False)
    lens = torch.tensor([300, 10], dtype=torch.int32, device="cuda")
    out = la.llama_attn_decode(to_dev(inp["q"]), to_dev(inp["kcache"]), to_dev(inp["vcache"]), lens)
    assert la.llama_attn_get_device_error() == la.DEVERR_CACHE_LEN
    assert torch.all(out[0].float() == 0)


# ---------------------------------------------------------------- full-size workloads (sampled rows)

def sample_rows(B, S, seed, n_random=512, edge_tiles=48):
    """First and last 256 rows of each batch row, rows on both sides of
    128-row tile edges, and uniform random rows."""
    g = torch.Generator().manual_seed(seed)
    rows = set()
    for b in range(B):
        base = b * S
        rows.update(base + i for i in range(min(256, S)))
        rows.update(base + i for i in range(max(0, S - 256), S))
        for t in torch.randint(1, max(2, S // 128), (edge_tiles,), generator=g).tolist():
            rows.update(base + i for i in (128 * t - 1, 128 * t) if 0 <= i < S)
    rows.update(torch.randint(0, B * S, (n_random,), generator=g).tolist())
    return np.array(sorted(rows), dtype=np.int64)


@pytest.mark.parametrize("w", [W.PACKED_8B, W.PACKED_405B, W.LONG_128K], ids=lambda w: w.name)
def test_prefill_full_config_sampled(w):
    """The full-size workloads in the launch configuration the benchmark
    times, checked on a stratified row sample (all heads of each row): the
    first and last 256 rows of every batch row, rows on both sides of 128-row
    tile edges, and 512 uniform random rows."""
    inp = W.make_prefill_inputs(w)
    q, k, v = (to_dev(inp[n]) for n in ("q", "k", "v"))
    offs = to_dev(inp["doc_offsets"])
    buf, out = guarded(q.shape)
    la.llama_attn_prefill(q, k, v, out=out, doc_offsets=offs, rope_theta=w.rope_theta)
    torch.cuda.synchronize()
    check_guard(buf)
    rows = sample_rows(w.B, w.S, w.seed, n_random=512, edge_tiles=16 if w.S > 100000 else 48)
    got = out.view(w.B * w.S, w.Hq, w.D)[torch.from_numpy(rows).cuda()].float().cpu().numpy()
    ref = O.prefill(inp["q"], inp["k"], inp["v"], inp["doc_offsets"], w.rope_theta, rows=rows)
    report(got, ref, TOL_BF16, w.name, rows=rows)


def test_decode_full_config():
    w = W.DECODE_70B
    inp = W.make_decode_inputs(w, poison=True)
    buf, out = guarded(tuple(inp["q"].shape))
    la.llama_attn_decode(*(to_dev(inp[n]) for n in ("q", "kcache", "vcache", "cache_lens")), out=out)
    torch.cuda.synchronize()
    check_guard(buf)
    ref = O.decode(inp["q"], inp["kcache"], inp["vcache"], inp["cache_lens"])
    report(out.float().cpu().numpy(), ref, TOL_BF16, w.name)
