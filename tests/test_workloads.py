"""The seeded input recipe both the oracle and the CUDA path read
(gqa_attention_rope_b200/workloads.py): shapes, dtypes, reproducibility,
document-length ranges, cache-length ranges, the NaN poison past each cached
sequence, and the unmasked-pair count that the throughput metric divides by
(checked against a brute-force count of the mask)."""
import os

import numpy as np
import torch

from gqa_attention_rope_b200 import workloads as W
from oracle import oracle as O


def _doc_lengths(offs, B, S):
    o = offs.to(torch.int64).numpy()
    assert o[0] == 0 and o[-1] == B * S and np.all(np.diff(o) > 0)
    rows = []
    for b in range(B):
        inside = o[(o >= b * S) & (o <= (b + 1) * S)] - b * S
        assert inside[0] == 0 and inside[-1] == S, "a document crosses a batch-row boundary"
        rows.append(np.diff(inside))
    return rows


def test_packed_prefill_recipe():
    w = W.PACKED_8B
    a, b = W.make_prefill_inputs(w), W.make_prefill_inputs(w)
    for n in ("q", "k", "v"):
        assert a[n].dtype == torch.bfloat16 and torch.equal(a[n], b[n]), "same seed, same bits"
    assert a["q"].shape == (w.B, w.S, w.Hq, w.D) and a["k"].shape == (w.B, w.S, w.Hkv, w.D)
    q = a["q"].float()
    assert abs(float(q.mean())) < 0.01 and abs(float(q.std()) - 1.0) < 0.01
    lo, hi = w.doc_range
    for lens in _doc_lengths(a["doc_offsets"], w.B, w.S):
        assert np.all(lens[:-1] >= lo) and np.all(lens <= hi) and lens[-1] >= 1
    # a different seed gives different data
    other = W.PrefillWorkload(w.name, w.seed + 1, w.B, w.S, w.Hq, w.Hkv, w.D, w.dtype, w.doc_range, w.rope_theta)
    assert not torch.equal(W.make_prefill_inputs(other)["q"], a["q"])


def test_single_document_and_fp32_recipes():
    for w in (W.TINY_F32,):
        inp = W.make_prefill_inputs(w)
        assert inp["doc_offsets"] is None and inp["q"].dtype == torch.float32
        assert inp["q"].shape == (w.B, w.S, w.Hq, w.D)


def test_decode_recipe_and_poison():
    w = W.custom_decode(5, 6, 16, 2, 128, 300, (10, 300))
    inp = W.make_decode_inputs(w, poison=True)
    lens = inp["cache_lens"].numpy()
    assert np.all((lens >= 10) & (lens <= 300))
    kc = inp["kcache"].float().numpy()
    for b, n in enumerate(lens):
        assert np.all(np.isfinite(kc[b, :, :n])), "cached rows are finite"
        assert np.all(np.isnan(kc[b, :, n:])), "rows past the length are poisoned"
    again = W.make_decode_inputs(w, poison=True)
    assert torch.equal(again["q"], inp["q"]) and torch.equal(again["cache_lens"], inp["cache_lens"])


def test_unmasked_pairs_matches_mask_count():
    w = W.custom_prefill(9, 2, 97, 2, 1, 16, "f32", (5, 30))
    inp = W.make_prefill_inputs(w)
    ds, _ = O.doc_layout(inp["doc_offsets"], w.B, w.S)
    count = 0
    for b in range(w.B):
        for i in range(w.S):
            for j in range(i + 1):
                count += ds[b * w.S + i] == ds[b * w.S + j]  # same document (starts are row-local)
    assert W.unmasked_pairs(inp["doc_offsets"], w.B, w.S) == count
    assert W.unmasked_pairs(None, 3, 10) == 3 * 55


def _page_numbers():
    vals = {}
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "page_shapes.txt")
    for line in open(path):
        line = line.split("#")[0].strip()
        if line:
            k, v = (x.strip() for x in line.split("="))
            vals[k] = int(v)
    return vals


def test_workloads_follow_the_pages_head_layouts():
    """The synthetic workloads carry the head layouts and RoPE base the pages
    print (tests/golden/page_shapes.txt, each number cited there)."""
    pg = _page_numbers()
    for w in (W.PACKED_8B, W.PACKED_405B, W.LONG_128K, W.DECODE_70B):
        assert w.Hkv == pg["kv_heads_all"], w.name
        assert w.D * w.Hq // w.Hq == 128 and w.rope_theta == pg["rope_base"], w.name
    w = W.PACKED_405B
    assert (w.Hq, w.Hkv) == (pg["heads_405b"], pg["kv_heads_405b"])
    assert pg["d_model_405b"] // pg["heads_405b"] == w.D  # head_dim = hidden / heads
    # the long-context base is a value the library accepts as an argument, not the default
    assert pg["rope_base_long"] == 10 * pg["rope_base"] and pg["rope_base_original"] < pg["rope_base"]
