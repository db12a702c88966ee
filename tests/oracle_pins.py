"""Checks that pin the float64 oracle to facts outside itself.

Each ``check_*`` function takes an oracle library handle (the real one, or a
deliberately broken copy built by the mutation test) and raises
AssertionError when the oracle disagrees with:

* an independent torch float64 formulation (complex-number RoPE, explicit
  ``repeat_interleave`` of the KV heads, and
  ``torch.nn.functional.scaled_dot_product_attention`` with a boolean mask);
* closed forms (the RoPE frequency formula, a hand-derived worked example);
* invariants the mathematics fixes (RoPE relative-position identity, norm
  preservation, softmax rows summing to 1, constant V, packing = separate
  documents, decode consistent with prefill).
"""
from __future__ import annotations

import math
import os

import numpy as np
import torch
import torch.nn.functional as F

from oracle import oracle as O

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


# ----------------------------------------------------------------------------
# independent torch float64 formulation (used only as a pin)

def torch_doc_ids_positions(row_lengths, S):
    B = len(row_lengths)
    pos = torch.zeros(B, S, dtype=torch.float64)
    doc = torch.zeros(B, S, dtype=torch.long)
    for b, lengths in enumerate(row_lengths):
        t = 0
        for d, n in enumerate(lengths):
            pos[b, t:t + n] = torch.arange(n, dtype=torch.float64)
            doc[b, t:t + n] = d
            t += n
    return doc, pos


def torch_rope_complex(x, pos, base):
    """x [B,S,H,D] float64, pos [B,S] -> rotated via complex multiplication."""
    D = x.shape[-1]
    inv = base ** (-torch.arange(0, D, 2, dtype=torch.float64) / D)
    ang = pos[..., None] * inv  # [B,S,D/2]
    rot = torch.polar(torch.ones_like(ang), ang)[:, :, None, :]
    xc = torch.view_as_complex(x.reshape(*x.shape[:-1], D // 2, 2).contiguous())
    return torch.view_as_real(xc * rot).reshape(x.shape)


def torch_reference(q, k, v, row_lengths, base, global_positions=False):
    q, k, v = (t.to(torch.float64) for t in (q, k, v))
    B, S, Hq, D = q.shape
    Hkv = k.shape[2]
    doc, pos = torch_doc_ids_positions(row_lengths, S)
    if global_positions:
        pos = torch.arange(S, dtype=torch.float64).expand(B, S).clone()
    qr = torch_rope_complex(q, pos, base)
    kr = torch_rope_complex(k, pos, base)
    kr = kr.repeat_interleave(Hq // Hkv, dim=2)
    vr = v.repeat_interleave(Hq // Hkv, dim=2)
    i = torch.arange(S)
    mask = (doc[:, :, None] == doc[:, None, :]) & (i[None, None, :] <= i[None, :, None])
    out = F.scaled_dot_product_attention(qr.transpose(1, 2), kr.transpose(1, 2), vr.transpose(1, 2),
                                         attn_mask=mask[:, None])
    return out.transpose(1, 2)


def offsets_of(row_lengths, S):
    from gqa_attention_rope_b200.workloads import doc_offsets_from_lengths
    return doc_offsets_from_lengths(row_lengths, S)


def _rand(gen, *shape):
    return torch.randn(*shape, generator=gen, dtype=torch.float64)


# ----------------------------------------------------------------------------
# checks

def check_rope_freqs_closed_form(lib):
    for D in (2, 8, 64, 128):
        for base in (10000.0, 500000.0, 5000000.0):
            f = O.rope_freqs(D, base, lib=lib)
            assert f.shape == (D // 2,)
            assert f[0] == 1.0
            # theta_{D/2-1} = base^(-(D-2)/D)
            assert math.isclose(f[-1], base ** (-(D - 2) / D), rel_tol=1e-14)
            # geometric progression with ratio base^(-2/D)
            if D > 2:
                r = f[1:] / f[:-1]
                assert np.allclose(r, base ** (-2.0 / D), rtol=1e-13, atol=0)
    f = O.rope_freqs(128, 500000.0, lib=lib)
    assert math.isclose(f[63], math.exp(-(126 / 128) * math.log(500000.0)), rel_tol=1e-13)


def check_rope_identities(lib):
    gen = torch.Generator().manual_seed(11)
    D, base = 16, 500000.0
    x = _rand(gen, 5, D).numpy()
    y = _rand(gen, 5, D).numpy()
    # R(0) = I
    assert np.array_equal(O.rope_rotate(x, np.zeros(5), base, lib=lib), x)
    # norm preservation
    p = np.array([1.0, 7.0, 100.0, 4095.0, 131071.0])
    xr = O.rope_rotate(x, p, base, lib=lib)
    assert np.allclose(np.linalg.norm(xr, axis=1), np.linalg.norm(x, axis=1), rtol=1e-13)
    # <R(m) x, R(n) y> = <x, R(n - m) y>
    m = np.array([3.0, 10.0, 0.0, 500.0, 2.0])
    n = np.array([9.0, 4.0, 77.0, 500.0, 131000.0])
    lhs = np.sum(O.rope_rotate(x, m, base, lib=lib) * O.rope_rotate(y, n, base, lib=lib), axis=1)
    rhs = np.sum(x * O.rope_rotate(y, n - m, base, lib=lib), axis=1)
    assert np.allclose(lhs, rhs, rtol=1e-9, atol=1e-9)
    # agrees with the complex-number form
    xt = torch.from_numpy(x).reshape(1, 5, 1, D)
    ref = torch_rope_complex(xt, torch.from_numpy(p).reshape(1, 5), base).reshape(5, D).numpy()
    assert np.allclose(xr, ref, rtol=1e-12, atol=1e-12)
    # multi-head layout: every head of a token uses the token's position
    xh = _rand(gen, 3, 4, D).numpy()
    ph = np.array([2.0, 5.0, 1000.0])
    yh = O.rope_rotate(xh, ph, base, lib=lib)
    for h in range(4):
        assert np.array_equal(yh[:, h], O.rope_rotate(xh[:, h], ph, base, lib=lib))


def torch_rope_rotate_half(x, pos, base):
    """The other common RoPE layout, written out independently: dimension k is
    paired with dimension k + D/2 (first half, second half) and the pair turns
    by pos * base^(-2k/D). x [..., T, D] float64, pos [T]."""
    D = x.shape[-1]
    inv = base ** (-torch.arange(0, D, 2, dtype=torch.float64) / D)
    ang = pos[:, None] * inv
    c, s = torch.cos(ang), torch.sin(ang)
    x1, x2 = x[..., : D // 2], x[..., D // 2:]
    return torch.cat([x1 * c - x2 * s, x2 * c + x1 * s], dim=-1)


def check_rotate_half_is_a_permutation(lib):
    """The adjacent-pair rotation (RoFormer's, which the oracle follows) and
    the rotate-half layout are one method under a fixed permutation of the
    head dimensions: with P putting the even dimensions first and the odd ones
    after, rotate_half(P x) = P R(p) x. So attention computed in either layout
    from correspondingly permuted q and k is the same."""
    gen = torch.Generator().manual_seed(23)
    D, base, T = 16, 500000.0, 6
    perm = torch.cat([torch.arange(0, D, 2), torch.arange(1, D, 2)])
    x = _rand(gen, T, D)
    pos = torch.tensor([0.0, 1.0, 5.0, 37.0, 4096.0, 131071.0], dtype=torch.float64)
    ours = torch.from_numpy(O.rope_rotate(x.numpy(), pos.numpy(), base, lib=lib))
    half = torch_rope_rotate_half(x[:, perm], pos, base)
    assert torch.allclose(half, ours[:, perm], rtol=1e-12, atol=1e-12)
    # attention: the rotate-half layout on permuted q and k = the oracle on the originals
    B, S, Hq, Hkv = 1, 9, 4, 2
    q, k, v = _rand(gen, B, S, Hq, D), _rand(gen, B, S, Hkv, D), _rand(gen, B, S, Hkv, D)
    p = torch.arange(S, dtype=torch.float64)
    qh = torch_rope_rotate_half(q[..., perm].permute(0, 2, 1, 3), p, base)      # [B, Hq, S, D]
    kh = torch_rope_rotate_half(k[..., perm].permute(0, 2, 1, 3), p, base)
    kh = kh.repeat_interleave(Hq // Hkv, dim=1)
    vh = v.permute(0, 2, 1, 3).repeat_interleave(Hq // Hkv, dim=1)
    ref = F.scaled_dot_product_attention(qh, kh, vh, is_causal=True).permute(0, 2, 1, 3).numpy()
    got = O.prefill(q, k, v, None, base, lib=lib)
    assert np.allclose(got, ref, rtol=1e-10, atol=1e-12)


def check_worked_example(lib):
    vals = {}
    with open(os.path.join(GOLDEN, "worked_example_rope_attention.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if "=" in line:
                key, val = (s.strip() for s in line.split("="))
                vals[key] = val
    vec = lambda s: [float(t) for t in s.split()]
    q = torch.tensor([[vec(vals["q0"])], [vec(vals["q1"])]], dtype=torch.float64)[None]
    k = torch.tensor([[vec(vals["k0"])], [vec(vals["k1"])]], dtype=torch.float64)[None]
    v = torch.tensor([[vec(vals["v0"])], [vec(vals["v1"])]], dtype=torch.float64)[None]
    v0, v1 = np.array(vec(vals["v0"])), np.array(vec(vals["v1"]))
    w0 = 1.0 / (1.0 + math.exp(math.sin(1.0) / math.sqrt(2.0)))
    expect1 = w0 * v0 + (1.0 - w0) * v1
    for base in (10000.0, 500000.0):
        out = O.prefill(q, k, v, None, base, lib=lib)
        assert np.array_equal(out[0, 0, 0], np.array(vec(vals["expect_out0"])))
        assert np.allclose(out[0, 1, 0], expect1, rtol=1e-14, atol=1e-14)


def check_bruteforce_vs_torch(lib):
    gen = torch.Generator().manual_seed(12)
    cases = [
        # (B, S, Hq, Hkv, D, row_lengths)
        (1, 7, 4, 2, 4, [[7]]),
        (2, 16, 4, 1, 8, [[5, 11], [16]]),
        (2, 13, 6, 3, 8, [[1, 4, 8], [2, 2, 9]]),
        (1, 16, 4, 4, 8, [[3, 3, 3, 7]]),  # MHA: Hkv = Hq
        (2, 9, 8, 2, 4, [[1, 1, 1, 1, 1, 1, 1, 1, 1], [9]]),
    ]
    for (B, S, Hq, Hkv, D, lens) in cases:
        q, k, v = _rand(gen, B, S, Hq, D), _rand(gen, B, S, Hkv, D), _rand(gen, B, S, Hkv, D)
        for base in (500000.0, 10000.0):
            ref = torch_reference(q, k, v, lens, base).numpy()
            offs = offsets_of(lens, S)
            got = O.prefill(q, k, v, offs, base, lib=lib)
            assert np.allclose(got, ref, rtol=1e-11, atol=1e-11), (B, S, Hq, Hkv, D, lens)
            # the sampled-rows entry point gives the same rows
            rows = np.array([0, S - 1, B * S - 1, (B - 1) * S + S // 2])
            got_rows = O.prefill(q, k, v, offs, base, rows=rows, lib=lib)
            assert np.array_equal(got_rows, got.reshape(B * S, Hq, D)[rows])


def check_mha_equals_sdpa(lib):
    gen = torch.Generator().manual_seed(13)
    B, S, H, D = 2, 12, 3, 8
    q, k, v = _rand(gen, B, S, H, D), _rand(gen, B, S, H, D), _rand(gen, B, S, H, D)
    pos = torch.arange(S, dtype=torch.float64).expand(B, S)
    qr = torch_rope_complex(q, pos, 500000.0).transpose(1, 2)
    kr = torch_rope_complex(k, pos, 500000.0).transpose(1, 2)
    ref = F.scaled_dot_product_attention(qr, kr, v.transpose(1, 2), is_causal=True).transpose(1, 2)
    got = O.prefill(q, k, v, None, 500000.0, lib=lib)
    assert np.allclose(got, ref.numpy(), rtol=1e-11, atol=1e-11)


def check_restart_equals_global_positions(lib):
    """Positions restarting per document give the same result as global
    positions (the score depends only on the position difference)."""
    gen = torch.Generator().manual_seed(14)
    B, S, Hq, Hkv, D = 1, 40, 4, 2, 8
    lens = [[9, 20, 11]]
    q, k, v = _rand(gen, B, S, Hq, D), _rand(gen, B, S, Hkv, D), _rand(gen, B, S, Hkv, D)
    ref = torch_reference(q, k, v, lens, 500000.0, global_positions=True).numpy()
    got = O.prefill(q, k, v, offsets_of(lens, S), 500000.0, lib=lib)
    assert np.allclose(got, ref, rtol=1e-10, atol=1e-10)


def check_packing_equals_separate(lib):
    gen = torch.Generator().manual_seed(15)
    S, Hq, Hkv, D = 30, 4, 2, 8
    lens = [4, 1, 13, 12]
    q, k, v = _rand(gen, 1, S, Hq, D), _rand(gen, 1, S, Hkv, D), _rand(gen, 1, S, Hkv, D)
    packed = O.prefill(q, k, v, offsets_of([lens], S), 500000.0, lib=lib)
    t = 0
    for n in lens:
        alone = O.prefill(q[:, t:t + n], k[:, t:t + n], v[:, t:t + n], None, 500000.0, lib=lib)
        assert np.allclose(packed[:, t:t + n], alone, rtol=1e-12, atol=1e-12)
        t += n


def check_softmax_invariants(lib):
    gen = torch.Generator().manual_seed(16)
    B, S, Hq, Hkv, D = 2, 20, 4, 2, 8
    lens = [[6, 14], [20]]
    offs = offsets_of(lens, S)
    q, k, v = _rand(gen, B, S, Hq, D), _rand(gen, B, S, Hkv, D), _rand(gen, B, S, Hkv, D)
    doc, _ = torch_doc_ids_positions(lens, S)
    for (b, h, i) in [(0, 0, 0), (0, 3, 5), (0, 1, 6), (0, 2, 19), (1, 0, 19), (1, 3, 7)]:
        w = O.prefill_weights(q, k, b, h, i, offs, lib=lib)
        assert math.isclose(w.sum(), 1.0, rel_tol=0, abs_tol=1e-13)
        vis = np.array([(j <= i) and (doc[b, j] == doc[b, i]) for j in range(S)])
        assert np.all(w[~vis] == 0.0) and np.all(w[vis] > 0.0)
        # the output row is the weighted sum of the visible value rows
        out = O.prefill(q, k, v, offs, lib=lib)
        g = h // (Hq // Hkv)
        assert np.allclose(out[b, i, h], w @ v[b, :, g].numpy(), rtol=1e-12, atol=1e-12)
    # constant V returns the constant
    c = torch.full((B, S, Hkv, D), 0.0, dtype=torch.float64)
    c[..., :] = torch.arange(D, dtype=torch.float64) - 2.5
    out = O.prefill(q, k, c, offs, lib=lib)
    assert np.allclose(out, np.broadcast_to(c[:, :, :1].numpy(), out.shape), rtol=0, atol=1e-13)
    # the first row of every document returns its own value row exactly
    out = O.prefill(q, k, v, offs, lib=lib)
    for b, i in [(0, 0), (0, 6), (1, 0)]:
        for h in range(Hq):
            assert np.array_equal(out[b, i, h], v[b, i, h // (Hq // Hkv)].numpy())


def check_decode_consistent_with_prefill(lib):
    gen = torch.Generator().manual_seed(17)
    Hq, Hkv, D, base = 8, 2, 8, 500000.0
    for L in (1, 2, 5, 33):
        q = _rand(gen, 1, L + 1, Hq, D)
        k = _rand(gen, 1, L + 1, Hkv, D)
        v = _rand(gen, 1, L + 1, Hkv, D)
        # the cache holds keys 0..L-1 rotated at their positions
        kc = O.rope_rotate(k[0, :L].numpy(), np.arange(L, dtype=np.float64), base, lib=lib)
        kc = torch.from_numpy(kc).permute(1, 0, 2)[None].contiguous()  # [1, Hkv, L, D]
        vc = v[0, :L].permute(1, 0, 2)[None].contiguous()
        dec = O.decode(q[:, L], kc, vc, torch.tensor([L], dtype=torch.int32), base, lib=lib)
        if L == 1:
            for h in range(Hq):
                assert np.array_equal(dec[0, h], vc[0, h // (Hq // Hkv), 0].numpy())
        # With v_L set to the decode output, prefill row L (which also sees key L)
        # must return that same vector: a convex mix of equal vectors.
        for h in range(Hq):
            g = h // (Hq // Hkv)
            v2 = v.clone()
            v2[0, L, g] = torch.from_numpy(dec[0, h])
            pre = O.prefill(q, k, v2, None, base, rows=np.array([L]), lib=lib)
            assert np.allclose(pre[0, h], dec[0, h], rtol=1e-11, atol=1e-11), (L, h)
    # an independent torch evaluation of the decode definition
    B, L, Lmax = 3, 11, 16
    q = _rand(gen, B, Hq, D)
    kc = _rand(gen, B, Hkv, Lmax, D)
    vc = _rand(gen, B, Hkv, Lmax, D)
    lens = torch.tensor([11, 1, 16], dtype=torch.int32)
    got = O.decode(q, kc, vc, lens, base, lib=lib)
    for b in range(B):
        n = int(lens[b])
        qr = torch_rope_complex(q[b][None, None], torch.tensor([[float(n)]], dtype=torch.float64), base)[0, 0]
        kk = kc[b, :, :n].repeat_interleave(Hq // Hkv, dim=0)
        vv = vc[b, :, :n].repeat_interleave(Hq // Hkv, dim=0)
        ref = F.scaled_dot_product_attention(qr[:, None], kk, vv)[:, 0]
        assert np.allclose(got[b], ref.numpy(), rtol=1e-11, atol=1e-11)
    # len = 0 gives zeros
    z = O.decode(q[:1], kc[:1], vc[:1], torch.tensor([0], dtype=torch.int32), base, lib=lib)
    assert np.array_equal(z, np.zeros_like(z))


def check_doc_layout(lib):
    S = 8
    ds, pos = O.doc_layout(torch.tensor([0, 3, 8, 9, 16], dtype=torch.int32), 2, S, lib=lib)
    assert ds.tolist() == [0, 0, 0, 3, 3, 3, 3, 3, 0, 1, 1, 1, 1, 1, 1, 1]
    assert pos.tolist() == [0, 1, 2, 0, 1, 2, 3, 4, 0, 0, 1, 2, 3, 4, 5, 6]
    ds, pos = O.doc_layout(None, 2, 3, lib=lib)
    assert ds.tolist() == [0] * 6 and pos.tolist() == [0, 1, 2, 0, 1, 2]
    bad = [[1, 16], [0, 3, 3, 16], [0, 5, 12, 16], [0, 10, 8, 16]]
    for b in bad:
        try:
            O.doc_layout(torch.tensor(b, dtype=torch.int32), 2, S, lib=lib)
        except ValueError:
            continue
        raise AssertionError(f"accepted malformed offsets {b}")


def check_lse(lib):
    """The log-sum-exp the oracle reports equals torch.logsumexp of the
    independently formed masked scores, and out = sum exp(s - lse) v."""
    if not hasattr(lib, "oracle_prefill_lse"):
        return
    gen = torch.Generator().manual_seed(18)
    B, S, Hq, Hkv, D, base = 2, 14, 4, 2, 8, 500000.0
    lens = [[5, 9], [14]]
    q, k, v = _rand(gen, B, S, Hq, D), _rand(gen, B, S, Hkv, D), _rand(gen, B, S, Hkv, D)
    out, lse = O.prefill_lse(q, k, v, offsets_of(lens, S), base, lib=lib)
    doc, pos = torch_doc_ids_positions(lens, S)
    qr = torch_rope_complex(q, pos, base)
    kr = torch_rope_complex(k, pos, base).repeat_interleave(Hq // Hkv, dim=2)
    vr = v.repeat_interleave(Hq // Hkv, dim=2)
    scores = torch.einsum("bihd,bjhd->bhij", qr, kr) / math.sqrt(D)
    i = torch.arange(S)
    mask = (doc[:, :, None] == doc[:, None, :]) & (i[None, None, :] <= i[None, :, None])
    scores = scores.masked_fill(~mask[:, None], float("-inf"))
    ref = torch.logsumexp(scores, dim=-1).permute(0, 2, 1)  # [B, S, Hq]
    assert np.allclose(lse, ref.numpy(), rtol=1e-12, atol=1e-12)
    rebuilt = torch.einsum("bhij,bjhd->bihd", torch.exp(scores - ref.permute(0, 2, 1)[..., None]), vr)
    assert np.allclose(out, rebuilt.numpy(), rtol=1e-11, atol=1e-11)
    # the plain entry point gives the same output
    assert np.array_equal(out, O.prefill(q, k, v, offsets_of(lens, S), base, lib=lib))


ALL_CHECKS = [
    check_rope_freqs_closed_form,
    check_rope_identities,
    check_rotate_half_is_a_permutation,
    check_worked_example,
    check_bruteforce_vs_torch,
    check_mha_equals_sdpa,
    check_restart_equals_global_positions,
    check_packing_equals_separate,
    check_softmax_invariants,
    check_decode_consistent_with_prefill,
    check_doc_layout,
    check_lse,
]
