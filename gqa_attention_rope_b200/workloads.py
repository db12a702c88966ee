"""Seeded synthetic inputs for the attention library and its CPU oracle.

This module draws random numbers and lays out document / cache-length
structure. It holds none of the attention arithmetic (no RoPE, no softmax,
no masking), so both the CUDA path and the float64 oracle can consume the
exact same bit patterns from it without sharing any of the method's code.

Recipe (one torch CPU generator per workload, seeded as listed):

* values: float32 N(0, 1), rounded to nearest-even into bf16 for the bf16
  workloads (``Tensor.to(torch.bfloat16)`` rounds RNE);
* document lengths: uniform integers in the inclusive range, drawn one after
  another for each batch row until the row is full; the last document is
  truncated to fit (so it may be shorter than the lower bound);
* decode cache lengths: uniform integers in the inclusive range; cache rows
  at or past a sequence's length are filled with NaN so that any read of the
  padding shows up in the output.

The shapes mirror the Llama 3 / 3.1 attention layouts named on the pages:
8 KV heads shared by 32, 64 or 128 query heads with head_dim 128 ("The Llama
3 Herd of Models" overview: GQA with 8 KV heads; "Llama 3.1 Architecture",
405B hyper-parameters: 128 heads, 8 KV heads, d_model 16384).
"""
from __future__ import annotations

import dataclasses
from typing import Optional, Tuple

import torch

BF16_NAN_BITS = 0x7FC0


@dataclasses.dataclass(frozen=True)
class PrefillWorkload:
    name: str
    seed: int
    B: int
    S: int
    Hq: int
    Hkv: int
    D: int
    dtype: str  # "bf16" or "f32"
    doc_range: Optional[Tuple[int, int]]  # None: one document per batch row
    rope_theta: float = 500000.0


@dataclasses.dataclass(frozen=True)
class DecodeWorkload:
    name: str
    seed: int
    B: int
    Hq: int
    Hkv: int
    D: int
    Lmax: int
    len_range: Tuple[int, int]
    dtype: str = "bf16"
    rope_theta: float = 500000.0


# The five workloads the library is specified and measured on.
TINY_F32 = PrefillWorkload("tiny_f32_B1_S256_Hq8_Hkv2_D64", 1, 1, 256, 8, 2, 64, "f32", None)
PACKED_8B = PrefillWorkload("llama8b_packed_B4_S8192_Hq32_Hkv8_D128_docs512-4096", 2,
                            4, 8192, 32, 8, 128, "bf16", (512, 4096))
PACKED_405B = PrefillWorkload("llama405b_packed_B1_S16384_Hq128_Hkv8_D128_docs1024-8192", 3,
                              1, 16384, 128, 8, 128, "bf16", (1024, 8192))
LONG_128K = PrefillWorkload("long128k_B1_S131072_Hq32_Hkv8_D128_causal", 4,
                            1, 131072, 32, 8, 128, "bf16", None)
DECODE_70B = DecodeWorkload("llama70b_decode_B64_Hq64_Hkv8_D128_len1024-32768", 5,
                            64, 64, 8, 128, 32768, (1024, 32768))

WORKLOADS = {w.name: w for w in (TINY_F32, PACKED_8B, PACKED_405B, LONG_128K, DECODE_70B)}

# A shorter single-document prefill with the 128K workload's head layout, used
# only where hardware-counter captures need a smaller launch of the same
# kernel; it is not one of the measured workloads.
LONG_32K_CAPTURE = PrefillWorkload("long32k_B1_S32768_Hq32_Hkv8_D128_causal", 4, 1, 32768, 32, 8, 128, "bf16", None)
CAPTURE_WORKLOADS = {LONG_32K_CAPTURE.name: LONG_32K_CAPTURE}


def draw_doc_lengths(gen: torch.Generator, S: int, lo: int, hi: int) -> list:
    """Uniform integer document lengths in [lo, hi] filling one row of S tokens."""
    lengths = []
    used = 0
    while used < S:
        n = int(torch.randint(lo, hi + 1, (1,), generator=gen).item())
        n = min(n, S - used)
        lengths.append(n)
        used += n
    return lengths


def doc_offsets_from_lengths(row_lengths: list, S: int) -> torch.Tensor:
    """Cumulative document starts in flattened B*S token coordinates, ending with
    the sentinel B*S (the library's ``doc_offsets`` format)."""
    offs = []
    base = 0
    for lengths in row_lengths:
        assert sum(lengths) == S
        t = base
        for n in lengths:
            offs.append(t)
            t += n
        base += S
    offs.append(base)
    return torch.tensor(offs, dtype=torch.int32)


def _randn(gen: torch.Generator, shape, dtype: str) -> torch.Tensor:
    x = torch.randn(shape, generator=gen, dtype=torch.float32)
    if dtype == "bf16":
        return x.to(torch.bfloat16)
    assert dtype == "f32"
    return x


def make_prefill_inputs(w: PrefillWorkload):
    """Returns dict(q, k, v, doc_offsets) as CPU tensors.

    q is [B, S, Hq, D], k and v are [B, S, Hkv, D]; doc_offsets is an int32
    tensor (or None when every batch row is one document)."""
    gen = torch.Generator().manual_seed(w.seed)
    doc_offsets = None
    if w.doc_range is not None:
        rows = [draw_doc_lengths(gen, w.S, *w.doc_range) for _ in range(w.B)]
        doc_offsets = doc_offsets_from_lengths(rows, w.S)
    q = _randn(gen, (w.B, w.S, w.Hq, w.D), w.dtype)
    k = _randn(gen, (w.B, w.S, w.Hkv, w.D), w.dtype)
    v = _randn(gen, (w.B, w.S, w.Hkv, w.D), w.dtype)
    return dict(q=q, k=k, v=v, doc_offsets=doc_offsets)


def custom_prefill(seed: int, B: int, S: int, Hq: int, Hkv: int, D: int, dtype: str = "bf16",
                   doc_range: Optional[Tuple[int, int]] = None, rope_theta: float = 500000.0,
                   name: str = "custom") -> PrefillWorkload:
    return PrefillWorkload(name, seed, B, S, Hq, Hkv, D, dtype, doc_range, rope_theta)


def make_decode_inputs(w: DecodeWorkload, poison: bool = True, lens=None):
    """Returns dict(q, kcache, vcache, cache_lens) as CPU tensors.

    q is [B, Hq, D]; kcache and vcache are [B, Hkv, Lmax, D] and hold keys that
    the caller has already rotated at their cache positions. An iid N(0, 1)
    draw is used directly as those rotated keys: a rotation maps an iid
    Gaussian vector to an iid Gaussian vector, so the distribution is the one
    the workload names. Rows at or past cache_lens[b] are NaN when ``poison``.
    ``lens`` (optional) replaces the drawn cache lengths.
    """
    gen = torch.Generator().manual_seed(w.seed)
    drawn = torch.randint(w.len_range[0], w.len_range[1] + 1, (w.B,), generator=gen,
                          dtype=torch.int64).to(torch.int32)
    lens = drawn if lens is None else torch.as_tensor(lens, dtype=torch.int32)
    q = _randn(gen, (w.B, w.Hq, w.D), w.dtype)
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    fill = float("nan") if poison else 0.0
    kc = torch.full((w.B, w.Hkv, w.Lmax, w.D), fill, dtype=tdt)
    vc = torch.full((w.B, w.Hkv, w.Lmax, w.D), fill, dtype=tdt)
    for b in range(w.B):
        n = int(lens[b])
        kc[b, :, :n] = _randn(gen, (w.Hkv, n, w.D), w.dtype)
        vc[b, :, :n] = _randn(gen, (w.Hkv, n, w.D), w.dtype)
    return dict(q=q, kcache=kc, vcache=vc, cache_lens=lens)


def custom_decode(seed: int, B: int, Hq: int, Hkv: int, D: int, Lmax: int,
                  len_range: Tuple[int, int], dtype: str = "bf16", rope_theta: float = 500000.0,
                  name: str = "custom") -> DecodeWorkload:
    return DecodeWorkload(name, seed, B, Hq, Hkv, D, Lmax, len_range, dtype, rope_theta)


def unmasked_pairs(doc_offsets: Optional[torch.Tensor], B: int, S: int) -> int:
    """Number of (i, j) pairs per head that the causal + cross-document mask keeps.

    A document of n tokens contributes n (n + 1) / 2 pairs. This counts the
    work a step does (the FLOP numerator of the prefill metric); it is
    bookkeeping over lengths, not attention arithmetic."""
    if doc_offsets is None:
        return B * S * (S + 1) // 2
    o = doc_offsets.to(torch.int64)
    n = o[1:] - o[:-1]
    return int((n * (n + 1) // 2).sum().item())


def cache_tokens(cache_lens: torch.Tensor) -> int:
    return int(cache_lens.to(torch.int64).sum().item())
