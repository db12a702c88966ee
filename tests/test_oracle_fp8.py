"""Pins of the FP8 (E4M3) oracle to facts outside itself.

- The code table against the format's fixed points (448 the largest finite
  value, 2^-9 the smallest subnormal, 2^-6 the smallest normal, 254 finite
  codes, monotone order).
- Rounding against a brute-force nearest-value search over the table (ties to
  the even code) and against torch's float8_e4m3fn conversion, a library
  routine, inside the finite range.
- Per-tensor scaling: the largest magnitude lands on 448, power-of-two
  rescaling of the input leaves the codes unchanged, zeros give scale 1.
- The projection: exact integer matmul when every operand is an exactly
  representable integer and the scales are 1, and one-hot weight rows that
  fix which output column lands in which head of Q, K, V.
- The rotation after it: an independent complex-number RoPE in this file.
Each pin is also run against planted mistakes in a copy of the oracle, and
every mistake must be caught.
"""
import os
import types

import numpy as np
import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
FP8_SRC = os.path.join(ROOT, "oracle", "fp8.py")

from oracle import fp8 as F  # noqa: E402


# ---------------------------------------------------------------- pins

def pin_table(F):
    t = F.e4m3_table()
    assert t[0x7E] == 448.0 and t[0xFE] == -448.0
    assert np.isnan(t[0x7F]) and np.isnan(t[0xFF])
    assert t[0x01] == 2.0 ** -9 and t[0x08] == 2.0 ** -6 and t[0x07] == 7 * 2.0 ** -9
    assert t[0x38] == 1.0 and t[0x39] == 1.125
    assert np.sum(np.isfinite(t)) == 254
    pos = t[:0x7F]
    assert np.all(np.diff(pos) > 0), "codes 0..126 must increase"
    assert np.array_equal(t[0x80:0xFF], -t[0x00:0x7F])


def _brute_round(x: np.ndarray, t: np.ndarray) -> np.ndarray:
    finite = np.where(np.isfinite(t))[0]
    vals = t[finite]
    out = np.empty(x.shape, np.uint8)
    for i, xi in enumerate(x.reshape(-1)):
        xc = min(max(xi, -448.0), 448.0)
        d = np.abs(vals - xc)
        best = np.where(d == d.min())[0]
        cand = finite[best]
        if len(cand) > 1:  # a tie: the code with the even mantissa (last bit 0)
            cand = [c for c in cand if (c & 1) == 0]
        code = int(cand[0])
        if t[code] == 0.0:  # a value that rounds to zero keeps its sign
            code = 0x80 if np.signbit(xi) else 0x00
        out.reshape(-1)[i] = code
    return out


def pin_round_brute(F):
    t = F.e4m3_table()
    rng = np.random.default_rng(7)
    x = np.concatenate([
        rng.standard_normal(3000) * 4.0,
        rng.standard_normal(1000) * 2.0 ** -7,                    # subnormal range
        rng.uniform(300.0, 1000.0, 200) * rng.choice([-1, 1], 200),  # near and past the top
        # exact midpoints between neighbouring codes: the ties
        (t[0x01:0x7E] + t[0x02:0x7F]) / 2.0,
        -(t[0x31:0x50] + t[0x32:0x51]) / 2.0,
        np.array([0.0, -0.0, 448.0, 464.0, 480.0, 1e9, 2.0 ** -10, 2.0 ** -11 * 3]),
    ]).astype(np.float32).astype(np.float64)
    got = F.e4m3_round(x)
    ref = _brute_round(x, t)
    bad = np.where(got != ref)[0]
    assert bad.size == 0, f"rounding differs at {x[bad[:5]]}: {got[bad[:5]]} vs {ref[bad[:5]]}"


def pin_round_torch(F):
    rng = np.random.default_rng(8)
    x = np.concatenate([rng.standard_normal(20000) * 30.0, rng.standard_normal(5000) * 0.01]).astype(np.float32)
    x = np.clip(x, -448.0, 448.0)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = F.e4m3_round(x.astype(np.float64))
    assert np.array_equal(got, ref)


def pin_roundtrip(F):
    t = F.e4m3_table()
    codes = np.array([c for c in range(256) if np.isfinite(t[c])], np.uint8)
    back = F.e4m3_round(t[codes])
    zero = codes == 0x80  # -0 rounds to -0
    assert np.array_equal(back[~zero], codes[~zero])


def pin_scaling(F):
    rng = np.random.default_rng(9)
    x = (rng.standard_normal(4096) * 3.0).astype(np.float32)
    codes, s = F.quantize_per_tensor(x)
    i = int(np.argmax(np.abs(x)))
    assert F.e4m3_decode(codes[i]) == np.sign(x[i]) * 448.0
    assert s == np.float32(np.max(np.abs(x)) / np.float32(448.0))
    assert np.all(np.abs(F.e4m3_decode(codes)) <= 448.0)
    codes4, s4 = F.quantize_per_tensor(x * np.float32(4.0))
    assert np.array_equal(codes4, codes) and s4 == s * 4
    zc, zs = F.quantize_per_tensor(np.zeros(64, np.float32))
    assert zs == 1.0 and np.all(zc == 0)
    # the dequantized tensor is within half a grid step (relative 2^-4) of x
    deq = F.e4m3_decode(codes) * float(s)
    big = np.abs(x) > float(s) * 2.0 ** -6
    assert np.all(np.abs(deq[big] - x[big]) <= np.abs(x[big]) * 2.0 ** -4 + 1e-12)


def pin_projection_integer(F):
    rng = np.random.default_rng(10)
    Hq, Hkv, D, T, K = 2, 1, 4, 5, 24
    N = (Hq + 2 * Hkv) * D
    xi = rng.integers(-8, 9, (T, K))
    wi = rng.integers(-8, 9, (N, K))
    xc, wc = F.e4m3_round(xi.astype(np.float64)), F.e4m3_round(wi.astype(np.float64))
    q, k, v = F.qkv_projection(xc, np.float32(1.0), wc, np.float32(1.0), Hq, Hkv, D)
    Y = xi @ wi.T  # exact integers
    assert np.array_equal(np.concatenate([q.reshape(T, -1), k.reshape(T, -1), v.reshape(T, -1)], 1), Y)
    q2, _, _ = F.qkv_projection(xc, np.float32(0.5), wc, np.float32(4.0), Hq, Hkv, D)
    assert np.array_equal(q2, 2.0 * q)


def pin_projection_head_order(F):
    Hq, Hkv, D, K = 2, 1, 4, 8
    N = (Hq + 2 * Hkv) * D
    x = np.zeros((1, K)); x[0, 0] = 1.0
    w = np.zeros((N, K))
    w[:, 0] = np.arange(1, N + 1)  # output column n carries the value n + 1 (all exact in E4M3 up to 16)
    q, k, v = F.qkv_projection(F.e4m3_round(x), 1.0, F.e4m3_round(w), 1.0, Hq, Hkv, D)
    assert np.array_equal(q[0, 1], [5, 6, 7, 8])          # query head 1 = rows D..2D-1
    assert np.array_equal(k[0, 0], [9, 10, 11, 12])       # key head after the Hq query heads
    assert np.array_equal(v[0, 0], [13, 14, 15, 16])      # value head last


def _rope_complex(x, pos, base):
    """RoPE by complex multiplication: pair (x_2k, x_2k+1) as x_2k + i x_2k+1
    times exp(i pos theta_k), theta_k = base^(-2k/D)."""
    D = x.shape[-1]
    theta = base ** (-2.0 * np.arange(D // 2) / D)
    z = x[..., 0::2] + 1j * x[..., 1::2]
    z = z * np.exp(1j * pos[:, None, None] * theta[None, None, :])
    out = np.empty_like(x)
    out[..., 0::2] = z.real
    out[..., 1::2] = z.imag
    return out


def pin_projection_rope(F):
    rng = np.random.default_rng(11)
    B, S, Hq, Hkv, D, K = 2, 7, 2, 1, 8, 16
    T, N = B * S, (Hq + 2 * Hkv) * D
    xc, sx = F.quantize_per_tensor(rng.standard_normal((T, K)).astype(np.float32))
    wc, sw = F.quantize_per_tensor((rng.standard_normal((N, K)) * 0.1).astype(np.float32))
    offs = torch.tensor([0, 3, 7, 9, 14], dtype=torch.int32)  # documents 3, 4 | 2, 5
    base = 500000.0
    qr, kr, vr = F.qkv_projection_rope(xc, sx, wc, sw, Hq, Hkv, D, B, S, offs, base)
    q, k, v = F.qkv_projection(xc, sx, wc, sw, Hq, Hkv, D)
    pos = np.array([0, 1, 2, 0, 1, 2, 3, 0, 1, 0, 1, 2, 3, 4], np.float64)
    np.testing.assert_allclose(qr.reshape(T, Hq, D), _rope_complex(q, pos, base), rtol=0, atol=1e-12)
    np.testing.assert_allclose(kr.reshape(T, Hkv, D), _rope_complex(k, pos, base), rtol=0, atol=1e-12)
    assert np.array_equal(vr.reshape(T, Hkv, D), v)


GOLDEN = os.path.join(ROOT, "tests", "golden", "e4m3_rounding_examples.txt")


def pin_golden_examples(F):
    """Hand-worked values from the format definition (tests/golden)."""
    rows = [ln.split() for ln in open(GOLDEN) if ln.strip() and not ln.startswith("#")]
    for r in rows:
        value, code = float(r[0]), int(r[1], 16)
        got = int(F.e4m3_round(np.array([value]))[0])
        assert got == code, f"{value}: code {got:#04x}, expected {code:#04x}"


PINS = [pin_table, pin_round_brute, pin_round_torch, pin_roundtrip, pin_scaling, pin_projection_integer,
        pin_projection_head_order, pin_projection_rope, pin_golden_examples]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_fp8_oracle_pin(pin):
    pin(F)


# ---------------------------------------------------------------- planted mistakes

MUTANTS = {
    "bias_8": ("s * (1.0 + m / 8.0) * 2.0 ** (e - 7)", "s * (1.0 + m / 8.0) * 2.0 ** (e - 8)"),
    "round_half_up": ("q = np.round(a / spacing) * spacing", "q = np.floor(a / spacing + 0.5) * spacing"),
    "no_saturation": ("q = np.minimum(q, E4M3_MAX)", "q = np.minimum(q, 480.0)"),
    "two_mantissa_bits": ("_MANT_BITS = 3", "_MANT_BITS = 2"),
    "scale_240": ("s = np.float32(amax / np.float32(E4M3_MAX))", "s = np.float32(amax / np.float32(240.0))"),
    "scale_multiplied": ("quotient = (xf / s)", "quotient = (xf * s)"),
    "w_not_transposed": ("Y = (float(s_x) * float(s_w)) * (X @ W.T)",
                         "Y = (float(s_x) * float(s_w)) * (X @ W.T[::-1])"),
    "kv_swapped": ("k = Y[:, Hq * D:(Hq + Hkv) * D]", "k = Y[:, (Hq + Hkv) * D:]"),
    "v_rotated": ("v.reshape(B, S, Hkv, D))", "O.rope_rotate(v, pos, rope_theta).reshape(B, S, Hkv, D))"),
    "no_doc_positions": ("_, pos = O.doc_layout(doc_offsets, B, S)", "_, pos = O.doc_layout(None, B, S)"),
    "one_scale": ("Y = (float(s_x) * float(s_w))", "Y = (float(s_x))"),
}


def _load_mutant(old, new):
    src = open(FP8_SRC).read()
    assert src.count(old) == 1, old
    mod = types.ModuleType("oracle.fp8_mutant")
    mod.__package__ = "oracle"
    mod.__file__ = FP8_SRC
    exec(compile(src.replace(old, new), FP8_SRC, "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_fp8_pins_catch_planted_mistake(name):
    old, new = MUTANTS[name]
    M = _load_mutant(old, new)
    caught = []
    for pin in PINS:
        try:
            pin(M)
        except Exception:
            caught.append(pin.__name__)
    assert caught, f"no pin caught the planted mistake {name}"
