"""Float64 CPU oracle of the FP8 QKV projection with RoPE.

TEST INFRASTRUCTURE ONLY: imported by the tests and the smoke check, never by
the library itself.

What it follows ("Llama 3.1 Architecture: Dense Scaling to 405B and 128K
Context", section "FP8 Quantization: Fitting 405B on an 8xH100 Node"):
  - E4M3: 1 sign, 4 exponent, 3 mantissa bits, largest magnitude 448
    ("FP8 Format Breakdown (E4M3 vs E5M2)").
  - Per-tensor dynamic scaling: X_fp8 = clip(round(X / s_X), -448, 448),
    W_fp8 likewise, Y ~= (s_X * s_W) * (X_fp8 . W_fp8) ("Scaling Formulation
    and Tensor Core Acceleration"); the attention QKV projection is one of the
    GEMMs quantized this way (the figure in the same section).
Readings (the page leaves these open):
  - round() is round-to-nearest-even onto the E4M3 grid (the grid is not the
    integers), and clip saturates at +-448.
  - The dynamic per-tensor scale is s = amax(|X|) / 448 (so the largest
    magnitude maps to 448), formed in float32; s = 1 when X is all zeros.
    X / s is a float32 division, so the rounding decision is taken on the
    same float32 quotient as the kernel's.
  - W is stored [N, K] (output features by input features), the transpose of
    the page's K x N matrix; its N rows are the Hq query heads, then the Hkv
    key heads, then the Hkv value heads, D rows each.
  - RoPE is then applied to the query and key heads at each token's document
    position (the attention's rotation, here moved into the projection).
"""
from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0
_MIN_NORMAL_EXP = -6   # 2^-6 smallest normal
_MANT_BITS = 3


def e4m3_table() -> np.ndarray:
    """Value of each of the 256 codes, decoded from the format: bias 7,
    exponent field 0 = subnormal (m/8 * 2^-6), S.1111.111 = NaN, no infinity."""
    vals = np.empty(256, np.float64)
    for code in range(256):
        s = -1.0 if code & 0x80 else 1.0
        e = (code >> 3) & 0xF
        m = code & 0x7
        if e == 0xF and m == 0x7:
            vals[code] = np.nan
        elif e == 0:
            vals[code] = s * (m / 8.0) * 2.0 ** _MIN_NORMAL_EXP
        else:
            vals[code] = s * (1.0 + m / 8.0) * 2.0 ** (e - 7)
    return vals


def e4m3_round(x) -> np.ndarray:
    """Codes (uint8) of x rounded to nearest-even on the E4M3 grid and
    saturated to +-448. NaN maps to 0x7F."""
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    sign = np.signbit(x)
    # spacing of the grid at |x|: 2^(e-3) in binade [2^e, 2^(e+1)), 2^-9 below 2^-6
    _, e2 = np.frexp(np.where(a > 0, a, 1.0))  # a = f * 2^e2, f in [0.5, 1)
    e = np.maximum(e2 - 1, _MIN_NORMAL_EXP)
    spacing = np.ldexp(1.0, e - _MANT_BITS)
    q = np.round(a / spacing) * spacing      # numpy rounds halves to even
    q = np.minimum(q, E4M3_MAX)
    # encode
    codes = np.zeros(x.shape, np.uint8)
    nz = q > 0
    _, qe2 = np.frexp(np.where(nz, q, 1.0))
    qe = qe2 - 1
    normal = nz & (qe >= _MIN_NORMAL_EXP)
    sub = nz & ~normal
    mant_n = np.where(normal, np.round((q / np.ldexp(1.0, qe) - 1.0) * 8.0), 0).astype(np.int64)
    exp_n = np.where(normal, qe + 7, 0).astype(np.int64)
    mant_s = np.where(sub, np.round(q / 2.0 ** -9), 0).astype(np.int64)
    code = np.where(normal, (exp_n << 3) | mant_n, mant_s)
    codes = (code.astype(np.int64) | (sign.astype(np.int64) << 7)).astype(np.uint8)
    codes = np.where(np.isnan(x), np.uint8(0x7F), codes)
    return codes


def e4m3_decode(codes) -> np.ndarray:
    return e4m3_table()[np.asarray(codes, dtype=np.uint8)]


def quantize_per_tensor(x):
    """(codes uint8, scale float32) of x (any float array) under the
    per-tensor dynamic scale s = amax / 448."""
    xf = np.asarray(x, dtype=np.float32)
    amax = np.float32(np.max(np.abs(xf))) if xf.size else np.float32(0.0)
    s = np.float32(amax / np.float32(E4M3_MAX)) if amax > 0 else np.float32(1.0)
    quotient = (xf / s).astype(np.float32)   # float32 division, as on the GPU
    return e4m3_round(quotient), s


def qkv_projection(x_codes, s_x, w_codes, s_w, Hq: int, Hkv: int, D: int):
    """Un-rotated (Q, K, V) in float64 from FP8 codes: Y = (s_x s_w) X W^T
    with X [T, K] and W [N, K], N = (Hq + 2 Hkv) D. Shapes [T, H, D]."""
    X = e4m3_decode(x_codes)
    W = e4m3_decode(w_codes)
    Y = (float(s_x) * float(s_w)) * (X @ W.T)
    T = X.shape[0]
    q = Y[:, :Hq * D].reshape(T, Hq, D)
    k = Y[:, Hq * D:(Hq + Hkv) * D].reshape(T, Hkv, D)
    v = Y[:, (Hq + Hkv) * D:].reshape(T, Hkv, D)
    return q, k, v


def qkv_projection_rope(x_codes, s_x, w_codes, s_w, Hq: int, Hkv: int, D: int, B: int, S: int,
                        doc_offsets=None, rope_theta: float = 500000.0):
    """(Q rotated, K rotated, V) in float64, each [B, S, H, D]: the projection
    followed by RoPE at each token's document position."""
    from . import oracle as O
    q, k, v = qkv_projection(x_codes, s_x, w_codes, s_w, Hq, Hkv, D)
    _, pos = O.doc_layout(doc_offsets, B, S)
    pos = pos.astype(np.float64)
    qr = O.rope_rotate(q, pos, rope_theta)
    kr = O.rope_rotate(k, pos, rope_theta)
    return (qr.reshape(B, S, Hq, D), kr.reshape(B, S, Hkv, D), v.reshape(B, S, Hkv, D))
