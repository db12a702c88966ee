"""Python front end of the float64 CPU oracle (``oracle.c``).

TEST INFRASTRUCTURE ONLY: imported by the tests, the smoke check and the
bench's CPU-baseline / reference legs, never by the library itself.

Inputs are taken as torch CPU tensors or numpy arrays of any float dtype and
upcast exactly to float64 (bf16 and fp32 both embed exactly in float64), so
the oracle sees the very bit patterns the GPU receives.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so (gcc, OpenMP, no fast-math)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
                               "-fno-fast-math", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def load_library(path: str):
    """Load an oracle shared object and declare its signatures."""
    lib = ctypes.CDLL(path)
    P = ctypes.c_void_p
    i32, i64, f64 = ctypes.c_int, ctypes.c_int64, ctypes.c_double
    lib.oracle_num_threads.restype = i32
    lib.oracle_rope_freqs.argtypes = [i32, f64, P]
    lib.oracle_rope_rotate.argtypes = [P, i64, i32, i32, P, f64, P]
    lib.oracle_doc_layout.argtypes = [P, i32, i32, P, P]
    lib.oracle_doc_layout.restype = i32
    lib.oracle_prefill.argtypes = [P, P, P, P, P, i32, i32, i32, i32, i32, f64, P, i64, P]
    lib.oracle_prefill_weights.argtypes = [P, P, P, P, i32, i32, i32, i32, i32, f64, i32, i32, i32, P]
    lib.oracle_decode.argtypes = [P, P, P, P, i32, i32, i32, i32, i32, f64, P]
    if hasattr(lib, "oracle_prefill_lse"):
        lib.oracle_prefill_lse.argtypes = [P, P, P, P, P, i32, i32, i32, i32, i32, f64, P, i64, P, P]
    return lib


def _get():
    global _lib
    with _lock:
        if _lib is None:
            _lib = load_library(build())
    return _lib


def _f64(x) -> np.ndarray:
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().to("cpu", torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _i32(x) -> np.ndarray:
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().to("cpu", torch.int32).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(x, dtype=np.int32))


def _take_rows(x, rows_arr: np.ndarray):
    try:
        import torch
        if isinstance(x, torch.Tensor):
            return x[torch.from_numpy(rows_arr)]
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(x)[rows_arr]


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def num_threads(lib=None) -> int:
    return int((lib or _get()).oracle_num_threads())


def rope_freqs(D: int, base: float, lib=None) -> np.ndarray:
    out = np.empty(D // 2, np.float64)
    (lib or _get()).oracle_rope_freqs(D, float(base), _p(out))
    return out


def rope_rotate(x, pos, base: float, lib=None) -> np.ndarray:
    """x: [n, H, D] (or [n, D]); pos: [n] positions (float). Returns rotated x."""
    x = _f64(x)
    squeeze = x.ndim == 2
    if squeeze:
        x = x[:, None, :]
    n, H, D = x.shape
    pos = np.ascontiguousarray(np.asarray(pos, dtype=np.float64).reshape(n))
    y = np.empty_like(x)
    (lib or _get()).oracle_rope_rotate(_p(x), n, H, D, _p(pos), float(base), _p(y))
    return y[:, 0, :] if squeeze else y


def doc_layout(doc_offsets, B: int, S: int, lib=None):
    """(doc_start, pos) int32 arrays of length B*S, or raises ValueError."""
    ds = np.empty(B * S, np.int32)
    pos = np.empty(B * S, np.int32)
    offs = None if doc_offsets is None else _i32(doc_offsets)
    rc = (lib or _get()).oracle_doc_layout(None if offs is None else _p(offs), B, S, _p(ds), _p(pos))
    if rc != 0:
        raise ValueError("malformed doc_offsets")
    return ds, pos


def prefill(q, k, v, doc_offsets=None, rope_theta: float = 500000.0, rows=None, lib=None,
            layout=None) -> np.ndarray:
    """Attention output in float64.

    q: [B, S, Hq, D]; k, v: [B, S, Hkv, D]. rows: optional 1-D array of
    flattened token indices b*S+i; then the result is [len(rows), Hq, D],
    otherwise [B, S, Hq, D]. ``layout`` may pass precomputed (doc_start, pos)."""
    lib = lib or _get()
    B, S, Hq, D = q.shape
    Hkv = k.shape[2]
    if Hq % Hkv != 0:
        raise ValueError("Hq must be a multiple of Hkv")
    ds, pos = layout if layout is not None else doc_layout(doc_offsets, B, S, lib)
    kf, vf = _f64(k), _f64(v)
    if rows is None:
        qf = _f64(q).reshape(B * S, Hq, D)
        n_rows = B * S
        rows_arr = None
    else:
        rows_arr = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
        n_rows = rows_arr.shape[0]
        qf = _f64(_take_rows(q.reshape(B * S, Hq, D), rows_arr))
    out = np.empty((n_rows, Hq, D), np.float64)
    lib.oracle_prefill(_p(qf), _p(kf), _p(vf), _p(ds), _p(pos), B, S, Hq, Hkv, D, float(rope_theta),
                       None if rows_arr is None else _p(rows_arr), n_rows, _p(out))
    return out.reshape(B, S, Hq, D) if rows is None else out


def prefill_lse(q, k, v, doc_offsets=None, rope_theta: float = 500000.0, rows=None, lib=None):
    """(out, lse): attention output and the per-row, per-head log-sum-exp of
    the visible scaled scores (natural log). Shapes as in prefill; lse is
    [B, S, Hq] or [len(rows), Hq]."""
    lib = lib or _get()
    B, S, Hq, D = q.shape
    Hkv = k.shape[2]
    ds, pos = doc_layout(doc_offsets, B, S, lib)
    kf, vf = _f64(k), _f64(v)
    if rows is None:
        qf = _f64(q).reshape(B * S, Hq, D)
        n_rows, rows_arr = B * S, None
    else:
        rows_arr = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
        n_rows = rows_arr.shape[0]
        qf = _f64(_take_rows(q.reshape(B * S, Hq, D), rows_arr))
    out = np.empty((n_rows, Hq, D), np.float64)
    lse = np.empty((n_rows, Hq), np.float64)
    lib.oracle_prefill_lse(_p(qf), _p(kf), _p(vf), _p(ds), _p(pos), B, S, Hq, Hkv, D, float(rope_theta),
                           None if rows_arr is None else _p(rows_arr), n_rows, _p(out), _p(lse))
    if rows is None:
        return out.reshape(B, S, Hq, D), lse.reshape(B, S, Hq)
    return out, lse


def prefill_weights(q, k, b: int, h: int, i: int, doc_offsets=None, rope_theta: float = 500000.0,
                    lib=None) -> np.ndarray:
    """Attention weights of query (b, h, i) over the S keys of batch row b."""
    lib = lib or _get()
    B, S, Hq, D = q.shape
    Hkv = k.shape[2]
    ds, pos = doc_layout(doc_offsets, B, S, lib)
    qf, kf = _f64(q), _f64(k)
    w = np.empty(S, np.float64)
    lib.oracle_prefill_weights(_p(qf), _p(kf), _p(ds), _p(pos), B, S, Hq, Hkv, D, float(rope_theta),
                               b, h, i, _p(w))
    return w


def decode(q, kcache, vcache, cache_lens, rope_theta: float = 500000.0, lib=None,
           max_f64_bytes: int = 1 << 31) -> np.ndarray:
    """Decode output in float64. q: [B, Hq, D]; caches [B, Hkv, Lmax, D] (pre-rotated keys).

    Only cache rows below max(cache_lens) are read, and sequences are handed
    to the C code in groups whose float64 copies stay under ``max_f64_bytes``."""
    lib = lib or _get()
    B, Hq, D = q.shape
    Hkv = kcache.shape[1]
    lens = _i32(cache_lens)
    out = np.empty((B, Hq, D), np.float64)
    b0 = 0
    while b0 < B:
        b1 = b0 + 1
        lm = max(int(lens[b0]), 1)
        while b1 < B:
            lm2 = max(lm, int(lens[b1]))
            if (b1 + 1 - b0) * Hkv * lm2 * D * 16 > max_f64_bytes:
                break
            lm = lm2
            b1 += 1
        qf = _f64(q[b0:b1])
        kf = _f64(kcache[b0:b1, :, :lm])
        vf = _f64(vcache[b0:b1, :, :lm])
        ln = np.ascontiguousarray(lens[b0:b1])
        o = np.empty((b1 - b0, Hq, D), np.float64)
        lib.oracle_decode(_p(qf), _p(kf), _p(vf), _p(ln), b1 - b0, Hq, Hkv, D, lm, float(rope_theta),
                          _p(o))
        out[b0:b1] = o
        b0 = b1
    return out
