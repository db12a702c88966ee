"""CPU tests of the C-ABI library: it loads, exports every function the header
declares, and rejects bad arguments on the host before launching anything."""
import ctypes
import os
import re

import pytest

import gqa_attention_rope_b200 as la
from gqa_attention_rope_b200 import build as labuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

OK, INVALID, UNSUPPORTED, WORKSPACE = 0, -1, -2, -3


@pytest.fixture(scope="module")
def lib():
    labuild.build()
    return la.load_library()


def header_functions():
    names = []
    inc = os.path.join(ROOT, "include")
    for fn in os.listdir(inc):
        if fn.endswith(".h"):
            src = open(os.path.join(inc, fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names += re.findall(r"\b(llama_attn_\w+)\s*\(", src)
    return sorted(set(names))


def test_header_symbols_exported(lib):
    names = header_functions()
    assert "llama_attn_prefill" in names and "llama_attn_decode" in names
    for n in names:
        assert hasattr(lib, n), f"{n} declared in include/ but not exported"
    assert set(la.EXPORTED) <= set(names)


def test_status_strings_and_version(lib):
    for st in (0, -1, -2, -3, -4, -5, 7):
        s = lib.llama_attn_status_string(st)
        assert isinstance(s, bytes) and len(s) > 0
    assert lib.llama_attn_version() >= 100


def test_workspace_size(lib):
    f = lib.llama_attn_decode_workspace_size
    assert f(0, 64, 32768, 128) == 0
    assert f(64, 64, 32768, 64) == 0
    n = f(64, 64, 32768, 128)
    nchunk = 32
    assert n >= 64 * 64 * nchunk * 129 * 4 and n % 256 == 0
    assert f(1, 1, 1, 128) >= 129 * 4


FAKE = ctypes.c_void_p(4096)  # never dereferenced: every case below fails validation first


@pytest.mark.parametrize("args,expect", [
    # q, k, v, out, offs, B, S, Hq, Hkv, D, theta
    ((None, FAKE, FAKE, FAKE, None, 1, 128, 8, 2, 128, 5e5), INVALID),
    ((FAKE, FAKE, FAKE, None, None, 1, 128, 8, 2, 128, 5e5), INVALID),
    ((FAKE, FAKE, FAKE, FAKE, None, 0, 128, 8, 2, 128, 5e5), INVALID),
    ((FAKE, FAKE, FAKE, FAKE, None, 1, 0, 8, 2, 128, 5e5), INVALID),
    ((FAKE, FAKE, FAKE, FAKE, None, 1, 128, 8, 3, 128, 5e5), INVALID),
    ((FAKE, FAKE, FAKE, FAKE, None, 1, 128, 8, 2, 128, -1.0), INVALID),
    ((FAKE, FAKE, FAKE, FAKE, None, 1, 128, 8, 2, 64, 5e5), UNSUPPORTED),
    ((ctypes.c_void_p(4098), FAKE, FAKE, FAKE, None, 1, 128, 8, 2, 128, 5e5), INVALID),
])
def test_prefill_rejects(lib, args, expect):
    assert lib.llama_attn_prefill(*args, None) == expect


@pytest.mark.parametrize("args,expect", [
    ((None, FAKE, FAKE, FAKE, None, 1, 128, 8, 2, 64, 5e5), INVALID),
    ((FAKE, FAKE, FAKE, FAKE, None, 1, 128, 8, 2, 63, 5e5), UNSUPPORTED),
    ((FAKE, FAKE, FAKE, FAKE, None, 1, 128, 8, 2, 256, 5e5), UNSUPPORTED),
    ((FAKE, FAKE, FAKE, FAKE, None, 1, 128, 8, 0, 64, 5e5), INVALID),
])
def test_prefill_f32_rejects(lib, args, expect):
    assert lib.llama_attn_prefill_f32(*args, None) == expect


def test_decode_rejects(lib):
    f = lib.llama_attn_decode
    big = 1 << 40
    # q, kc, vc, lens, out, B, Hq, Hkv, D, Lmax, theta, ws, ws_bytes
    assert f(None, FAKE, FAKE, FAKE, FAKE, 2, 16, 2, 128, 64, 5e5, FAKE, big, None) == INVALID
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, 2, 16, 3, 128, 64, 5e5, FAKE, big, None) == INVALID
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, 2, 16, 2, 64, 64, 5e5, FAKE, big, None) == UNSUPPORTED
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, 2, 64, 2, 128, 64, 5e5, FAKE, big, None) == UNSUPPORTED  # G = 32
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, 2, 16, 2, 128, 0, 5e5, FAKE, big, None) == INVALID
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, 2, 16, 2, 128, 64, 5e5, None, big, None) == WORKSPACE
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, 2, 16, 2, 128, 64, 5e5, FAKE, 16, None) == WORKSPACE
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, 2, 16, 2, 128, 64, 5e5, ctypes.c_void_p(4100), big, None) == WORKSPACE


@pytest.mark.parametrize("args,expect", [
    # q, k, v, out, lse, B, Sq, Skv, Hq, Hkv, D, q_pos_a, q_split, q_pos_b, theta
    ((FAKE, FAKE, FAKE, FAKE, None, 1, 256, 1024, 8, 2, 128, 64, 128, 512, 5e5), INVALID),   # position not /128
    ((FAKE, FAKE, FAKE, FAKE, None, 1, 256, 1024, 8, 2, 128, 0, 100, 512, 5e5), INVALID),    # split not /128
    ((FAKE, FAKE, FAKE, FAKE, None, 1, 256, 1024, 8, 2, 128, 0, 384, 0, 5e5), INVALID),      # split > Sq
    ((FAKE, FAKE, FAKE, FAKE, None, 1, 256, 1024, 8, 2, 128, 0, 128, 1000, 5e5), INVALID),   # chunk b past Skv
    ((FAKE, FAKE, FAKE, FAKE, None, 1, 256, 1024, 8, 2, 128, 1024, 128, 0, 5e5), INVALID),   # chunk a past Skv
    ((FAKE, FAKE, FAKE, FAKE, None, 1, 256, 0, 8, 2, 128, 0, 128, 0, 5e5), INVALID),         # Skv = 0
    ((None, FAKE, FAKE, FAKE, None, 1, 256, 1024, 8, 2, 128, 0, 128, 512, 5e5), INVALID),
    ((FAKE, FAKE, FAKE, FAKE, None, 1, 256, 1024, 8, 2, 64, 0, 128, 512, 5e5), UNSUPPORTED),
])
def test_prefill_cp_rejects(lib, args, expect):
    assert lib.llama_attn_prefill_cp(*args, None) == expect


def test_fp8_entries_reject(lib):
    q = lib.llama_attn_quantize_e4m3
    assert q(None, 64, FAKE, FAKE, None) == INVALID
    assert q(FAKE, 12, FAKE, FAKE, None) == INVALID              # n % 8 != 0
    assert q(FAKE, 0, FAKE, FAKE, None) == INVALID
    assert q(ctypes.c_void_p(4104), 64, FAKE, FAKE, None) == INVALID  # x not 16-byte aligned
    g = lib.llama_attn_qkv_fp8_rope
    # x, s_x, w, s_w, q, k, v, offs, B, S, d_model, Hq, Hkv, D, theta
    assert g(None, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, 1, 128, 256, 4, 2, 128, 5e5, None) == INVALID
    assert g(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, 1, 128, 200, 4, 2, 128, 5e5, None) == UNSUPPORTED
    assert g(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, 1, 128, 256, 4, 2, 64, 5e5, None) == UNSUPPORTED
    assert g(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, 0, 128, 256, 4, 2, 128, 5e5, None) == INVALID
    assert g(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, 1, 128, 256, 4, 2, 128, 0.0, None) == INVALID
    r = lib.llama_attn_prefill_rotated
    assert r(None, FAKE, FAKE, FAKE, None, None, 1, 128, 8, 2, 128, None) == INVALID
    assert r(FAKE, FAKE, FAKE, FAKE, None, None, 1, 128, 8, 2, 64, None) == UNSUPPORTED


def test_prefill_workspace_and_table_sizes(lib):
    ws = lib.llama_attn_prefill_workspace_size
    assert ws(0, 128, 8, 128) == 0 and ws(1, 128, 8, 64) == 0 and ws(1, 0, 8, 128) == 0
    B, S, Hkv = 4, 8192, 8
    n = ws(B, S, Hkv, 128)
    # counter (256 B) + document starts (B*S int32) + rotated keys (B*S*Hkv*128 bf16), each 256-aligned
    assert n == 256 + B * S * 4 + B * S * Hkv * 256
    assert ws(1, 1, 1, 128) == 256 + 256 + 256
    ts = lib.llama_attn_rope_table_size
    assert ts(131072, 128) == 131072 * 64 * 8
    assert ts(0, 128) == 0 and ts(16, 7) == 0 and ts(16, 130) == 0


T16 = ctypes.c_void_p(4096 * 16)  # 16- and 256-byte aligned, never dereferenced


def _ws_args(**kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, out=FAKE, lse=None, offs=None, B=1, S=256, Hq=8, Hkv=2, D=128, table=T16,
             rows=256, kc=None, vc=None, Lmax=0, ws=T16, ws_bytes=1 << 40)
    a.update(kw)
    return tuple(a.values())


@pytest.mark.parametrize("kw,expect", [
    (dict(ws_bytes=256 + 256 * 4 + 256 * 2 * 256 - 1), WORKSPACE),   # one byte short
    (dict(ws=None), WORKSPACE),
    (dict(ws=ctypes.c_void_p(4096 + 16)), WORKSPACE),                  # not 256-byte aligned
    (dict(table=None), INVALID),
    (dict(rows=255), INVALID),                                        # table shorter than S positions
    (dict(table=ctypes.c_void_p(4104)), INVALID),                     # table not 16-byte aligned
    (dict(q=None), INVALID),
    (dict(Hkv=3), INVALID),
    (dict(D=64), UNSUPPORTED),
    (dict(kc=FAKE), INVALID),                                         # one cache without the other
    (dict(kc=FAKE, vc=FAKE, Lmax=100), INVALID),                      # Lmax < S
])
def test_prefill_ws_rejects_before_any_launch(lib, kw, expect):
    """Every failing check returns before the library touches CUDA (this host
    has no GPU, so any CUDA call would report LLAMA_ATTN_ERR_CUDA instead)."""
    assert lib.llama_attn_prefill_ws(*_ws_args(**kw), None) == expect


def test_prefill_cp_ws_rejects(lib):
    f = lib.llama_attn_prefill_cp_ws
    need = lib.llama_attn_prefill_workspace_size(1, 1024, 2, 128)
    # q, k, v, out, lse, B, Sq, Skv, Hq, Hkv, D, q_pos_a, q_split, q_pos_b, table, rows, ws, ws_bytes
    assert f(FAKE, FAKE, FAKE, FAKE, None, 1, 256, 1024, 8, 2, 128, 0, 128, 512, T16, 1024, T16, need - 1,
             None) == WORKSPACE
    assert f(FAKE, FAKE, FAKE, FAKE, None, 1, 256, 1024, 8, 2, 128, 0, 128, 512, T16, 1023, T16, need,
             None) == INVALID  # rows < Skv
    assert f(FAKE, FAKE, FAKE, FAKE, None, 1, 256, 1024, 8, 2, 128, 64, 128, 512, T16, 1024, T16, need,
             None) == INVALID  # position not a multiple of 128


def test_rope_table_build_rejects(lib):
    f = lib.llama_attn_rope_table_build
    need = lib.llama_attn_rope_table_size(1000, 128)
    assert f(None, need, 1000, 128, 5e5, None) == INVALID
    assert f(T16, need - 1, 1000, 128, 5e5, None) == WORKSPACE
    assert f(T16, need, 1000, 128, 0.0, None) == INVALID
    assert f(T16, need, 0, 128, 5e5, None) == INVALID
    assert f(ctypes.c_void_p(4100), need, 1000, 128, 5e5, None) == INVALID


def test_binding_wraps_every_exported_name():
    for n in la.EXPORTED:
        assert callable(getattr(la, n, None)), f"no Python wrapper named {n}"


def test_python_binding_fails_loudly_without_library(tmp_path):
    with pytest.raises(RuntimeError, match="not found"):
        la.load_library(str(tmp_path / "missing.so"))


def test_shard_units_partition():
    for n in (0, 1, 7, 32, 100):
        for w in (1, 2, 3, 8):
            seen = []
            for r in range(w):
                rg = la.shard_units(n, w, r)
                seen += list(rg)
                assert len(rg) in (n // w, n // w + 1)
            assert seen == list(range(n))
