"""Python binding of the B200 attention library (libllama_attn.so).

The functions carry the names of the C ABI in include/llama_attn.h and only
marshal arguments: shapes are read off the tensors, device pointers and the
current CUDA stream are passed through ctypes, and a negative status becomes
a RuntimeError. Every step of the computation runs in the library's CUDA
kernels; there is no CPU or PyTorch fallback, and calling an op without the
built library raises.
"""
from __future__ import annotations

import ctypes
import os
import threading

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libllama_attn.so")

EXPORTED = (
    "llama_attn_prefill",
    "llama_attn_prefill_f32",
    "llama_attn_decode_workspace_size",
    "llama_attn_decode",
    "llama_attn_status_string",
    "llama_attn_get_device_error",
    "llama_attn_version",
    "llama_attn_profile_begin",
    "llama_attn_profile_end",
    "llama_attn_decode_noalloc",
    "llama_attn_prefill_ex",
    "llama_attn_decode_paged",
    "llama_attn_prefill_cp",
    "llama_attn_prefill_rotated",
    "llama_attn_quantize_e4m3",
    "llama_attn_qkv_fp8_rope",
    "llama_attn_rope_table_size",
    "llama_attn_rope_table_build",
    "llama_attn_prefill_workspace_size",
    "llama_attn_prefill_ws",
    "llama_attn_prefill_cp_ws",
)

DEVERR_TIMEOUT = 0x1
DEVERR_DOC_OFFSETS = 0x2
DEVERR_CACHE_LEN = 0x4
DEVERR_BLOCK_TABLE = 0x8

_lock = threading.Lock()
_lib = None


class LlamaAttnError(RuntimeError):
    def __init__(self, fn: str, status: int, text: str):
        super().__init__(f"{fn} failed: status {status} ({text})")
        self.status = status


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load the shared library and declare the C signatures. Raises if missing."""
    if not os.path.exists(path):
        raise RuntimeError(
            f"libllama_attn.so not found at {path}; build it with "
            "`python -m gqa_attention_rope_b200.build` (nvcc, sm_100a)")
    lib = ctypes.CDLL(path)
    P, I, F, Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    lib.llama_attn_prefill.argtypes = [P, P, P, P, P, I, I, I, I, I, F, P]
    lib.llama_attn_prefill.restype = I
    lib.llama_attn_prefill_f32.argtypes = [P, P, P, P, P, I, I, I, I, I, F, P]
    lib.llama_attn_prefill_f32.restype = I
    lib.llama_attn_decode_workspace_size.argtypes = [I, I, I, I]
    lib.llama_attn_decode_workspace_size.restype = Z
    lib.llama_attn_decode.argtypes = [P, P, P, P, P, I, I, I, I, I, F, P, Z, P]
    lib.llama_attn_decode.restype = I
    lib.llama_attn_status_string.argtypes = [I]
    lib.llama_attn_status_string.restype = ctypes.c_char_p
    lib.llama_attn_get_device_error.argtypes = [P]
    lib.llama_attn_get_device_error.restype = I
    lib.llama_attn_version.argtypes = []
    lib.llama_attn_version.restype = I
    lib.llama_attn_profile_begin.argtypes = []
    lib.llama_attn_profile_begin.restype = I
    lib.llama_attn_profile_end.argtypes = [P, P, P]
    lib.llama_attn_profile_end.restype = I
    lib.llama_attn_decode_noalloc.argtypes = [P, P, P, P, P, I, I, I, I, I, F, P]
    lib.llama_attn_decode_noalloc.restype = I
    lib.llama_attn_prefill_ex.argtypes = [P, P, P, P, P, P, I, I, I, I, I, F, P, P, I, P]
    lib.llama_attn_prefill_ex.restype = I
    lib.llama_attn_decode_paged.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, I, F, P, Z, P]
    lib.llama_attn_decode_paged.restype = I
    lib.llama_attn_prefill_cp.argtypes = [P, P, P, P, P, I, I, I, I, I, I, I, I, I, F, P]
    lib.llama_attn_prefill_cp.restype = I
    lib.llama_attn_prefill_rotated.argtypes = [P, P, P, P, P, P, I, I, I, I, I, P]
    lib.llama_attn_prefill_rotated.restype = I
    lib.llama_attn_quantize_e4m3.argtypes = [P, ctypes.c_int64, P, P, P]
    lib.llama_attn_quantize_e4m3.restype = I
    lib.llama_attn_qkv_fp8_rope.argtypes = [P, P, P, P, P, P, P, P, I, I, I, I, I, I, F, P]
    lib.llama_attn_qkv_fp8_rope.restype = I
    lib.llama_attn_rope_table_size.argtypes = [I, I]
    lib.llama_attn_rope_table_size.restype = Z
    lib.llama_attn_rope_table_build.argtypes = [P, Z, I, I, F, P]
    lib.llama_attn_rope_table_build.restype = I
    lib.llama_attn_prefill_workspace_size.argtypes = [I, I, I, I]
    lib.llama_attn_prefill_workspace_size.restype = Z
    lib.llama_attn_prefill_ws.argtypes = [P, P, P, P, P, P, I, I, I, I, I, P, I, P, P, I, P, Z, P]
    lib.llama_attn_prefill_ws.restype = I
    lib.llama_attn_prefill_cp_ws.argtypes = [P, P, P, P, P, I, I, I, I, I, I, I, I, I, P, I, P, Z, P]
    lib.llama_attn_prefill_cp_ws.restype = I
    return lib


def lib() -> ctypes.CDLL:
    global _lib
    with _lock:
        if _lib is None:
            _lib = load_library()
    return _lib


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _check(fn: str, status: int):
    if status != 0:
        raise LlamaAttnError(fn, status, lib().llama_attn_status_string(status).decode())


def _require(cond: bool, msg: str):
    if not cond:
        raise ValueError(msg)


def llama_attn_status_string(status: int) -> str:
    return lib().llama_attn_status_string(int(status)).decode()


def llama_attn_version() -> int:
    return int(lib().llama_attn_version())


def llama_attn_get_device_error(stream=None) -> int:
    st = lib().llama_attn_get_device_error(_stream(stream))
    if st < 0:
        _check("llama_attn_get_device_error", st)
    return st


def llama_attn_profile_begin() -> None:
    _check("llama_attn_profile_begin", lib().llama_attn_profile_begin())


def llama_attn_profile_end():
    """Returns (main_kernel_ms_total, main_kernels_timed, kernels_launched)."""
    ms = ctypes.c_double(0.0)
    n_main = ctypes.c_int(0)
    n_all = ctypes.c_int(0)
    _check("llama_attn_profile_end", lib().llama_attn_profile_end(ctypes.byref(ms), ctypes.byref(n_main),
                                                                 ctypes.byref(n_all)))
    return ms.value, n_main.value, n_all.value


def llama_attn_prefill(q, k, v, out=None, doc_offsets=None, rope_theta: float = 500000.0, stream=None):
    """bf16 prefill. q [B,S,Hq,D], k/v [B,S,Hkv,D] contiguous CUDA bf16; returns out [B,S,Hq,D]."""
    import torch
    _require(q.dim() == 4 and k.dim() == 4 and v.dim() == 4, "q, k, v must be [B, S, H, D]")
    for t in (q, k, v):
        _require(t.is_cuda and t.dtype == torch.bfloat16 and t.is_contiguous(), "bf16 contiguous CUDA tensors expected")
    B, S, Hq, D = q.shape
    Hkv = k.shape[2]
    _require(k.shape == (B, S, Hkv, D) and v.shape == k.shape, "k and v must be [B, S, Hkv, D]")
    if out is None:
        out = torch.empty_like(q)
    _require(out.shape == q.shape and out.dtype == torch.bfloat16 and out.is_contiguous(), "bad out")
    if doc_offsets is not None:
        _require(doc_offsets.is_cuda and doc_offsets.dtype == torch.int32, "doc_offsets: int32 CUDA tensor")
    st = lib().llama_attn_prefill(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(doc_offsets), B, S, Hq, Hkv, D,
                                  float(rope_theta), _stream(stream))
    _check("llama_attn_prefill", st)
    return out


def llama_attn_prefill_ex(q, k, v, out=None, lse=None, doc_offsets=None, rope_theta: float = 500000.0,
                          kcache=None, vcache=None, stream=None):
    """bf16 prefill that can also return the per-row log-sum-exp (``lse``,
    float32 [B, S, Hq]) and append rotated K and V to a decode-layout cache
    (``kcache``/``vcache`` [B, Hkv, Lmax, D]). Returns (out, lse)."""
    import torch
    _require(q.dim() == 4 and k.dim() == 4 and v.dim() == 4, "q, k, v must be [B, S, H, D]")
    for t in (q, k, v):
        _require(t.is_cuda and t.dtype == torch.bfloat16 and t.is_contiguous(), "bf16 contiguous CUDA tensors expected")
    B, S, Hq, D = q.shape
    Hkv = k.shape[2]
    _require(k.shape == (B, S, Hkv, D) and v.shape == k.shape, "k and v must be [B, S, Hkv, D]")
    if out is None:
        out = torch.empty_like(q)
    if lse is not None:
        _require(lse.is_cuda and lse.dtype == torch.float32 and lse.is_contiguous() and lse.shape == (B, S, Hq),
                 "lse: float32 [B, S, Hq]")
    Lmax = 0
    if kcache is not None or vcache is not None:
        _require(kcache is not None and vcache is not None and kcache.shape == vcache.shape, "kcache and vcache")
        for t in (kcache, vcache):
            _require(t.is_cuda and t.dtype == torch.bfloat16 and t.is_contiguous(), "bf16 contiguous caches")
        _require(kcache.shape[0] == B and kcache.shape[1] == Hkv and kcache.shape[3] == D, "cache shape")
        Lmax = kcache.shape[2]
    if doc_offsets is not None:
        _require(doc_offsets.is_cuda and doc_offsets.dtype == torch.int32, "doc_offsets: int32 CUDA tensor")
    st = lib().llama_attn_prefill_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(doc_offsets), B, S, Hq,
                                     Hkv, D, float(rope_theta), _ptr(kcache), _ptr(vcache), Lmax, _stream(stream))
    _check("llama_attn_prefill_ex", st)
    return out, lse


def llama_attn_prefill_cp(q, k, v, q_pos_a: int, q_split: int, q_pos_b: int = 0, out=None, lse=None,
                          rope_theta: float = 500000.0, stream=None):
    """bf16 prefill of query chunks against a whole sequence (one step of
    context parallelism). q [B,Sq,Hq,D]: rows [0, q_split) sit at global
    positions q_pos_a.., rows [q_split, Sq) at q_pos_b..; k/v [B,Skv,Hkv,D]
    are the whole sequence. Returns (out, lse)."""
    import torch
    _require(q.dim() == 4 and k.dim() == 4 and v.dim() == 4, "q, k, v must be [B, S, H, D]")
    for t in (q, k, v):
        _require(t.is_cuda and t.dtype == torch.bfloat16 and t.is_contiguous(), "bf16 contiguous CUDA tensors expected")
    B, Sq, Hq, D = q.shape
    Skv, Hkv = k.shape[1], k.shape[2]
    _require(k.shape == (B, Skv, Hkv, D) and v.shape == k.shape, "k and v must be [B, Skv, Hkv, D]")
    if out is None:
        out = torch.empty_like(q)
    _require(out.shape == q.shape and out.dtype == torch.bfloat16 and out.is_contiguous(), "bad out")
    if lse is not None:
        _require(lse.is_cuda and lse.dtype == torch.float32 and lse.is_contiguous() and lse.shape == (B, Sq, Hq),
                 "lse: float32 [B, Sq, Hq]")
    st = lib().llama_attn_prefill_cp(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, Sq, Skv, Hq, Hkv, D,
                                     int(q_pos_a), int(q_split), int(q_pos_b), float(rope_theta), _stream(stream))
    _check("llama_attn_prefill_cp", st)
    return out, lse


def llama_attn_rope_table_size(maxpos: int, D: int = 128) -> int:
    return int(lib().llama_attn_rope_table_size(int(maxpos), int(D)))


def llama_attn_rope_table_build(maxpos: int, D: int = 128, rope_theta: float = 500000.0, table=None, device=None,
                                stream=None):
    """Caller-owned RoPE table for the *_ws entry points: float32 [maxpos, D/2, 2]
    holding (cos, sin) of p * theta_k. Allocated here unless ``table`` is given."""
    import torch
    need = llama_attn_rope_table_size(maxpos, D)
    _require(need > 0, "maxpos >= 1 and even D in [2, 128]")
    if table is None:
        table = torch.empty(maxpos, D // 2, 2, dtype=torch.float32,
                            device=device if device is not None else torch.cuda.current_device())
    _require(table.is_cuda and table.is_contiguous(), "table: contiguous CUDA tensor")
    st = lib().llama_attn_rope_table_build(_ptr(table), table.numel() * table.element_size(), int(maxpos), int(D),
                                           float(rope_theta), _stream(stream))
    _check("llama_attn_rope_table_build", st)
    return table


def llama_attn_prefill_workspace_size(B: int, S: int, Hkv: int, D: int = 128) -> int:
    return int(lib().llama_attn_prefill_workspace_size(int(B), int(S), int(Hkv), int(D)))


def _table_rows(table):
    return table.shape[0] if table.dim() >= 1 else 0


def llama_attn_prefill_ws(q, k, v, rope_table, workspace, out=None, lse=None, doc_offsets=None, kcache=None,
                          vcache=None, stream=None):
    """llama_attn_prefill_ex with caller-owned memory: ``rope_table`` from
    llama_attn_rope_table_build (rows >= S) and ``workspace`` a CUDA buffer of at
    least llama_attn_prefill_workspace_size(B, S, Hkv) bytes. The call allocates
    nothing and does not synchronise (``out`` is allocated here only when not
    given). Returns (out, lse)."""
    import torch
    _require(q.dim() == 4 and k.dim() == 4 and v.dim() == 4, "q, k, v must be [B, S, H, D]")
    for t in (q, k, v):
        _require(t.is_cuda and t.dtype == torch.bfloat16 and t.is_contiguous(), "bf16 contiguous CUDA tensors expected")
    B, S, Hq, D = q.shape
    Hkv = k.shape[2]
    _require(k.shape == (B, S, Hkv, D) and v.shape == k.shape, "k and v must be [B, S, Hkv, D]")
    if out is None:
        out = torch.empty_like(q)
    _require(out.shape == q.shape and out.dtype == torch.bfloat16 and out.is_contiguous(), "bad out")
    if lse is not None:
        _require(lse.is_cuda and lse.dtype == torch.float32 and lse.is_contiguous() and lse.shape == (B, S, Hq),
                 "lse: float32 [B, S, Hq]")
    Lmax = 0
    if kcache is not None or vcache is not None:
        _require(kcache is not None and vcache is not None and kcache.shape == vcache.shape, "kcache and vcache")
        _require(kcache.shape[0] == B and kcache.shape[1] == Hkv and kcache.shape[3] == D, "cache shape")
        Lmax = kcache.shape[2]
    if doc_offsets is not None:
        _require(doc_offsets.is_cuda and doc_offsets.dtype == torch.int32, "doc_offsets: int32 CUDA tensor")
    _require(rope_table.is_cuda and workspace.is_cuda, "rope_table and workspace: CUDA tensors")
    st = lib().llama_attn_prefill_ws(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(doc_offsets), B, S, Hq,
                                     Hkv, D, _ptr(rope_table), _table_rows(rope_table), _ptr(kcache), _ptr(vcache),
                                     Lmax, _ptr(workspace), workspace.numel() * workspace.element_size(),
                                     _stream(stream))
    _check("llama_attn_prefill_ws", st)
    return out, lse


def llama_attn_prefill_cp_ws(q, k, v, q_pos_a: int, q_split: int, q_pos_b: int, rope_table, workspace, out=None,
                             lse=None, stream=None):
    """llama_attn_prefill_cp with caller-owned memory (rope_table rows >= Skv,
    workspace of llama_attn_prefill_workspace_size(B, Skv, Hkv) bytes). Returns (out, lse)."""
    import torch
    _require(q.dim() == 4 and k.dim() == 4 and v.dim() == 4, "q, k, v must be [B, S, H, D]")
    for t in (q, k, v):
        _require(t.is_cuda and t.dtype == torch.bfloat16 and t.is_contiguous(), "bf16 contiguous CUDA tensors expected")
    B, Sq, Hq, D = q.shape
    Skv, Hkv = k.shape[1], k.shape[2]
    _require(k.shape == (B, Skv, Hkv, D) and v.shape == k.shape, "k and v must be [B, Skv, Hkv, D]")
    if out is None:
        out = torch.empty_like(q)
    if lse is not None:
        _require(lse.is_cuda and lse.dtype == torch.float32 and lse.is_contiguous() and lse.shape == (B, Sq, Hq),
                 "lse: float32 [B, Sq, Hq]")
    st = lib().llama_attn_prefill_cp_ws(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, Sq, Skv, Hq, Hkv, D,
                                        int(q_pos_a), int(q_split), int(q_pos_b), _ptr(rope_table),
                                        _table_rows(rope_table), _ptr(workspace),
                                        workspace.numel() * workspace.element_size(), _stream(stream))
    _check("llama_attn_prefill_cp_ws", st)
    return out, lse


def llama_attn_prefill_rotated(q, k, v, out=None, lse=None, doc_offsets=None, stream=None):
    """bf16 prefill on already-rotated q [B,S,Hq,D] and k [B,S,Hkv,D] (no RoPE
    step). Returns (out, lse)."""
    import torch
    _require(q.dim() == 4 and k.dim() == 4 and v.dim() == 4, "q, k, v must be [B, S, H, D]")
    for t in (q, k, v):
        _require(t.is_cuda and t.dtype == torch.bfloat16 and t.is_contiguous(), "bf16 contiguous CUDA tensors expected")
    B, S, Hq, D = q.shape
    Hkv = k.shape[2]
    _require(k.shape == (B, S, Hkv, D) and v.shape == k.shape, "k and v must be [B, S, Hkv, D]")
    if out is None:
        out = torch.empty_like(q)
    _require(out.shape == q.shape and out.dtype == torch.bfloat16 and out.is_contiguous(), "bad out")
    if lse is not None:
        _require(lse.is_cuda and lse.dtype == torch.float32 and lse.is_contiguous() and lse.shape == (B, S, Hq),
                 "lse: float32 [B, S, Hq]")
    if doc_offsets is not None:
        _require(doc_offsets.is_cuda and doc_offsets.dtype == torch.int32, "doc_offsets: int32 CUDA tensor")
    st = lib().llama_attn_prefill_rotated(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(doc_offsets), B, S,
                                          Hq, Hkv, D, _stream(stream))
    _check("llama_attn_prefill_rotated", st)
    return out, lse


def llama_attn_quantize_e4m3(x, y=None, scale=None, stream=None):
    """Per-tensor dynamic E4M3 quantization of a bf16 CUDA tensor. Returns
    (codes uint8 tensor of x's shape, scale float32 CUDA tensor of one element)."""
    import torch
    _require(x.is_cuda and x.dtype == torch.bfloat16 and x.is_contiguous(), "x: bf16 contiguous CUDA tensor")
    if y is None:
        y = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    if scale is None:
        scale = torch.empty(1, dtype=torch.float32, device=x.device)
    _require(y.is_cuda and y.dtype == torch.uint8 and y.is_contiguous() and y.numel() == x.numel(), "bad y")
    _require(scale.is_cuda and scale.dtype == torch.float32 and scale.numel() >= 1, "bad scale")
    st = lib().llama_attn_quantize_e4m3(_ptr(x), x.numel(), _ptr(y), _ptr(scale), _stream(stream))
    _check("llama_attn_quantize_e4m3", st)
    return y, scale


def llama_attn_qkv_fp8_rope(x, s_x, w, s_w, B: int, S: int, Hq: int, Hkv: int, doc_offsets=None,
                            rope_theta: float = 500000.0, q=None, k=None, v=None, stream=None):
    """FP8 QKV projection with RoPE. x [B*S, d_model] and w [(Hq+2Hkv)*128,
    d_model] are uint8 E4M3 codes, s_x / s_w one-element float32 CUDA tensors.
    Returns (q rotated [B,S,Hq,128], k rotated [B,S,Hkv,128], v [B,S,Hkv,128]) bf16."""
    import torch
    D = 128
    for t in (x, w):
        _require(t.is_cuda and t.dtype == torch.uint8 and t.is_contiguous() and t.dim() == 2, "uint8 2-D codes")
    d_model = x.shape[1]
    _require(x.shape[0] == B * S and w.shape == ((Hq + 2 * Hkv) * D, d_model), "x / w shapes")
    for t in (s_x, s_w):
        _require(t.is_cuda and t.dtype == torch.float32, "scales: float32 CUDA tensors")
    dev = x.device
    if q is None:
        q = torch.empty(B, S, Hq, D, dtype=torch.bfloat16, device=dev)
    if k is None:
        k = torch.empty(B, S, Hkv, D, dtype=torch.bfloat16, device=dev)
    if v is None:
        v = torch.empty(B, S, Hkv, D, dtype=torch.bfloat16, device=dev)
    if doc_offsets is not None:
        _require(doc_offsets.is_cuda and doc_offsets.dtype == torch.int32, "doc_offsets: int32 CUDA tensor")
    st = lib().llama_attn_qkv_fp8_rope(_ptr(x), _ptr(s_x), _ptr(w), _ptr(s_w), _ptr(q), _ptr(k), _ptr(v),
                                       _ptr(doc_offsets), B, S, d_model, Hq, Hkv, D, float(rope_theta),
                                       _stream(stream))
    _check("llama_attn_qkv_fp8_rope", st)
    return q, k, v


def llama_attn_prefill_f32(q, k, v, out=None, doc_offsets=None, rope_theta: float = 500000.0, stream=None):
    """fp32 prefill on CUDA cores; same layout as llama_attn_prefill with float32 tensors."""
    import torch
    _require(q.dim() == 4 and k.dim() == 4 and v.dim() == 4, "q, k, v must be [B, S, H, D]")
    for t in (q, k, v):
        _require(t.is_cuda and t.dtype == torch.float32 and t.is_contiguous(), "f32 contiguous CUDA tensors expected")
    B, S, Hq, D = q.shape
    Hkv = k.shape[2]
    _require(k.shape == (B, S, Hkv, D) and v.shape == k.shape, "k and v must be [B, S, Hkv, D]")
    if out is None:
        out = torch.empty_like(q)
    if doc_offsets is not None:
        _require(doc_offsets.is_cuda and doc_offsets.dtype == torch.int32, "doc_offsets: int32 CUDA tensor")
    st = lib().llama_attn_prefill_f32(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(doc_offsets), B, S, Hq, Hkv, D,
                                      float(rope_theta), _stream(stream))
    _check("llama_attn_prefill_f32", st)
    return out


def llama_attn_decode_workspace_size(B: int, Hq: int, Lmax: int, D: int = 128) -> int:
    return int(lib().llama_attn_decode_workspace_size(B, Hq, Lmax, D))


def llama_attn_decode(q, kcache, vcache, cache_lens, out=None, workspace=None, rope_theta: float = 500000.0,
                      stream=None):
    """bf16 decode. q [B,Hq,D]; kcache/vcache [B,Hkv,Lmax,D] (keys pre-rotated); cache_lens int32 [B]."""
    import torch
    _require(q.dim() == 3 and kcache.dim() == 4 and vcache.shape == kcache.shape, "bad shapes")
    for t in (q, kcache, vcache):
        _require(t.is_cuda and t.dtype == torch.bfloat16 and t.is_contiguous(), "bf16 contiguous CUDA tensors expected")
    _require(cache_lens.is_cuda and cache_lens.dtype == torch.int32, "cache_lens: int32 CUDA tensor")
    B, Hq, D = q.shape
    Hkv, Lmax = kcache.shape[1], kcache.shape[2]
    _require(kcache.shape == (B, Hkv, Lmax, D) and cache_lens.numel() == B, "bad shapes")
    if out is None:
        out = torch.empty_like(q)
    need = llama_attn_decode_workspace_size(B, Hq, Lmax, D)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    st = lib().llama_attn_decode(_ptr(q), _ptr(kcache), _ptr(vcache), _ptr(cache_lens), _ptr(out), B, Hq, Hkv, D,
                                 Lmax, float(rope_theta), _ptr(workspace), workspace.numel() * workspace.element_size(),
                                 _stream(stream))
    _check("llama_attn_decode", st)
    return out


def llama_attn_decode_paged(q, kpages, vpages, block_table, cache_lens, out=None, workspace=None,
                            rope_theta: float = 500000.0, stream=None):
    """bf16 decode against a paged cache. q [B,Hq,D]; kpages/vpages
    [n_pages,Hkv,page_size,D] (keys pre-rotated); block_table int32 [B,max_blocks]
    (logical block j of sequence b is page block_table[b, j]); cache_lens int32 [B]."""
    import torch
    _require(q.dim() == 3 and kpages.dim() == 4 and vpages.shape == kpages.shape, "bad shapes")
    for t in (q, kpages, vpages):
        _require(t.is_cuda and t.dtype == torch.bfloat16 and t.is_contiguous(), "bf16 contiguous CUDA tensors expected")
    for t in (block_table, cache_lens):
        _require(t.is_cuda and t.dtype == torch.int32 and t.is_contiguous(), "block_table / cache_lens: int32 CUDA")
    B, Hq, D = q.shape
    n_pages, Hkv, page_size = kpages.shape[0], kpages.shape[1], kpages.shape[2]
    _require(kpages.shape[3] == D and block_table.dim() == 2 and block_table.shape[0] == B
             and cache_lens.numel() == B, "bad shapes")
    max_blocks = block_table.shape[1]
    if out is None:
        out = torch.empty_like(q)
    need = llama_attn_decode_workspace_size(B, Hq, max_blocks * page_size, D)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    st = lib().llama_attn_decode_paged(_ptr(q), _ptr(kpages), _ptr(vpages), _ptr(block_table), _ptr(cache_lens),
                                       _ptr(out), B, Hq, Hkv, D, page_size, max_blocks, n_pages, float(rope_theta),
                                       _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream))
    _check("llama_attn_decode_paged", st)
    return out


def llama_attn_decode_noalloc(q, kcache, vcache, cache_lens, out, rope_theta: float = 500000.0, stream=None):
    """llama_attn_decode without a workspace or any device allocation, for
    callers that cannot allocate: the partials go to a fixed 72 MiB array in the
    library. ``out`` must be supplied by the caller (nothing is allocated here)."""
    import torch
    _require(q.dim() == 3 and kcache.dim() == 4 and vcache.shape == kcache.shape, "bad shapes")
    for t in (q, kcache, vcache, out):
        _require(t.is_cuda and t.dtype == torch.bfloat16 and t.is_contiguous(), "bf16 contiguous CUDA tensors expected")
    _require(cache_lens.is_cuda and cache_lens.dtype == torch.int32, "cache_lens: int32 CUDA tensor")
    B, Hq, D = q.shape
    Hkv, Lmax = kcache.shape[1], kcache.shape[2]
    _require(out.shape == q.shape and cache_lens.numel() == B, "bad shapes")
    st = lib().llama_attn_decode_noalloc(_ptr(q), _ptr(kcache), _ptr(vcache), _ptr(cache_lens), _ptr(out), B, Hq,
                                         Hkv, D, Lmax, float(rope_theta), _stream(stream))
    _check("llama_attn_decode_noalloc", st)
    return out


def shard_units(n_units: int, world_size: int, rank: int):
    """Contiguous, balanced split of independent work units (e.g. (batch row,
    KV group) pairs of a prefill, or sequences of a decode) over ranks."""
    if world_size <= 0 or not (0 <= rank < world_size):
        raise ValueError("bad world_size / rank")
    base, extra = divmod(n_units, world_size)
    start = rank * base + min(rank, extra)
    return range(start, start + base + (1 if rank < extra else 0))
