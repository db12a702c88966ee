"""The allocation-free decode entry point against the regular one.

llama_attn_decode_noalloc serves callers that cannot allocate device memory
(for example a host whose allocator owns all of device memory): its split-KV
partials live in a fixed array inside the library instead of a caller
workspace. This test calls both entry points through the C ABI on the same
inputs, twice in a row, and requires the no-allocation results to match the
regular ones within the bf16 tolerance the other decode tests use; the second
call must leave the device's free memory unchanged. It sits in its own file,
collected last.
"""
import ctypes

import pytest
import torch

import gqa_attention_rope_b200 as la
from gqa_attention_rope_b200 import build as labuild
from gqa_attention_rope_b200 import workloads as W

pytestmark = pytest.mark.gpu

TOL_BF16 = 1.5e-2


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def test_noalloc_decode_matches_regular_decode_twice():
    labuild.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    lib = la.lib()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    cases = [
        W.custom_decode(41, 5, 16, 2, 128, 3000, (1, 3000)),
        W.custom_decode(42, 3, 8, 1, 128, 2100, (1, 2100)),
    ]
    lens_list = [[1, 1024, 1025, 2999, 3000], [0, 700, 2100]]
    for w, lens in zip(cases, lens_list):
        inp = W.make_decode_inputs(w, poison=True, lens=lens)
        q, kc, vc, ln = (inp[n].cuda() for n in ("q", "kcache", "vcache", "cache_lens"))
        ws_bytes = lib.llama_attn_decode_workspace_size(w.B, w.Hq, w.Lmax, w.D)
        ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
        ref = torch.empty_like(q)
        st = lib.llama_attn_decode(_p(q), _p(kc), _p(vc), _p(ln), _p(ref), w.B, w.Hq, w.Hkv, w.D, w.Lmax,
                                   ctypes.c_float(w.rope_theta), _p(ws), ws_bytes, stream)
        assert st == 0
        outs = [torch.full_like(q, float("nan")) for _ in range(2)]
        torch.cuda.synchronize()
        for i, out in enumerate(outs):
            free0 = torch.cuda.mem_get_info()[0]
            st = lib.llama_attn_decode_noalloc(_p(q), _p(kc), _p(vc), _p(ln), _p(out), w.B, w.Hq, w.Hkv, w.D,
                                               w.Lmax, ctypes.c_float(w.rope_theta), stream)
            assert st == 0
            torch.cuda.synchronize()
            if i > 0:  # the first call on a device may still load the kernels
                assert torch.cuda.mem_get_info()[0] == free0, "the no-alloc decode changed device free memory"
            assert torch.isfinite(out.float()).all()
            err = (out.float() - ref.float()).abs().max().item()
            assert err <= TOL_BF16, f"no-alloc decode differs from decode by {err}"
    assert la.llama_attn_get_device_error() == 0


def test_noalloc_decode_rejects_requests_beyond_its_scratch():
    labuild.build()
    lib = la.lib()
    fake = ctypes.c_void_p(4096)
    # 64 sequences x 64 heads x ceil(65536 / 1024) chunks needs ~135 MB > 72 MiB
    st = lib.llama_attn_decode_noalloc(fake, fake, fake, fake, fake, 64, 64, 8, 128, 65536,
                                       ctypes.c_float(5e5), None)
    assert st == -3
