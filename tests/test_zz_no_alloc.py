"""attn_decode_gqa_noalloc: the decode entry point for callers that cannot
allocate device memory (code inside another runtime's fixed memory pool, code
where a cudaMalloc would synchronise the device, C callers with no allocator).
It keeps its scratch in a static device array instead of a caller workspace.

Called here directly through the C ABI (ctypes) and compared with
attn_decode_gqa on the same inputs, on two calls in a row with different
inputs (the static scratch keeps the previous call's contents, which must not
matter).  Kept in a file that pytest collects last."""
import ctypes

import pytest
import torch

from mqa_kv_cache_b200 import workloads as W
from tests.gpu_util import assert_attn_close, to_np_f64

pytestmark = pytest.mark.gpu

_vp = ctypes.c_void_p


def _p(t):
    return None if t is None else _vp(t.data_ptr())


def _noalloc(lib, q, k, v, lens, scale, out, lse):
    B, H, d = q.shape
    _, Hk, T_max, _ = k.shape
    stream = _vp(torch.cuda.current_stream().cuda_stream)
    return lib.attn_decode_gqa_noalloc(_p(q), _p(k), _p(v), _p(lens), B, H, Hk, d, T_max, ctypes.c_float(scale),
                                       _p(out), _p(lse), None, stream)


def test_noalloc_matches_workspace_entry_point_on_two_calls():
    from mqa_kv_cache_b200 import kvattn as K
    lib = K.library()
    lib.attn_decode_gqa_noalloc.restype = ctypes.c_int
    cases = [(W.LLAMA3_8B_DECODE, 4, 3000, 11), (W.LLAMA2_70B_MQA_32K, 3, 1500, 12)]
    for wl, B, T_max, seed in cases:
        inp = W.decode_inputs(wl, B=B, T_max=T_max, seed=seed)
        q, k, v = inp["q"].cuda(), inp["k"].cuda(), inp["v"].cuda()
        lens = inp["seq_lens"].cuda()
        ref_out, ref_lse = K.attn_decode_gqa(q, k, v, lens, wl.scale)
        out = torch.empty_like(q)
        lse = torch.empty((B, wl.H), dtype=torch.float32, device="cuda")
        rc = _noalloc(lib, q, k, v, lens, wl.scale, out, lse)
        assert rc == 0, lib.kvattn_last_error_string()
        torch.cuda.synchronize()
        assert_attn_close(out, to_np_f64(ref_out), lse, to_np_f64(ref_lse), f"noalloc {wl.name}")


def test_noalloc_rejects_shapes_beyond_the_static_scratch():
    from mqa_kv_cache_b200 import kvattn as K
    lib = K.library()
    lib.kvattn_last_error_string.restype = ctypes.c_char_p
    # 1024 sequences x 8 heads of width 128 in one group: far more scratch than the array holds
    need = K.attn_decode_gqa_workspace_bytes(1024, 64, 1, 128, 4096)
    assert need > (8 << 20)
    fake = _vp(1 << 20)
    rc = lib.attn_decode_gqa_noalloc(fake, fake, fake, fake, 1024, 64, 1, 128, 4096, ctypes.c_float(0.1), fake, None,
                                     None, None)
    assert rc == -6
    assert b"static" in lib.kvattn_last_error_string()
