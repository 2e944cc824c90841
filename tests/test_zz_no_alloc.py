"""attn_decode_gqa_noalloc: the decode entry point for callers that cannot
allocate device memory (code inside another runtime's fixed memory pool, code
where a cudaMalloc would synchronise the device, C callers with no allocator).
It keeps its scratch in a static device array instead of a caller workspace.

Called here directly through the C ABI (ctypes).  Each shape runs twice in a
row with different inputs, so that the second call runs on the scratch its
predecessor left behind: a split-heavy shape on the mma.sync kernel (units cut
over many CTAs, merged through the counters at the start of the array) and a
64-head group on the tcgen05 kernel (partials merged by its combine pass).  Every
call is compared with attn_decode_gqa on the same inputs, and the first shape
also with the CPU oracle; dev_status must stay zero.  A stalled call (a bounded
wait made to run out) leaves counters behind, and attn_decode_gqa_noalloc_reset
clears them.  Kept in a file that pytest collects last."""
import ctypes

import pytest
import torch

import oracle
from mqa_kv_cache_b200 import workloads as W
from tests.gpu_util import assert_attn_close, to_np_f64

pytestmark = pytest.mark.gpu

_vp = ctypes.c_void_p


def _p(t):
    return None if t is None else _vp(t.data_ptr())


def _noalloc(lib, q, k, v, lens, scale, out, lse, st):
    B, H, d = q.shape
    _, Hk, T_max, _ = k.shape
    stream = _vp(torch.cuda.current_stream().cuda_stream)
    return lib.attn_decode_gqa_noalloc(_p(q), _p(k), _p(v), _p(lens), B, H, Hk, d, T_max, ctypes.c_float(scale),
                                       _p(out), _p(lse), _p(st), stream)


def _case(B, H, Hk, d, T, seed):
    gen = W.generator(seed)
    q = W.normal_bf16((B, H, d), gen)
    k = W.normal_bf16((B, Hk, T, d), gen)
    v = W.normal_bf16((B, Hk, T, d), gen)
    lens = torch.randint(T // 2, T + 1, (B,), generator=torch.Generator().manual_seed(seed), dtype=torch.int32)
    return q, k, v, lens


# (B, H, Hk, d, T): 4 units of ~100 tiles over 148 CTAs (every unit split, g = 4, mma.sync);
# 3 units of 64 heads (tcgen05 kernel and its combine pass)
SHAPES = [(2, 8, 2, 128, 8000), (3, 64, 1, 128, 3000)]


@pytest.mark.parametrize("shape", SHAPES, ids=["split_g4", "mqa_g64"])
def test_noalloc_matches_workspace_entry_point_on_two_calls(shape):
    from mqa_kv_cache_b200 import kvattn as K
    lib = K.library()
    lib.attn_decode_gqa_noalloc.restype = ctypes.c_int
    lib.kvattn_last_error_string.restype = ctypes.c_char_p
    B, H, Hk, d, T = shape
    scale = d ** -0.5
    assert K.attn_decode_gqa_workspace_bytes(B, H, Hk, d, T) <= (8 << 20)
    for call, seed in enumerate((11, 12)):
        q, k, v, lens = _case(B, H, Hk, d, T, seed + H)
        qg, kg, vg, lg = q.cuda(), k.cuda(), v.cuda(), lens.cuda()
        ref_out, ref_lse = K.attn_decode_gqa(qg, kg, vg, lg, scale)
        out = torch.empty_like(qg)
        lse = torch.empty((B, H), dtype=torch.float32, device="cuda")
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        rc = _noalloc(lib, qg, kg, vg, lg, scale, out, lse, st)
        assert rc == 0, lib.kvattn_last_error_string()
        torch.cuda.synchronize()
        assert int(st.item()) == 0, f"dev_status {int(st.item()):#x} on call {call}"
        assert_attn_close(out, to_np_f64(ref_out), lse, to_np_f64(ref_lse), f"noalloc {shape} call {call}")
        if shape == SHAPES[0]:
            ro, rl = oracle.attn_decode(W.bf16_bits(q), W.bf16_bits(k), W.bf16_bits(v), lens.numpy(), scale)
            assert_attn_close(out, ro, lse, rl, f"noalloc vs oracle {shape} call {call}")


def test_noalloc_reset_clears_counters_after_a_timeout():
    from mqa_kv_cache_b200 import kvattn as K
    lib = K.library()
    lib.attn_decode_gqa_noalloc.restype = ctypes.c_int
    B, H, Hk, d, T = SHAPES[0]
    scale = d ** -0.5
    q, k, v, lens = _case(B, H, Hk, d, T, 21)
    qg, kg, vg, lg = q.cuda(), k.cuda(), v.cuda(), lens.cuda()
    out = torch.empty_like(qg)
    lse = torch.empty((B, H), dtype=torch.float32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    K.kvattn_test_decode_stall(0, 2_000_000)
    try:
        assert _noalloc(lib, qg, kg, vg, lg, scale, out, lse, st) == 0
        torch.cuda.synchronize()
    finally:
        K.kvattn_test_decode_stall(-1, 0)
    assert int(st.item()) & K.STATUS_TIMEOUT
    K.attn_decode_gqa_noalloc_reset()
    st.zero_()
    assert _noalloc(lib, qg, kg, vg, lg, scale, out, lse, st) == 0
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    ref_out, ref_lse = K.attn_decode_gqa(qg, kg, vg, lg, scale)
    torch.cuda.synchronize()
    assert_attn_close(out, to_np_f64(ref_out), lse, to_np_f64(ref_lse), "noalloc after reset")


def test_noalloc_rejects_shapes_beyond_the_static_scratch():
    from mqa_kv_cache_b200 import kvattn as K
    lib = K.library()
    lib.kvattn_last_error_string.restype = ctypes.c_char_p
    # 1024 sequences of one 64-head group at head width 128: far more partials than
    # the 8 MiB array holds
    need = K.attn_decode_gqa_workspace_bytes(1024, 64, 1, 128, 4096)
    assert need > (8 << 20)
    fake = _vp(1 << 20)
    rc = lib.attn_decode_gqa_noalloc(fake, fake, fake, fake, 1024, 64, 1, 128, 4096, ctypes.c_float(0.1), fake, None,
                                     None, None)
    assert rc == -6
    assert b"static" in lib.kvattn_last_error_string()
