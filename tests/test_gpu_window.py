"""GPU tests of the sliding window with attention sinks over a rolling cache:
kv_append_rope_ring (tokens appended one at a time into n_sink + window slots)
and attn_decode_gqa_rope_window (decode over the filled slots), against the
fp64 oracle's windowed decode on the linear cache (row t = token t)."""
import numpy as np
import pytest
import torch

import oracle
from mqa_kv_cache_b200 import workloads as W
from tests.gpu_util import assert_attn_close, chain_lse_tol

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def K():
    from mqa_kv_cache_b200 import kvattn
    return kvattn


def _slot(p, n_sink, window):
    return p if p < n_sink else n_sink + (p - n_sink) % window


@pytest.mark.parametrize("H,Hk,n_sink,window", [(8, 2, 4, 60), (16, 1, 0, 64), (64, 1, 2, 126), (4, 4, 8, 24)])
def test_ring_append_then_window_decode(K, H, Hk, n_sink, window):
    d, base = 128, 500000.0
    cap = n_sink + window
    lens = [3 * cap + 5, cap // 2, cap, cap + 1]  # past the capacity, inside it, exactly at it, one over
    B, N = len(lens), max(lens)
    gen = W.generator(61 + H + n_sink + window)
    k_raw = W.normal_bf16((B, Hk, N, d), gen)
    v_raw = W.normal_bf16((B, Hk, N, d), gen)
    q_raw = W.normal_bf16((B, H, d), gen)
    cos, sin = K.rope_table_build(K.rope_params(d, base=base), N + 1, device="cuda")
    kc = W.normal_bf16((B, Hk, cap, d), gen).cuda()  # stale contents must not matter
    vc = W.normal_bf16((B, Hk, cap, d), gen).cuda()
    kg, vg = k_raw.cuda(), v_raw.cuda()
    for b in range(B):
        for t in range(lens[b]):
            pos = torch.tensor([t], dtype=torch.int32, device="cuda")
            K.kv_append_rope_ring(kg[b:b + 1, :, t].contiguous(), vg[b:b + 1, :, t].contiguous(), pos,
                                  kc[b:b + 1], vc[b:b + 1], cos, sin, n_sink, window)
    lens_t = torch.tensor(lens, dtype=torch.int32, device="cuda")
    scale = d ** -0.5
    out, lse = K.attn_decode_gqa_rope_window(q_raw.cuda(), lens_t, cos, sin, kc, vc, lens_t, scale, n_sink, window)
    # the same slots as a plain cache of min(len, cap) rows: bit-identical
    filled = torch.clamp(lens_t, max=cap)
    ref_out, ref_lse = K.attn_decode_gqa_rope(q_raw.cuda(), lens_t, cos, sin, kc, vc, filled, scale)
    # every surviving slot holds the token rotated at its own position
    k_rot = kg.clone()
    pos_all = torch.arange(N, dtype=torch.int32, device="cuda").repeat(B, 1)
    K.rope_apply_qk(None, None, k_rot, pos_all, cos, sin, k_layout="bhtd")
    torch.cuda.synchronize()
    assert torch.equal(out, ref_out) and torch.equal(lse, ref_lse)
    for b in range(B):
        for p in oracle.window_positions(lens[b], n_sink, window):
            s = _slot(p, n_sink, window)
            assert torch.equal(kc[b, :, s], k_rot[b, :, p]) and torch.equal(vc[b, :, s], vg[b, :, p]), (b, p)
    # against the oracle: RoPE in fp64 on the linear cache, then the windowed decode
    c, s = oracle.rope_table(d, base, N + 1)
    kr = oracle.rope_apply(W.bf16_bits(k_raw), pos_all.cpu().numpy(), c, s, layout="bhtd")
    qr = oracle.rope_apply(W.bf16_bits(q_raw)[:, None], np.array(lens, np.int32)[:, None], c, s)[:, 0]
    vr = oracle.bf16_bits_to_f64(W.bf16_bits(v_raw))
    ro, rl = oracle.attn_decode_window(qr, kr, vr, np.array(lens, np.int32), scale, n_sink, window)
    qn = np.linalg.norm(qr, axis=-1)
    kmax = np.repeat(np.linalg.norm(kr, axis=-1).max(axis=-1), H // Hk, axis=1)
    assert_attn_close(out, ro, lse, rl, f"window s={n_sink} w={window}", lse_tol=chain_lse_tol(qn, kmax, scale))
    # on the GPU-rotated q (rope_apply_qk, bit-identical to the fused prologue) and keys:
    # the plain lse tolerance
    q_rot = q_raw.cuda()
    K.rope_apply_qk(q_rot, lens_t.view(B, 1), None, None, cos, sin, q_layout="bhd")
    torch.cuda.synchronize()
    ro2, rl2 = oracle.attn_decode_window(W.bf16_bits(q_rot.cpu()), W.bf16_bits(k_rot.cpu()), W.bf16_bits(v_raw),
                                         np.array(lens, np.int32), scale, n_sink, window)
    assert_attn_close(out, ro2, lse, rl2, f"window s={n_sink} w={window} on the GPU-rotated q/k")


def test_window_arguments_are_checked(K):
    d = 64
    q = torch.zeros((1, 2, d), dtype=torch.bfloat16, device="cuda")
    kc = torch.zeros((1, 1, 16, d), dtype=torch.bfloat16, device="cuda")
    lens = torch.tensor([5], dtype=torch.int32, device="cuda")
    cos, sin = K.rope_table_build(K.rope_params(d, base=10000.0), 32, device="cuda")
    with pytest.raises(K.KvattnError):
        K.attn_decode_gqa_rope_window(q, lens, cos, sin, kc, kc, lens, 0.1, 4, 13)  # 4 + 13 > 16 slots
    with pytest.raises(K.KvattnError):
        K.attn_decode_gqa_rope_window(q, lens, cos, sin, kc, kc, lens, 0.1, 0, 0)   # empty window
