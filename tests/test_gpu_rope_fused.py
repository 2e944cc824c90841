"""GPU tests of the two entry points that carry RoPE into the decode step:
attn_decode_gqa_rope (queries rotated inside the decode kernel) and
kv_append_rope (the new token's key rotated into its cache slot, value copied).

Both rotate with the same arithmetic as rope_apply_qk, so they are compared
bit for bit with rope_apply_qk followed by attn_decode_gqa (resp. a manual
placement), and the fused decode once more against the fp64 oracle chain."""
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


def _tables(K, d, max_pos, base=10000.0):
    return K.rope_table_build(K.rope_params(d, base=base), max_pos, device="cuda")


@pytest.mark.parametrize("pair_style", [0, 1])
@pytest.mark.parametrize("B,H,Hk,d,T_max", [(3, 8, 2, 64, 700), (5, 32, 8, 128, 1500), (2, 64, 1, 128, 2100),
                                            (4, 16, 16, 128, 300), (2, 64, 1, 64, 400)])
def test_fused_equals_rope_then_decode(K, pair_style, B, H, Hk, d, T_max):
    gen = W.generator(31 + H + d + pair_style)
    q = W.normal_bf16((B, H, d), gen).cuda()
    k = W.normal_bf16((B, Hk, T_max, d), gen).cuda()
    v = W.normal_bf16((B, Hk, T_max, d), gen).cuda()
    lens = torch.randint(1, T_max + 1, (B,), generator=torch.Generator().manual_seed(B * T_max), dtype=torch.int32)
    lens[0] = T_max
    lens = lens.cuda()
    pos = lens.clone()  # the query sits at the position after the cache
    cos, sin = _tables(K, d, T_max + 1)
    q_keep = q.clone()
    out_f, lse_f = K.attn_decode_gqa_rope(q, pos, cos, sin, k, v, lens, d ** -0.5, pair_style=pair_style)
    q_rot = q.clone()
    K.rope_apply_qk(q_rot, pos.view(B, 1), None, None, cos, sin, q_layout="bhd", pair_style=pair_style)
    out_u, lse_u = K.attn_decode_gqa(q_rot, k, v, lens, d ** -0.5)
    torch.cuda.synchronize()
    assert torch.equal(q, q_keep), "the fused call must not modify q"
    assert torch.equal(out_f, out_u) and torch.equal(lse_f, lse_u)


@pytest.mark.parametrize("B,H,Hk,d,T_max", [(3, 16, 2, 128, 2100), (2, 64, 1, 128, 2100), (2, 8, 8, 64, 900)])
def test_fused_equals_rope_then_decode_yarn(K, B, H, Hk, d, T_max):
    """As above with the YaRN s = 4 table, whose cos/sin carry the temperature
    factor 0.1 ln 4 + 1 (rows of magnitude other than 1)."""
    gen = W.generator(57 + H + d)
    q = W.normal_bf16((B, H, d), gen).cuda()
    k = W.normal_bf16((B, Hk, T_max, d), gen).cuda()
    v = W.normal_bf16((B, Hk, T_max, d), gen).cuda()
    lens = torch.randint(1, T_max + 1, (B,), generator=torch.Generator().manual_seed(T_max + H), dtype=torch.int32)
    lens = lens.cuda()
    p = K.rope_params(d, base=10000.0, scaling=K.ROPE_YARN, s=4.0, L_train=512.0, alpha=1.0, beta=32.0)
    cos, sin = K.rope_table_build(p, T_max + 1, device="cuda")
    assert abs(float(torch.hypot(cos[7], sin[7]).mean()) - (0.1 * np.log(4.0) + 1.0)) < 1e-5
    out_f, lse_f = K.attn_decode_gqa_rope(q, lens, cos, sin, k, v, lens, d ** -0.5)
    q_rot = q.clone()
    K.rope_apply_qk(q_rot, lens.view(B, 1), None, None, cos, sin, q_layout="bhd")
    out_u, lse_u = K.attn_decode_gqa(q_rot, k, v, lens, d ** -0.5)
    torch.cuda.synchronize()
    assert torch.equal(out_f, out_u) and torch.equal(lse_f, lse_u)


def test_fused_chain_against_oracle(K):
    wl = W.LLAMA3_8B_DECODE
    inp = W.decode_inputs(wl, B=4, T_max=3000, seed=77)
    r = wl.rope
    B = 4
    cos, sin = K.rope_table_build(K.rope_params(wl.d, base=r.base), 3001, device="cuda")
    k = inp["k"].cuda()
    K.rope_apply_qk(None, None, k, inp["k_pos"].cuda(), cos, sin, k_layout="bhtd")
    lens = inp["seq_lens"].cuda()
    out, lse = K.attn_decode_gqa_rope(inp["q"].cuda(), inp["q_pos"].view(B).cuda(), cos, sin, k, inp["v"].cuda(), lens,
                                      wl.scale)
    torch.cuda.synchronize()
    c, s = oracle.rope_table(wl.d, r.base, 3001)
    qr = oracle.rope_apply(W.bf16_bits(inp["q"])[:, None], inp["q_pos"].numpy(), c, s)[:, 0]
    kr = oracle.rope_apply(W.bf16_bits(inp["k"]), inp["k_pos"].numpy(), c, s, layout="bhtd")
    vr = oracle.bf16_bits_to_f64(W.bf16_bits(inp["v"]))
    ro, rl = oracle.attn_decode(qr, kr, vr, inp["seq_lens"].numpy(), wl.scale)
    qn = np.linalg.norm(qr, axis=-1)
    kmax = np.repeat(np.linalg.norm(kr, axis=-1).max(axis=-1), wl.g, axis=1)
    assert_attn_close(out, ro, lse, rl, "fused chain", lse_tol=chain_lse_tol(qn, kmax, wl.scale))
    # on the GPU's own rotated q (rope_apply_qk rotates bit-identically to the fused
    # prologue) and rotated cache: the plain lse tolerance
    q_rot = inp["q"].cuda()
    K.rope_apply_qk(q_rot, inp["q_pos"].view(B, 1).cuda(), None, None, cos, sin, q_layout="bhd")
    torch.cuda.synchronize()
    ro2, rl2 = oracle.attn_decode(W.bf16_bits(q_rot.cpu()), W.bf16_bits(k.cpu()), W.bf16_bits(inp["v"]),
                                  inp["seq_lens"].numpy(), wl.scale)
    assert_attn_close(out, ro2, lse, rl2, "fused chain on the GPU-rotated q/k")


@pytest.mark.parametrize("H,Hk", [(8, 2), (64, 1)])
def test_fused_bad_position_is_flagged_and_unrotated(K, H, Hk):
    B, d, T_max = 3, 128, 600
    gen = W.generator(5 + H)
    q = W.normal_bf16((B, H, d), gen).cuda()
    k = W.normal_bf16((B, Hk, T_max, d), gen).cuda()
    v = W.normal_bf16((B, Hk, T_max, d), gen).cuda()
    lens = torch.tensor([600, 200, 333], dtype=torch.int32).cuda()
    cos, sin = _tables(K, d, T_max + 1)
    pos = torch.tensor([600, 5000, 333], dtype=torch.int32).cuda()  # sequence 1 out of the table
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, lse = K.attn_decode_gqa_rope(q, pos, cos, sin, k, v, lens, d ** -0.5, dev_status=st)
    q_ref = q.clone()
    K.rope_apply_qk(q_ref, pos.view(B, 1), None, None, cos, sin, q_layout="bhd")  # skips sequence 1 as well
    ref_out, ref_lse = K.attn_decode_gqa(q_ref, k, v, lens, d ** -0.5)
    torch.cuda.synchronize()
    assert int(st.item()) & K.STATUS_BAD_POSITION
    assert torch.equal(out, ref_out) and torch.equal(lse, ref_lse)


@pytest.mark.parametrize("pair_style", [0, 1])
@pytest.mark.parametrize("d", [64, 128])
def test_kv_append_matches_rope_apply(K, pair_style, d):
    B, Hk, T_max = 4, 8, 50
    gen = W.generator(91 + d + pair_style)
    k_new = W.normal_bf16((B, Hk, d), gen).cuda()
    v_new = W.normal_bf16((B, Hk, d), gen).cuda()
    kc = W.normal_bf16((B, Hk, T_max, d), gen).cuda()
    vc = W.normal_bf16((B, Hk, T_max, d), gen).cuda()
    kc0, vc0 = kc.clone(), vc.clone()
    pos = torch.tensor([0, 17, 49, 30], dtype=torch.int32).cuda()
    cos, sin = _tables(K, d, 64)
    K.kv_append_rope(k_new, v_new, pos, kc, vc, cos, sin, pair_style=pair_style)
    k_ref = k_new.clone().view(B, Hk, 1, d)
    K.rope_apply_qk(None, None, k_ref, pos.view(B, 1), cos, sin, k_layout="bhtd", pair_style=pair_style)
    torch.cuda.synchronize()
    for b in range(B):
        p = int(pos[b])
        assert torch.equal(kc[b, :, p], k_ref[b, :, 0])
        assert torch.equal(vc[b, :, p], v_new[b])
        keep = torch.ones(T_max, dtype=torch.bool)
        keep[p] = False
        assert torch.equal(kc[b][:, keep], kc0[b][:, keep]) and torch.equal(vc[b][:, keep], vc0[b][:, keep])


def test_kv_append_bad_slot_is_flagged_and_untouched(K):
    B, Hk, d, T_max = 2, 2, 64, 10
    gen = W.generator(7)
    k_new = W.normal_bf16((B, Hk, d), gen).cuda()
    v_new = W.normal_bf16((B, Hk, d), gen).cuda()
    kc = W.normal_bf16((B, Hk, T_max, d), gen).cuda()
    vc = W.normal_bf16((B, Hk, T_max, d), gen).cuda()
    kc0, vc0 = kc.clone(), vc.clone()
    pos = torch.tensor([T_max, 3], dtype=torch.int32).cuda()  # sequence 0 has no room left
    cos, sin = _tables(K, d, 64)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    K.kv_append_rope(k_new, v_new, pos, kc, vc, cos, sin, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) & K.STATUS_BAD_POSITION
    assert torch.equal(kc[0], kc0[0]) and torch.equal(vc[0], vc0[0])
    assert torch.equal(vc[1, :, 3], v_new[1])


def test_append_then_fused_decode_sees_the_new_token(K):
    """One decode step as a server runs it: append the token's k/v at slot len,
    then attend with len + 1 rows; equal to the unfused ops on the same data."""
    B, H, Hk, d, T_max = 3, 32, 8, 128, 900
    gen = W.generator(12)
    q = W.normal_bf16((B, H, d), gen).cuda()
    k_new = W.normal_bf16((B, Hk, d), gen).cuda()
    v_new = W.normal_bf16((B, Hk, d), gen).cuda()
    kc = W.normal_bf16((B, Hk, T_max, d), gen).cuda()
    vc = W.normal_bf16((B, Hk, T_max, d), gen).cuda()
    lens = torch.tensor([100, 899, 0], dtype=torch.int32).cuda()
    cos, sin = _tables(K, d, T_max + 1, base=500000.0)
    kc2, vc2 = kc.clone(), vc.clone()
    K.kv_append_rope(k_new, v_new, lens, kc, vc, cos, sin)
    out, lse = K.attn_decode_gqa_rope(q, lens, cos, sin, kc, vc, lens + 1, d ** -0.5)
    # unfused: rotate k_new and q in place, place k/v by hand, decode
    kr = k_new.clone().view(B, Hk, 1, d)
    K.rope_apply_qk(None, None, kr, lens.view(B, 1), cos, sin, k_layout="bhtd")
    for b in range(B):
        kc2[b, :, int(lens[b])] = kr[b, :, 0]
        vc2[b, :, int(lens[b])] = v_new[b]
    qr = q.clone()
    K.rope_apply_qk(qr, lens.view(B, 1), None, None, cos, sin, q_layout="bhd")
    ref_out, ref_lse = K.attn_decode_gqa(qr, kc2, vc2, lens + 1, d ** -0.5)
    torch.cuda.synchronize()
    assert torch.equal(kc, kc2) and torch.equal(vc, vc2)
    assert torch.equal(out, ref_out) and torch.equal(lse, ref_lse)
