"""GPU parity of attn_decode_gqa (split-K decode over a KV cache) against the
fp64 oracle, through the C ABI: every supported group size and head width,
ragged and edge lengths, garbage past the lengths, the full Llama-3-8B-shaped
ragged batch, sampled heads of the 32K Llama-2-70B shapes, and the chain
raw q/k -> RoPE -> decode against the oracle's fp64 chain."""
import numpy as np
import pytest
import torch

import oracle
from mqa_kv_cache_b200 import workloads as W
from tests.gpu_util import assert_attn_close, chain_lse_tol, to_np_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def K():
    from mqa_kv_cache_b200 import kvattn
    return kvattn


def _run(K, q, k, v, lens, scale):
    out, lse = K.attn_decode_gqa(q.cuda(), k.cuda(), v.cuda(), lens.cuda(), scale)
    torch.cuda.synchronize()
    return out, lse


def _oracle(q, k, v, lens, scale, sel=None):
    return oracle.attn_decode(W.bf16_bits(q), W.bf16_bits(k), W.bf16_bits(v), lens.numpy(), scale, sel=sel)


def test_tiny_gqa_config(K):
    inp = W.decode_inputs(W.TINY_GQA)
    out, lse = _run(K, inp["q"], inp["k"], inp["v"], inp["seq_lens"], W.TINY_GQA.scale)
    ro, rl = _oracle(inp["q"], inp["k"], inp["v"], inp["seq_lens"], W.TINY_GQA.scale)
    assert_attn_close(out, ro, lse, rl, "tiny")


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("g,Hk", [(1, 4), (2, 2), (4, 2), (8, 1), (16, 1), (32, 1), (64, 1), (8, 3)])
def test_group_sizes(K, d, g, Hk):
    B, T_max = 3, 300
    H = g * Hk
    lens = torch.tensor([300, 1, 129], dtype=torch.int32)
    gen = W.generator(1000 + g * 7 + Hk + d)
    q = W.normal_bf16((B, H, d), gen)
    k = W.normal_bf16((B, Hk, T_max, d), gen)
    v = W.normal_bf16((B, Hk, T_max, d), gen)
    scale = d ** -0.5
    out, lse = _run(K, q, k, v, lens, scale)
    ro, rl = _oracle(q, k, v, lens, scale)
    assert_attn_close(out, ro, lse, rl, f"g={g} Hk={Hk} d={d}")


@pytest.mark.parametrize("H,Hk", [(8, 2), (64, 1), (128, 2)])
def test_edge_lengths_and_empty(K, H, Hk):
    # 64 query heads per KV head: the tcgen05 kernel, whose combine pass also writes
    # the empty sequences
    lens = torch.tensor([0, 1, 63, 64, 65, 127, 128, 129, 1000, 999, 0, 2], dtype=torch.int32)
    B, d, T_max = len(lens), 128, 1000
    gen = W.generator(42 + H)
    q = W.normal_bf16((B, H, d), gen)
    k = W.normal_bf16((B, Hk, T_max, d), gen)
    v = W.normal_bf16((B, Hk, T_max, d), gen)
    out, lse = _run(K, q, k, v, lens, d ** -0.5)
    ro, rl = _oracle(q, k, v, lens, d ** -0.5)
    for b in (0, 10):
        assert torch.all(out[b].float() == 0) and torch.all(torch.isneginf(lse[b]))
    assert_attn_close(out, ro, lse, rl, "edge lengths")


@pytest.mark.parametrize("H,Hk", [(8, 2), (64, 1)])
def test_all_sequences_empty(K, H, Hk):
    B, d, T_max = 5, 128, 256
    gen = W.generator(43)
    q = W.normal_bf16((B, H, d), gen)
    k = W.normal_bf16((B, Hk, T_max, d), gen)
    v = W.normal_bf16((B, Hk, T_max, d), gen)
    out, lse = _run(K, q, k, v, torch.zeros(B, dtype=torch.int32), d ** -0.5)
    assert torch.all(out.float() == 0) and torch.all(torch.isneginf(lse))


@pytest.mark.parametrize("H,Hk", [(16, 2), (64, 1)])
def test_rows_past_length_never_reach_the_output(K, H, Hk):
    B, d, T_max = 4, 128, 200
    lens = torch.tensor([200, 70, 1, 130], dtype=torch.int32)
    gen = W.generator(5)
    q = W.normal_bf16((B, H, d), gen)
    k = W.normal_bf16((B, Hk, T_max, d), gen)
    v = W.normal_bf16((B, Hk, T_max, d), gen)
    out1, lse1 = _run(K, q, k, v, lens, 0.1)
    k2, v2 = k.clone(), v.clone()
    for b in range(B):
        k2[b, :, lens[b]:] = float("nan")
        v2[b, :, lens[b]:] = float("inf")
    out2, lse2 = _run(K, q, k2, v2, lens, 0.1)
    assert torch.equal(out1, out2) and torch.equal(lse1, lse2)


def test_bad_length_is_clamped_and_flagged(K):
    B, H, Hk, d, T_max = 2, 8, 8, 64, 64
    gen = W.generator(6)
    q = W.normal_bf16((B, H, d), gen)
    k = W.normal_bf16((B, Hk, T_max, d), gen)
    v = W.normal_bf16((B, Hk, T_max, d), gen)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, lse = K.attn_decode_gqa(q.cuda(), k.cuda(), v.cuda(), torch.tensor([100, -3], dtype=torch.int32).cuda(),
                                 0.125, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) & K.STATUS_BAD_LENGTH
    ro, rl = _oracle(q, k, v, torch.tensor([64, 0], dtype=torch.int32), 0.125)
    assert_attn_close(out, ro, lse, rl, "clamped")


@pytest.mark.parametrize("B,H,Hk,d,T", [(2, 8, 1, 128, 9000), (5, 64, 1, 128, 5000), (3, 16, 2, 64, 4000),
                                        (16, 64, 1, 128, 3000), (7, 32, 1, 128, 2500)])
def test_equal_lengths_split_into_whole_ranges(K, B, H, Hk, d, T):
    """Units of one length: the plan may give each unit the same number of CTAs
    (a multiple of the unit count), so that no CTA crosses into the next unit."""
    gen = W.generator(300 + B + H + Hk + d)
    q = W.normal_bf16((B, H, d), gen)
    k = W.normal_bf16((B, Hk, T, d), gen)
    v = W.normal_bf16((B, Hk, T, d), gen)
    lens = torch.full((B,), T, dtype=torch.int32)
    scale = d ** -0.5
    out, lse = _run(K, q, k, v, lens, scale)
    ro, rl = _oracle(q, k, v, lens, scale)
    assert_attn_close(out, ro, lse, rl, f"equal B={B} H={H} Hk={Hk} d={d}")


def test_deterministic(K):
    inp = W.decode_inputs(W.LLAMA3_8B_DECODE, B=4, T_max=2048)
    a = _run(K, inp["q"], inp["k"], inp["v"], inp["seq_lens"], 0.088)
    b = _run(K, inp["q"], inp["k"], inp["v"], inp["seq_lens"], 0.088)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_llama3_8b_ragged_full_size(K):
    """The full B=16, H=32, Hk=8, d=128 ragged batch (lengths 1024..8192), every head."""
    w = W.LLAMA3_8B_DECODE
    inp = W.decode_inputs(w)
    out, lse = _run(K, inp["q"], inp["k"], inp["v"], inp["seq_lens"], w.scale)
    ro, rl = _oracle(inp["q"], inp["k"], inp["v"], inp["seq_lens"], w.scale)
    assert_attn_close(out, ro, lse, rl, "llama3-8b ragged")


@pytest.mark.parametrize("wl", [W.LLAMA2_70B_GQA_32K, W.LLAMA2_70B_MQA_32K, W.LLAMA2_70B_MHA_32K],
                         ids=["gqa", "mqa", "mha"])
def test_llama2_70b_32k_sampled_heads(K, wl):
    """Full-size 32K caches drawn on the device; the oracle checks sampled
    (batch, head) outputs one by one from host copies of their K/V slices."""
    dev = torch.device("cuda")
    gen = W.generator(W.SEED_BASE + wl.index + 100, dev)
    q = W.normal_bf16((wl.B, wl.H, wl.d), gen, dev)
    k = W.normal_bf16((wl.B, wl.Hk, wl.T_max, wl.d), gen, dev)
    v = W.normal_bf16((wl.B, wl.Hk, wl.T_max, wl.d), gen, dev)
    lens = torch.full((wl.B,), wl.T_max, dtype=torch.int32, device=dev)
    out, lse = K.attn_decode_gqa(q, k, v, lens, wl.scale)
    torch.cuda.synchronize()
    rng = np.random.default_rng(wl.index)
    picks = [(int(rng.integers(wl.B)), int(rng.integers(wl.H))) for _ in range(12)]
    picks += [(0, 0), (wl.B - 1, wl.H - 1)]
    for b, h in picks:
        kvh = h // wl.g
        ks = k[b:b + 1, kvh:kvh + 1].cpu()
        vs = v[b:b + 1, kvh:kvh + 1].cpu()
        qs = q[b:b + 1, h:h + 1].cpu()
        ro, rl = _oracle(qs, ks, vs, torch.tensor([wl.T_max], dtype=torch.int32), wl.scale)
        assert_attn_close(out[b:b + 1, h:h + 1], ro, lse[b:b + 1, h:h + 1], rl, f"{wl.name} b={b} h={h}")


@pytest.mark.parametrize("wl", [W.LLAMA2_70B_GQA_32K, W.LLAMA2_70B_MQA_32K, W.LLAMA2_70B_MHA_32K],
                         ids=["gqa", "mqa", "mha"])
def test_llama2_70b_32k_yarn_chain_full_size(K, wl):
    """The 32K shapes as the bench times them: raw keys rotated at positions
    0..32767 with the YaRN s = 4 table (cos/sin carrying 0.1 ln 4 + 1), then
    attn_decode_gqa_rope with the raw queries rotated at position 32768 inside
    the decode kernel (the tcgen05 kernel for MQA).  Sampled (batch, head)
    outputs are checked against the oracle's fp64 chain (RoPE then attention),
    and against the oracle's attention on the GPU's own rotated q and k with the
    plain lse tolerance."""
    dev = torch.device("cuda")
    T = wl.T_max
    gen = W.generator(W.SEED_BASE + wl.index + 200, dev)
    q = W.normal_bf16((wl.B, wl.H, wl.d), gen, dev)
    k = W.normal_bf16((wl.B, wl.Hk, T, wl.d), gen, dev)
    v = W.normal_bf16((wl.B, wl.Hk, T, wl.d), gen, dev)
    rng = np.random.default_rng(wl.index + 7)
    picks = [(int(rng.integers(wl.B)), int(rng.integers(wl.H))) for _ in range(10)]
    picks += [(0, 0), (wl.B - 1, wl.H - 1)]
    raw_k = {(b, h // wl.g): k[b:b + 1, h // wl.g:h // wl.g + 1].cpu() for b, h in picks}
    r = wl.rope
    p = K.rope_params(wl.d, base=r.base, scaling=r.scaling, s=r.s, L_train=r.L_train, alpha=r.alpha, beta=r.beta)
    cos, sin = K.rope_table_build(p, T + 1)
    K.rope_apply_qk(None, None, k, torch.arange(T, dtype=torch.int32, device=dev).repeat(wl.B, 1), cos, sin,
                    k_layout="bhtd")
    lens = torch.full((wl.B,), T, dtype=torch.int32, device=dev)
    out, lse = K.attn_decode_gqa_rope(q, lens, cos, sin, k, v, lens, wl.scale)
    q_rot = q.clone()
    K.rope_apply_qk(q_rot, lens.view(wl.B, 1), None, None, cos, sin, q_layout="bhd")
    torch.cuda.synchronize()
    c, s = oracle.rope_table(wl.d, r.base, T + 1, r.scaling, s=r.s, L_train=r.L_train, alpha=r.alpha, beta=r.beta)
    kpos = np.arange(T, dtype=np.int32)[None, :]
    one = np.array([T], np.int32)
    for b, h in picks:
        kvh = h // wl.g
        qr = oracle.rope_apply(W.bf16_bits(q[b:b + 1, h:h + 1].cpu())[:, None], np.array([[T]], np.int32), c, s)[:, 0]
        kr = oracle.rope_apply(W.bf16_bits(raw_k[(b, kvh)]), kpos, c, s, layout="bhtd")
        vb = W.bf16_bits(v[b:b + 1, kvh:kvh + 1].cpu())
        ro, rl = oracle.attn_decode(qr, kr, oracle.bf16_bits_to_f64(vb), one, wl.scale)
        tol = chain_lse_tol(np.linalg.norm(qr, axis=-1), np.linalg.norm(kr, axis=-1).max(axis=-1), wl.scale)
        o_bh, l_bh = out[b:b + 1, h:h + 1], lse[b:b + 1, h:h + 1]
        assert_attn_close(o_bh, ro, l_bh, rl, f"{wl.name} yarn chain b={b} h={h}", lse_tol=tol)
        ro2, rl2 = oracle.attn_decode(W.bf16_bits(q_rot[b:b + 1, h:h + 1].cpu()),
                                      W.bf16_bits(k[b:b + 1, kvh:kvh + 1].cpu()), vb, one, wl.scale)
        assert_attn_close(o_bh, ro2, l_bh, rl2, f"{wl.name} b={b} h={h} on the GPU-rotated q/k")


@pytest.mark.parametrize("wl,T_max", [(W.TINY_GQA, 256), (W.LLAMA3_8B_DECODE, 1500),
                                      (W.LLAMA2_70B_GQA_32K, 2048)], ids=["tiny", "llama3", "yarn"])
def test_chain_rope_then_decode(K, wl, T_max):
    """raw q, k -> rope_apply_qk (k at its row index, q at position len) ->
    attn_decode_gqa, against the oracle's fp64 rotation + fp64 attention."""
    B = min(wl.B, 4)
    inp = W.decode_inputs(wl, B=B, T_max=T_max)
    r = wl.rope
    max_pos = T_max + 1
    p = K.rope_params(wl.d, base=r.base, scaling=r.scaling, s=r.s, L_train=r.L_train, alpha=r.alpha, beta=r.beta)
    cos, sin = K.rope_table_build(p, max_pos)
    qg, kg = inp["q"].cuda(), inp["k"].cuda()
    K.rope_apply_qk(qg, inp["q_pos"].cuda(), kg, inp["k_pos"].cuda(), cos, sin, q_layout="bhd", k_layout="bhtd")
    out, lse = K.attn_decode_gqa(qg, kg, inp["v"].cuda(), inp["seq_lens"].cuda(), wl.scale)
    torch.cuda.synchronize()
    c, s = oracle.rope_table(wl.d, r.base, max_pos, r.scaling, s=r.s, L_train=r.L_train, alpha=r.alpha, beta=r.beta)
    qr = oracle.rope_apply(W.bf16_bits(inp["q"])[:, None], inp["q_pos"].numpy(), c, s)[:, 0]
    kr = oracle.rope_apply(W.bf16_bits(inp["k"]), inp["k_pos"].numpy(), c, s, layout="bhtd")
    vr = oracle.bf16_bits_to_f64(W.bf16_bits(inp["v"]))
    ro, rl = oracle.attn_decode(qr, kr, vr, inp["seq_lens"].numpy(), wl.scale)
    qn = np.linalg.norm(qr, axis=-1)                       # [B, H]
    kmax = np.linalg.norm(kr, axis=-1).max(axis=-1)        # [B, Hk] (rows past the length included: an upper bound)
    kmax_h = np.repeat(kmax, wl.g, axis=1)
    assert_attn_close(out, ro, lse, rl, f"chain {wl.name}", lse_tol=chain_lse_tol(qn, kmax_h, wl.scale))
    # the attention step alone, on the q and k the GPU rotated (its bf16 roundings
    # included): the plain lse tolerance applies
    ro2, rl2 = oracle.attn_decode(W.bf16_bits(qg.cpu()), W.bf16_bits(kg.cpu()), W.bf16_bits(inp["v"]),
                                  inp["seq_lens"].numpy(), wl.scale)
    assert_attn_close(out, ro2, lse, rl2, f"chain {wl.name} on the GPU-rotated q/k")


ZERO_BYTES = 64 << 10  # KVATTN_DECODE_WS_ZERO_BYTES: the per-unit counters at the start of the workspace


def test_workspace_partials_need_no_initialisation(K):
    """Only the counter region must start zero: NaN-filled partials give the
    same result, and the call leaves the counters zero."""
    B, H, Hk, d, T_max = 3, 4, 2, 64, 300
    lens = torch.tensor([300, 1, 129], dtype=torch.int32)  # 18 tiles: units split over up to 5 CTAs
    gen = W.generator(77)
    q = W.normal_bf16((B, H, d), gen).cuda()
    k = W.normal_bf16((B, Hk, T_max, d), gen).cuda()
    v = W.normal_bf16((B, Hk, T_max, d), gen).cuda()
    ws = K.workspace(K.attn_decode_gqa_workspace_bytes(B, H, Hk, d, T_max))
    ws.fill_(0xFF)
    ws[:ZERO_BYTES].zero_()
    o1, l1 = K.attn_decode_gqa(q, k, v, lens.cuda(), d ** -0.5, ws=ws)
    torch.cuda.synchronize()
    assert int(ws[:ZERO_BYTES].count_nonzero()) == 0
    ws.zero_()
    o2, l2 = K.attn_decode_gqa(q, k, v, lens.cuda(), d ** -0.5, ws=ws)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    ro, rl = _oracle(q.cpu(), k.cpu(), v.cpu(), lens, d ** -0.5)
    assert_attn_close(o1, ro, l1, rl, "nan workspace")


def test_one_workspace_serves_calls_of_every_shape(K):
    """Calls of different shapes (both kernels, split and unsplit units) share one
    workspace: each finds the counters zero and leaves them zero."""
    shapes = [(2, 8, 2, 128, 5000, 31), (16, 64, 1, 128, 3000, 32), (5, 4, 4, 64, 700, 33),
              (1, 16, 1, 128, 9000, 34), (7, 32, 8, 128, 2000, 35)]
    need = max(K.attn_decode_gqa_workspace_bytes(B, H, Hk, d, T) for B, H, Hk, d, T, _ in shapes)
    ws = K.workspace(need)
    for B, H, Hk, d, T, seed in shapes:
        gen = W.generator(seed)
        q = W.normal_bf16((B, H, d), gen).cuda()
        k = W.normal_bf16((B, Hk, T, d), gen).cuda()
        v = W.normal_bf16((B, Hk, T, d), gen).cuda()
        lens = torch.randint(1, T + 1, (B,), generator=torch.Generator().manual_seed(seed), dtype=torch.int32)
        out, lse = K.attn_decode_gqa(q, k, v, lens.cuda(), d ** -0.5, ws=ws)
        torch.cuda.synchronize()
        assert int(ws[:ZERO_BYTES].count_nonzero()) == 0, (B, H, Hk, d, T)
        ro, rl = _oracle(q.cpu(), k.cpu(), v.cpu(), lens, d ** -0.5)
        assert_attn_close(out, ro, lse, rl, f"shared workspace {(B, H, Hk, d, T)}")
