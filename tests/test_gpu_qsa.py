"""GPU parity of the block-level indexer path (4-token groups: block keys,
group scoring + top-n, expansion with the trailing partial group) and of the
sparse GQA decode over a token list, against the fp64 oracle, through the C ABI.

Block keys: fp32 arithmetic rounded once to bf16, so every element lies within
one bf16 spacing of the fp64 value (plus 2^-20 for the fp32 rounding of a
rotation whose result cancels to near zero).  Group scores: the lightning indexer's
bound (fp32 sums of 128 bf16 products plus the head sum).  Selection: bit-exact
against the oracle's top-n taken on the kernel's own fp32 scores (both sides
decide in fp32), ties to the lower group; expansion is integer work, bit-exact.
Attention: max-abs 2e-2, rel-L2 5e-3."""
import numpy as np
import pytest
import torch

import oracle
from mqa_kv_cache_b200 import workloads as W
from tests.gpu_util import assert_attn_close, bf16_ulp, to_np_f64

pytestmark = pytest.mark.gpu

WL = W.QSA_128K


@pytest.fixture(scope="module")
def K():
    from mqa_kv_cache_b200 import kvattn
    return kvattn


def _tables(K, max_pos, base=500000.0):
    return K.rope_table_build(K.rope_params(128, base=base), max_pos, device="cuda")


@pytest.mark.parametrize("pair_style", [0, 1])
def test_block_keys_against_oracle(K, pair_style):
    B, L = 3, 1024
    gen = W.generator(501 + pair_style)
    k_idx = W.normal_bf16((B, L, 128), gen)
    lens = torch.tensor([1024, 1023, 6], dtype=torch.int32)
    cos, sin = _tables(K, L)
    sentinel = torch.full((B, L // 4, 128), 7.0, dtype=torch.bfloat16, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    kb = K.qsa_block_keys(k_idx.cuda(), lens.cuda(), cos, sin, block_keys=sentinel, eps=1e-6, pair_style=pair_style,
                          dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    c, s = oracle.rope_table(128, 500000.0, L)
    ref = oracle.qsa_block_keys(W.bf16_bits(k_idx), lens.numpy(), c, s, 1e-6, pair_style)
    got = to_np_f64(kb)
    for b in range(B):
        nb = int(lens[b]) // 4
        e = np.abs(got[b, :nb] - ref[b, :nb])
        assert np.all(e <= bf16_ulp(ref[b, :nb]) + 2.0 ** -20), f"row {b}: worst {e.max():.3e}"
        exact = got[b, :nb] == to_np_f64(torch.from_numpy(ref[b, :nb]).to(torch.bfloat16))
        assert exact.mean() > 0.99, f"row {b}: only {exact.mean():.4f} round to the same bf16"
        assert np.all(got[b, nb:] == 7.0), "groups past the complete ones must stay untouched"


def test_block_keys_incremental_equals_full_build(K):
    """Decode steps append tokens; the step that completes a group builds just that
    key (block_from = its index, max_new = 1), bit-identical to a full build."""
    B, L = 4, 512
    gen = W.generator(503)
    k_idx = W.normal_bf16((B, L, 128), gen).cuda()
    cos, sin = _tables(K, L)
    lens0 = torch.tensor([100, 7, 256, 0], dtype=torch.int32, device="cuda")
    kb = K.qsa_block_keys(k_idx, lens0, cos, sin)
    lens = lens0.clone()
    for _ in range(9):  # nine tokens per row: two more groups complete in every row
        prev_nb = lens // 4
        lens += 1
        K.qsa_block_keys(k_idx, lens, cos, sin, block_keys=kb, block_from=prev_nb.to(torch.int32), max_new=1)
    full = K.qsa_block_keys(k_idx, lens, cos, sin)
    torch.cuda.synchronize()
    assert torch.equal(kb, full)


def test_block_keys_position_past_table_is_flagged(K):
    B, L = 1, 64
    k_idx = W.normal_bf16((B, L, 128), W.generator(504)).cuda()
    cos, sin = _tables(K, 40)  # groups at positions 40 .. 60 have no table row
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    K.qsa_block_keys(k_idx, torch.tensor([64], dtype=torch.int32, device="cuda"), cos, sin, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) & K.STATUS_BAD_POSITION


def _score_bound(q_bits, w, kb_bits):
    q = oracle.bf16_bits_to_f64(q_bits)
    k = oracle.bf16_bits_to_f64(kb_bits)
    absdot = np.einsum("bji,bti->btj", np.abs(q), np.abs(k))
    return 2.0 ** -16 * np.einsum("btj,bj->bt", absdot, w.astype(np.float64)) + 1e-30


@pytest.mark.parametrize("L_max,lens,n_top", [(4 * 3000, [4 * 3000, 4 * 700 + 3, 4 * 100 + 2], 512),
                                              (4 * 600, [4 * 600, 4 * 599 + 1, 3, 0], 64),
                                              (4 * 5000, [4 * 5000 - 1, 4 * 4096 + 2], 2048)])
def test_select_against_oracle(K, L_max, lens, n_top):
    """Stored block keys stand in as seeded bf16 inputs; the oracle scores them in
    fp64 and selects on the kernel's fp32 scores."""
    B = len(lens)
    gen = W.generator(505 + n_top)
    q_idx = W.normal_bf16((B, 64, 128), gen)
    w = W.uniform_f32((B, 64), gen)
    kb = W.normal_bf16((B, L_max // 4, 128), gen)
    lens_t = torch.tensor(lens, dtype=torch.int32)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    tok, cnt, sc = K.qsa_select(q_idx.cuda(), w.cuda(), kb.cuda(), lens_t.cuda(), n_top=n_top, want_scores=True,
                                dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    qb, kbb, wn = W.bf16_bits(q_idx), W.bf16_bits(kb), w.numpy()
    ref_sc = oracle.qsa_scores(qb, wn, kbb, lens_t.numpy())
    g = sc.cpu().numpy().astype(np.float64)
    fin = np.isfinite(ref_sc)
    assert np.array_equal(np.isfinite(g), fin)
    bound = _score_bound(qb, wn, kbb)
    with np.errstate(invalid="ignore"):
        err = np.abs(g - ref_sc)
    assert np.all(err[fin] <= bound[fin])
    ref_tok, ref_cnt = oracle.qsa_select(qb, wn, kbb, lens_t.numpy(), n_top, scores=g)
    np.testing.assert_array_equal(cnt.cpu().numpy(), ref_cnt)
    np.testing.assert_array_equal(tok.cpu().numpy(), ref_tok)


def _lists(B, T, n_idx, counts, rng, holes=False):
    tok = np.full((B, n_idx), -1, np.int32)
    for b, c in enumerate(counts):
        if c == 0:
            continue
        t = np.sort(rng.choice(T, size=min(c, T), replace=False)).astype(np.int32)
        if holes:
            t[rng.random(len(t)) < 0.1] = -1
        tok[b, :len(t)] = t
    return tok


@pytest.mark.parametrize("H,Hk,d", [(32, 8, 128), (8, 8, 128), (32, 1, 128), (16, 4, 64), (64, 1, 64), (24, 3, 128)])
def test_sparse_gqa_against_oracle(K, H, Hk, d):
    T, n_idx = 3000, 2051
    counts = [2051, 1, 63, 64, 65, 0, 700]
    B = len(counts)
    gen = W.generator(600 + H + Hk + d)
    q = W.normal_bf16((B, H, d), gen)
    k = W.normal_bf16((B, Hk, T, d), gen)
    v = W.normal_bf16((B, Hk, T, d), gen)
    rng = np.random.default_rng(H * 7 + Hk + d)
    tok = _lists(B, T, n_idx, counts, rng, holes=(H == 32 and Hk == 8))
    cnt = np.array(counts, np.int32)
    scale = d ** -0.5
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, lse = K.attn_decode_gqa_sparse(q.cuda(), k.cuda(), v.cuda(), torch.from_numpy(tok).cuda(), scale,
                                        tok_count=torch.from_numpy(cnt).cuda(), dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    ro, rl = oracle.attn_decode_gqa_sparse(W.bf16_bits(q), W.bf16_bits(k), W.bf16_bits(v), tok, cnt, scale)
    assert_attn_close(out, ro, lse, rl, f"sparse gqa H={H} Hk={Hk} d={d}")


def test_sparse_gqa_bad_and_skipped_entries(K):
    """Entries outside [0, T_max) are skipped and flagged; a row whose entries are
    all -1 (a long one, split over several CTAs) gives zeros and lse = -inf."""
    B, H, Hk, d, T, n_idx = 3, 16, 2, 128, 900, 1500
    gen = W.generator(607)
    q = W.normal_bf16((B, H, d), gen)
    k = W.normal_bf16((B, Hk, T, d), gen)
    v = W.normal_bf16((B, Hk, T, d), gen)
    rng = np.random.default_rng(7)
    tok = _lists(B, T, n_idx, [800, 0, 0], rng)
    tok[0, [5, 77, 300]] = [T, 10 ** 6, -7]  # out of range: skipped, flagged
    cnt = np.array([800, 1500, 1], np.int32)  # row 1: 1500 entries, all -1; row 2: one -1
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, lse = K.attn_decode_gqa_sparse(q.cuda(), k.cuda(), v.cuda(), torch.from_numpy(tok).cuda(), d ** -0.5,
                                        tok_count=torch.from_numpy(cnt).cuda(), dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) & K.STATUS_BAD_INDEX
    clean = tok.copy()
    clean[0, [5, 77, 300]] = -1
    ro, rl = oracle.attn_decode_gqa_sparse(W.bf16_bits(q), W.bf16_bits(k), W.bf16_bits(v), clean, cnt, d ** -0.5)
    assert_attn_close(out, ro, lse, rl, "bad entries")
    assert torch.all(out[1:] == 0) and torch.all(torch.isneginf(lse[1:]))


def test_sparse_gqa_full_list_equals_dense_decode(K):
    """Listing every row 0 .. len-1 is the dense decode (same kernel family, rows
    gathered instead of tiled): equal within rounding of the different tiling."""
    inp = W.decode_inputs(W.LLAMA3_8B_DECODE, B=4, T_max=3000, seed=608)
    lens = inp["seq_lens"]
    B = 4
    tok = np.full((B, 3000), -1, np.int32)
    for b in range(B):
        tok[b, :int(lens[b])] = np.arange(int(lens[b]))
    out, lse = K.attn_decode_gqa_sparse(inp["q"].cuda(), inp["k"].cuda(), inp["v"].cuda(), torch.from_numpy(tok).cuda(),
                                        W.LLAMA3_8B_DECODE.scale, tok_count=lens.cuda())
    dout, dlse = K.attn_decode_gqa(inp["q"].cuda(), inp["k"].cuda(), inp["v"].cuda(), lens.cuda(),
                                   W.LLAMA3_8B_DECODE.scale)
    torch.cuda.synchronize()
    assert torch.equal(out, dout) and torch.equal(lse, dlse)


def _hot_inputs(B, L_max, lens, n_top, rng, gen):
    """Indexer inputs whose selection is unambiguous: n_top 'hot' groups per row carry
    a common direction u that every indexer query shares."""
    u = rng.standard_normal(128)
    k_idx = 0.3 * rng.standard_normal((B, L_max, 128))
    hot = []
    for b in range(B):
        nb = lens[b] // 4
        h = rng.choice(nb, size=min(n_top, nb), replace=False)
        hot.append(np.sort(h))
        for j in h:
            k_idx[b, 4 * j:4 * j + 4] += 2.0 * u
    q_idx = u[None, None] + 0.1 * rng.standard_normal((B, 64, 128))
    to_bf16 = lambda x: torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16)
    return to_bf16(q_idx), W.uniform_f32((B, 64), gen), to_bf16(k_idx), hot


def test_chain_block_keys_select_attend(K):
    """k_idx -> block keys -> group top-n + expand -> sparse GQA decode, all on the
    GPU, against the oracle's fp64 chain (identity rotation, so that the hot groups
    are the clear winners on both sides)."""
    B, L_max, n_top, H, Hk, d = 2, 4 * 1500, 512, 32, 8, 128
    lens = [4 * 1500 - 2, 4 * 1200 + 3]
    rng = np.random.default_rng(609)
    gen = W.generator(609)
    q_idx, w, k_idx, hot = _hot_inputs(B, L_max, lens, n_top, rng, gen)
    q = W.normal_bf16((B, H, d), gen)
    k = W.normal_bf16((B, Hk, L_max, d), gen)
    v = W.normal_bf16((B, Hk, L_max, d), gen)
    cos = torch.ones((L_max, 64), dtype=torch.float32, device="cuda")
    sin = torch.zeros((L_max, 64), dtype=torch.float32, device="cuda")
    lens_t = torch.tensor(lens, dtype=torch.int32)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    kb = K.qsa_block_keys(k_idx.cuda(), lens_t.cuda(), cos, sin, dev_status=st)
    tok, cnt, _ = K.qsa_select(q_idx.cuda(), w.cuda(), kb, lens_t.cuda(), n_top=n_top, dev_status=st)
    out, lse = K.attn_decode_gqa_sparse(q.cuda(), k.cuda(), v.cuda(), tok, d ** -0.5, tok_count=cnt, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    c, s = np.ones((L_max, 64)), np.zeros((L_max, 64))
    ref_kb = oracle.qsa_block_keys(W.bf16_bits(k_idx), lens_t.numpy(), c, s, 1e-6)
    ref_tok, ref_cnt = oracle.qsa_select(W.bf16_bits(q_idx), w.numpy(), ref_kb, lens_t.numpy(), n_top)
    for b in range(B):
        sel = sorted({int(t) // 4 for t in ref_tok[b, :ref_cnt[b]] if t < 4 * (lens[b] // 4)})
        assert sel == list(hot[b]), "the oracle must pick exactly the hot groups"
    np.testing.assert_array_equal(cnt.cpu().numpy(), ref_cnt)
    np.testing.assert_array_equal(tok.cpu().numpy(), ref_tok)
    ro, rl = oracle.attn_decode_gqa_sparse(W.bf16_bits(q), W.bf16_bits(k), W.bf16_bits(v), ref_tok, ref_cnt,
                                           d ** -0.5)
    assert_attn_close(out, ro, lse, rl, "qsa chain")


def test_full_size_selection_properties_and_sampled_heads(K):
    """The measured shape (B 8, up to 131072 tokens, 512 groups of 4, H 32 / Hk 8):
    every selected group scores at least as high as every unselected one (ties to
    the lower group), the list is the expansion of those groups plus the tail, and
    sampled heads of the decode over a seeded list agree with the oracle."""
    dev = torch.device("cuda")
    inp = W.qsa_inputs(WL, device=dev)
    lens = inp["seq_lens"]
    cos, sin = _tables(K, WL.L)
    kb = K.qsa_block_keys(inp["k_idx"], lens.to(dev), cos, sin)
    tok, cnt, sc = K.qsa_select(inp["q_idx"], inp["w"], kb, lens.to(dev), n_top=WL.n_top, want_scores=True)
    torch.cuda.synchronize()
    tok, cnt, sc = tok.cpu().numpy(), cnt.cpu().numpy(), sc.cpu().numpy()
    for b in range(WL.B):
        L = int(lens[b])
        nb = L // 4
        assert cnt[b] == 4 * min(nb, WL.n_top) + L % 4
        t = tok[b, :cnt[b]]
        assert np.all(np.diff(t) > 0) and np.all(tok[b, cnt[b]:] == -1)
        groups = t[:4 * WL.n_top].reshape(-1, 4)
        assert np.all(groups == groups[:, :1] + np.arange(4)) and np.all(groups[:, 0] % 4 == 0)
        np.testing.assert_array_equal(t[4 * WL.n_top:], np.arange(4 * nb, L))
        chosen = np.zeros(nb, bool)
        chosen[groups[:, 0] // 4] = True
        s_b = sc[b, :nb]
        kth = s_b[chosen].min()
        assert np.all(s_b[~chosen] <= kth)
        tie = (~chosen) & (s_b == kth)
        if tie.any():
            assert np.flatnonzero(tie).min() > np.flatnonzero(chosen & (s_b == kth)).max()
    # sampled block keys against the oracle
    c, s = oracle.rope_table(128, WL.rope.base, WL.L)
    for b, j in ((0, 0), (3, 12345), (7, int(lens[7]) // 4 - 1)):
        kslice = inp["k_idx"][b:b + 1, 4 * j:4 * j + 4].cpu()
        cs, sn = c[4 * j:4 * j + 1], s[4 * j:4 * j + 1]
        # the slice is group 0 of a 4-token row: rotate at 4j with the table rows shifted
        ref = oracle.qsa_block_keys(W.bf16_bits(kslice), np.array([4]), cs, sn, 1e-6)[0, 0]
        got = to_np_f64(kb[b, j])
        assert np.all(np.abs(got - ref) <= bf16_ulp(ref) + 2.0 ** -20)
    # sampled heads of the decode over a seeded list of the selection's shape
    rng = np.random.default_rng(610)
    n_idx = 4 * WL.n_top + 3
    lst = np.full((WL.B, n_idx), -1, np.int32)
    cnts = np.zeros(WL.B, np.int32)
    for b in range(WL.B):
        L = int(lens[b])
        g = np.sort(rng.choice(L // 4, size=WL.n_top, replace=False))
        t = np.concatenate([(4 * g[:, None] + np.arange(4)).ravel(), np.arange(4 * (L // 4), L)]).astype(np.int32)
        lst[b, :len(t)] = t
        cnts[b] = len(t)
    out, lse = K.attn_decode_gqa_sparse(inp["q"], inp["k"], inp["v"], torch.from_numpy(lst).to(dev), WL.scale,
                                        tok_count=torch.from_numpy(cnts).to(dev))
    torch.cuda.synchronize()
    for b, h in ((0, 0), (2, 17), (5, 8), (7, 31)):
        kvh = h // (WL.H // WL.Hk)
        rows = torch.from_numpy(lst[b, :cnts[b]].astype(np.int64)).to(dev)
        ks = inp["k"][b:b + 1, kvh:kvh + 1].index_select(2, rows).cpu()
        vs = inp["v"][b:b + 1, kvh:kvh + 1].index_select(2, rows).cpu()
        qs = inp["q"][b:b + 1, h:h + 1].cpu()
        ro, rl = oracle.attn_decode(W.bf16_bits(qs), W.bf16_bits(ks), W.bf16_bits(vs),
                                    np.array([len(rows)], np.int32), WL.scale)
        assert_attn_close(out[b:b + 1, h:h + 1], ro, lse[b:b + 1, h:h + 1], rl, f"qsa full b={b} h={h}")


def test_select_nan_groups_are_never_taken(K):
    """A group whose score is NaN is never selected (and flagged), so the list is
    shorter than 4 n_top and the tail still follows.  (A NaN inside a key is not
    enough: ReLU takes a NaN dot product to 0 on both sides.  A +inf key element met
    by a head of weight 0 gives 0 * inf = NaN.)"""
    B, L_max, n_top = 2, 4 * 400, 16
    lens = [4 * 400, 4 * 20 + 3]
    gen = W.generator(611)
    q_idx = W.normal_bf16((B, 64, 128), gen)
    w = W.uniform_f32((B, 64), gen)
    kb = W.normal_bf16((B, L_max // 4, 128), gen)
    q_idx[:, 0, 0] = 1.0
    w[:, 0] = 0.0
    kb[0, 7, 0] = float("inf")
    for j in range(20):  # row 1: only 20 groups, 16 of them NaN -> 4 selectable
        if j % 5:
            kb[1, j, 0] = float("inf")
    lens_t = torch.tensor(lens, dtype=torch.int32)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    tok, cnt, sc = K.qsa_select(q_idx.cuda(), w.cuda(), kb.cuda(), lens_t.cuda(), n_top=n_top, want_scores=True,
                                dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) & K.STATUS_NAN_SCORE
    g = sc.cpu().numpy().astype(np.float64)
    # the oracle's top-k takes no NaN: select among each row's finite group scores
    sel = np.full((B, n_top), -1, np.int64)
    for b in range(B):
        nb = lens[b] // 4
        fin = np.flatnonzero(np.isfinite(g[b, :nb]))
        assert len(fin) == nb - (1 if b == 0 else 16)
        pick = oracle.topk(g[b, fin][None], n_top, lens=np.array([len(fin)], np.int32))[0]
        sel[b, :np.count_nonzero(pick >= 0)] = fin[pick[pick >= 0]]
    ref_tok, ref_cnt = oracle.qsa_expand(sel, lens_t.numpy(), n_top)
    np.testing.assert_array_equal(cnt.cpu().numpy(), ref_cnt)
    np.testing.assert_array_equal(tok.cpu().numpy(), ref_tok)
    assert ref_cnt[1] == 4 * 4 + 3


def test_select_arguments_are_checked(K):
    q_idx = torch.zeros((1, 64, 128), dtype=torch.bfloat16, device="cuda")
    w = torch.ones((1, 64), dtype=torch.float32, device="cuda")
    lens = torch.tensor([8], dtype=torch.int32, device="cuda")
    kb = torch.zeros((1, 10, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(K.KvattnError):
        K.qsa_select(q_idx, w, kb, lens, n_top=0)
    with pytest.raises(K.KvattnError):
        K.qsa_select(q_idx, w, kb, lens, n_top=2049)
    with pytest.raises(K.KvattnError):  # the indexer keys' length must be a multiple of 4
        K.qsa_block_keys(torch.zeros((1, 10, 128), dtype=torch.bfloat16, device="cuda"), lens,
                         *_tables(K, 16))
    with pytest.raises(K.KvattnError):  # group size above 32 at head_dim 128
        q = torch.zeros((1, 64, 128), dtype=torch.bfloat16, device="cuda")
        kc = torch.zeros((1, 1, 16, 128), dtype=torch.bfloat16, device="cuda")
        K.attn_decode_gqa_sparse(q, kc, kc, torch.zeros((1, 4), dtype=torch.int32, device="cuda"), 0.1)
