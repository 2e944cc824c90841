"""GPU parity of the lightning indexer, the top-k selection and the sparse
latent attention against the fp64 oracle, through the C ABI.

Scores: the kernel's fp32 scores against the oracle's fp64 scores within the
error bound of fp32 dot products of 128 bf16 products plus the 64-term head
sum: |d| <= 2^-16 * sum_j w_j * sum_i |q_ji k_ti|.  Selection: bit-exact
against the oracle's top-k taken on the kernel's own fp32 scores (both sides
decide in fp32), ties to the lower index; the kernel lists the selected
indices in increasing order, so the oracle's list is compared after sorting.  The fp64 selection may differ only
at ranks whose fp64 scores lie within that bound of the k-th score.
"""
import numpy as np
import pytest
import torch

import oracle
from mqa_kv_cache_b200 import workloads as W
from tests.gpu_util import assert_attn_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def K():
    from mqa_kv_cache_b200 import kvattn
    return kvattn


def _score_bound(q_bits, w, k_bits):
    q = oracle.bf16_bits_to_f64(q_bits)  # [B, 64, 128]
    k = oracle.bf16_bits_to_f64(k_bits)  # [B, L, 128]
    absdot = np.einsum("bji,bti->btj", np.abs(q), np.abs(k))
    return 2.0 ** -16 * np.einsum("btj,bj->bt", absdot, w.astype(np.float64)) + 1e-30


def _check_scores(gpu_scores, q_bits, w, k_bits, lens):
    ref = oracle.dsa_scores(q_bits, w, k_bits, lens)
    g = gpu_scores.astype(np.float64)
    fin = np.isfinite(ref)
    assert np.array_equal(np.isfinite(g), fin)
    bound = _score_bound(q_bits, w, k_bits)
    with np.errstate(invalid="ignore"):  # -inf - -inf past the lengths; only finite entries are compared
        err = np.abs(g - ref)
    assert np.all(err[fin] <= bound[fin]), f"worst excess {(err - bound)[fin].max():.3e}"
    return ref, bound


def _index_order(idx):
    """The oracle's selection (score order, -1 padded) in increasing index order."""
    out = np.full_like(idx, -1)
    for b in range(idx.shape[0]):
        v = np.sort(idx[b][idx[b] >= 0])
        out[b, :len(v)] = v
    return out


def _run_index(K, inp, k, lens=None):
    q_idx, w, k_idx = inp["q_idx"].cuda(), inp["w"].cuda(), inp["k_idx"].cuda()
    lens_d = None if lens is None else lens.cuda()
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    idx, scores = K.dsa_index_topk(q_idx, w, k_idx, k, seq_lens=lens_d, dev_status=st)
    torch.cuda.synchronize()
    return idx.cpu().numpy(), scores.cpu().numpy(), int(st.item())


@pytest.mark.parametrize("L,k,lens", [(1000, 64, [1000, 777, 5]), (4096, 2048, [4096, 4000, 2049]),
                                      (300, 2048, [300, 1, 0])])
def test_indexer_and_topk_small(K, L, k, lens):
    wl = W.DSA_128K
    lens_t = torch.tensor(lens, dtype=torch.int32)
    inp = W.dsa_inputs(wl, B=len(lens), L=L, seed=31 + L + k, with_latent=False)
    idx, scores, st = _run_index(K, inp, k, lens_t)
    assert st == 0
    qb, kb, w = W.bf16_bits(inp["q_idx"]), W.bf16_bits(inp["k_idx"]), inp["w"].numpy()
    _check_scores(scores, qb, w, kb, lens_t.numpy())
    ref_idx = oracle.topk(scores, k, lens=lens_t.numpy())
    np.testing.assert_array_equal(idx, _index_order(ref_idx))


@pytest.mark.parametrize("B,L,k", [(160, 512, 64), (2, 700, 100), (5, 128, 16)])
def test_indexer_work_claims(K, B, L, k):
    """The indexer's CTAs claim each row's key tiles from a per-row counter: more rows
    than CTAs (a CTA serves several rows in turn), and rows of a few tiles shared by
    several CTAs (some of which may find the row already taken).  Scores and selection
    against the oracle, twice on the same workspace (the counters are left zero)."""
    wl = W.DSA_128K
    inp = W.dsa_inputs(wl, B=B, L=L, seed=71 + B + L, with_latent=False)
    lens = torch.randint(1, L + 1, (B,), generator=torch.Generator().manual_seed(B + L), dtype=torch.int32)
    q_idx, w, k_idx = inp["q_idx"].cuda(), inp["w"].cuda(), inp["k_idx"].cuda()
    ws = K.workspace(K.dsa_index_topk_workspace_bytes(B, L, k))
    qb, kb, wn = W.bf16_bits(inp["q_idx"]), W.bf16_bits(inp["k_idx"]), inp["w"].numpy()
    for call in range(2):
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        idx, scores = K.dsa_index_topk(q_idx, w, k_idx, k, seq_lens=lens.cuda(), ws=ws, dev_status=st)
        torch.cuda.synchronize()
        assert int(st.item()) == 0, call
        assert int(ws[:B * 2048 * 4 + B * 4].count_nonzero()) == 0, call
        scores = scores.cpu().numpy()
        _check_scores(scores, qb, wn, kb, lens.numpy())
        ref_idx = oracle.topk(scores, k, lens=lens.numpy())
        np.testing.assert_array_equal(idx.cpu().numpy(), _index_order(ref_idx))


def test_topk_ties_go_to_the_lower_index(K):
    # duplicated key rows give bit-identical scores; all-zero rows give exact 0 scores
    B, L, k = 2, 3000, 500
    wl = W.DSA_128K
    inp = W.dsa_inputs(wl, B=B, L=L, seed=77, with_latent=False)
    kk = inp["k_idx"]
    kk[:, 37:] = kk[:, :37].repeat(1, (L + 36) // 37, 1)[:, :L - 37]
    kk[1, ::5] = 0
    inp["k_idx"] = kk
    idx, scores, st = _run_index(K, inp, k)
    assert st == 0
    ref_idx = oracle.topk(scores, k)
    np.testing.assert_array_equal(idx, _index_order(ref_idx))
    # the k-th score is tied: only its lowest-index occurrences are taken
    for b in range(B):
        sel = scores[b, idx[b]]
        kth = sel.min()
        tied = np.flatnonzero(scores[b] == kth)
        taken = np.intersect1d(tied, idx[b])
        assert len(taken) < len(tied)  # the test data really has a tie at the boundary
        np.testing.assert_array_equal(taken, tied[:len(taken)])
        assert np.all(np.diff(idx[b]) > 0)


def test_dsa_full_size_indexer_and_topk(K):
    """B=8, L=131072, k=2048: selection bit-exact on the kernel's scores for every row;
    scores checked against the fp64 oracle on sampled token positions."""
    wl = W.DSA_128K
    dev = torch.device("cuda")
    gen = W.generator(W.SEED_BASE + wl.index + 100, dev)
    q_idx = W.normal_bf16((wl.B, wl.HI, wl.dI), gen, dev)
    w = W.uniform_f32((wl.B, wl.HI), gen, dev)
    k_idx = W.normal_bf16((wl.B, wl.L, wl.dI), gen, dev)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    idx, scores = K.dsa_index_topk(q_idx, w, k_idx, wl.k, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    idx, scores = idx.cpu().numpy(), scores.cpu().numpy()
    np.testing.assert_array_equal(idx, _index_order(oracle.topk(scores, wl.k)))
    rng = np.random.default_rng(5)
    sample = np.sort(rng.choice(wl.L, 3000, replace=False))
    sample_t = torch.from_numpy(sample).to(dev)
    kb = W.bf16_bits(k_idx[:, sample_t])
    qb, wn = W.bf16_bits(q_idx), w.cpu().numpy()
    ref, bound = _check_scores(scores[:, sample], qb, wn, kb, np.full(wl.B, len(sample), np.int32))
    # the fp64 top-k of the sampled scores differs from the fp32 one only inside the error band
    for b in range(wl.B):
        r64 = set(oracle.topk(ref[b:b + 1], 256)[0].tolist())
        r32 = set(oracle.topk(scores[b:b + 1, sample], 256)[0].tolist())
        kth = np.sort(ref[b])[::-1][255]
        for j in r64 ^ r32:
            assert abs(ref[b, j] - kth) <= 2 * bound[b, j]


def _sparse_ref(q, lat, idx, Dv, scale):
    return oracle.attn_sparse(W.bf16_bits(q), W.bf16_bits(lat), idx.numpy(), Dv, scale)


@pytest.mark.parametrize("Hq,L,k", [(128, 3000, 700), (64, 600, 2048), (128, 5000, 256), (128, 2100, 2048),
                                    (128, 300, 128), (64, 50, 1), (128, 1000, 129)])
def test_sparse_attention(K, Hq, L, k):
    wl = W.DSA_128K
    B = 2
    gen = W.generator(900 + Hq + L + k)
    q = W.normal_bf16((B, Hq, wl.Dk), gen)
    lat = W.normal_bf16((B, L, wl.Dk), gen)
    idx = torch.stack([torch.randperm(L, generator=gen)[:k] if k <= L else
                       torch.cat([torch.randperm(L, generator=gen), torch.full((k - L,), -1)])
                       for _ in range(B)]).to(torch.int32)
    idx[1, ::7] = -1  # unused slots anywhere in the list
    out, lse = K.attn_decode_sparse(q.cuda(), lat.cuda(), idx.cuda(), wl.Dv, wl.sparse_scale)
    torch.cuda.synchronize()
    ro, rl = _sparse_ref(q, lat, idx, wl.Dv, wl.sparse_scale)
    assert_attn_close(out, ro, lse, rl, f"sparse Hq={Hq} k={k}")


def test_sparse_attention_full_size(K):
    """B=8, 128 heads, 2048 of 131072 latent rows of width 576 (values 512)."""
    wl = W.DSA_128K
    dev = torch.device("cuda")
    gen = W.generator(W.SEED_BASE + wl.index + 200, dev)
    q = W.normal_bf16((wl.B, wl.Hq, wl.Dk), gen, dev)
    lat = W.normal_bf16((wl.B, wl.L, wl.Dk), gen, dev)
    cpu_gen = W.generator(4242)
    idx = torch.stack([torch.randperm(wl.L, generator=cpu_gen)[:wl.k] for _ in range(wl.B)]).to(torch.int32)
    out, lse = K.attn_decode_sparse(q, lat, idx.to(dev), wl.Dv, wl.sparse_scale)
    torch.cuda.synchronize()
    # the oracle needs only the selected rows: gather them on the host side
    rows = torch.stack([lat[b, idx[b].long().to(dev)] for b in range(wl.B)]).cpu()
    local = torch.arange(wl.k, dtype=torch.int32).repeat(wl.B, 1)
    ro, rl = _sparse_ref(q.cpu(), rows, local, wl.Dv, wl.sparse_scale)
    assert_attn_close(out, ro, lse, rl, "sparse full size")


def test_sparse_bad_index_is_skipped_and_flagged(K):
    wl = W.DSA_128K
    B, Hq, L, k = 1, 64, 100, 40
    gen = W.generator(3)
    q = W.normal_bf16((B, Hq, wl.Dk), gen)
    lat = W.normal_bf16((B, L, wl.Dk), gen)
    idx = torch.arange(k, dtype=torch.int32)[None].clone()
    bad = idx.clone()
    bad[0, 3] = 1000
    bad[0, 9] = -5
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, lse = K.attn_decode_sparse(q.cuda(), lat.cuda(), bad.cuda(), wl.Dv, 0.07, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) & K.STATUS_BAD_INDEX
    ok = idx.clone()
    ok[0, 3] = -1
    ok[0, 9] = -1
    ro, rl = _sparse_ref(q, lat, ok, wl.Dv, 0.07)
    assert_attn_close(out, ro, lse, rl, "bad index")


def test_sparse_row_without_valid_index(K):
    """A row whose selection is all -1 gives out = 0 and lse = -inf; the other row is unaffected."""
    wl = W.DSA_128K
    B, Hq, L, k = 2, 128, 400, 300
    gen = W.generator(17)
    q = W.normal_bf16((B, Hq, wl.Dk), gen)
    lat = W.normal_bf16((B, L, wl.Dk), gen)
    idx = torch.stack([torch.randperm(L, generator=gen)[:k] for _ in range(B)]).to(torch.int32)
    idx[0] = -1
    out, lse = K.attn_decode_sparse(q.cuda(), lat.cuda(), idx.cuda(), wl.Dv, wl.sparse_scale)
    torch.cuda.synchronize()
    assert torch.all(out[0] == 0) and torch.all(torch.isneginf(lse[0]))
    ro, rl = _sparse_ref(q[1:], lat[1:], idx[1:], wl.Dv, wl.sparse_scale)
    assert_attn_close(out[1:], ro, lse[1:], rl, "row 1 next to an empty row")


@pytest.mark.parametrize("B", [2, 10])
def test_sparse_merge_paths_and_workspace_counters(K, B):
    """B * 16 chunks <= the SM count: the kernel merges the chunk parts itself (cooperative
    launch, per-row counters in the workspace); B = 10 (160 CTAs): the merge kernel does.
    Both against the oracle; the counters are zero after each call, and a second call on
    the same workspace gives the same bits."""
    wl = W.DSA_128K
    Hq, L, k = 64, 3000, 2048
    gen = W.generator(2100 + B)
    q = W.normal_bf16((B, Hq, wl.Dk), gen)
    lat = W.normal_bf16((B, L, wl.Dk), gen)
    idx = torch.stack([torch.randperm(L, generator=gen)[:k] for _ in range(B)]).to(torch.int32)
    idx[0, 100:300] = -1
    ws = K.workspace(K.attn_decode_sparse_workspace_bytes(B, Hq, wl.Dv, k))
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    out1, lse1 = K.attn_decode_sparse(q.cuda(), lat.cuda(), idx.cuda(), wl.Dv, wl.sparse_scale, ws=ws, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert int(ws[:8 * B].count_nonzero()) == 0
    out2, lse2 = K.attn_decode_sparse(q.cuda(), lat.cuda(), idx.cuda(), wl.Dv, wl.sparse_scale, ws=ws)
    torch.cuda.synchronize()
    assert torch.equal(out1, out2) and torch.equal(lse1, lse2)
    ro, rl = _sparse_ref(q, lat, idx, wl.Dv, wl.sparse_scale)
    assert_attn_close(out1, ro, lse1, rl, f"sparse merge path B={B}")


def test_selection_workspace_counts_are_left_zero(K):
    """The indexers count the top-k's first digit into the workspace's histogram region
    and the top-k clears it: zero after every call, and calls on a reused workspace give
    the same selection (bf16 indexer, FP8 indexer, group selection)."""
    wl = W.DSA_128K
    B, L, k = 3, 6000, 2048
    inp = W.dsa_inputs(wl, B=B, L=L, seed=88, with_latent=False)
    q_idx, w, k_idx = inp["q_idx"].cuda(), inp["w"].cuda(), inp["k_idx"].cuda()
    lens = torch.tensor([6000, 2500, 1000], dtype=torch.int32).cuda()
    hist_bytes = B * 2048 * 4 + B * 4  # first-digit counts, then the indexer's per-row claim counters
    ws = K.workspace(K.dsa_index_topk_workspace_bytes(B, L, k))
    first = K.dsa_index_topk(q_idx, w, k_idx, k, seq_lens=lens, ws=ws)[0].clone()
    torch.cuda.synchronize()
    assert int(ws[:hist_bytes].count_nonzero()) == 0
    again = K.dsa_index_topk(q_idx, w, k_idx, k, seq_lens=lens, ws=ws)[0]
    torch.cuda.synchronize()
    assert torch.equal(first, again) and int(ws[:hist_bytes].count_nonzero()) == 0
    codes, sc = K.idx_key_quant_fp8(k_idx)
    f8 = K.dsa_index_topk_fp8(q_idx, w, codes, sc, k, seq_lens=lens, ws=ws)[0].clone()
    f8b = K.dsa_index_topk_fp8(q_idx, w, codes, sc, k, seq_lens=lens, ws=ws)[0]
    torch.cuda.synchronize()
    assert torch.equal(f8, f8b) and int(ws[:hist_bytes].count_nonzero()) == 0
    # group selection over 4-token group keys
    cos, sin = K.rope_table_build(K.rope_params(128, base=500000.0), L)
    kb = K.qsa_block_keys(k_idx, lens, cos, sin)
    ws2 = K.workspace(K.qsa_select_workspace_bytes(B, L, 512))
    t1, c1, _ = K.qsa_select(q_idx, w, kb, lens, n_top=512, ws=ws2)
    t1 = t1.clone()
    t2, c2, _ = K.qsa_select(q_idx, w, kb, lens, n_top=512, ws=ws2)
    torch.cuda.synchronize()
    assert torch.equal(t1, t2) and int(ws2[:hist_bytes].count_nonzero()) == 0
