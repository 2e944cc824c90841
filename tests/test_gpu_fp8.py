"""GPU parity of the FP8 (E4M3) cache path against the oracle, through the C ABI.

Quantisers: latent_quant_fp8 (656-byte rows: 512 codes, 4 fp32 scales, the
bf16 RoPE part) and idx_key_quant_fp8 (128 codes + one scale) are bit-exact
against the oracle's quantiser (scale = absmax / 448 and x / scale in fp32 on
both sides, E4M3 round-to-nearest-even, saturating), on normal data, data
spread over many binades, all-zero groups, signed zeros and ties.

Sparse attention on packed FP8 rows: against the oracle's sparse attention on
the oracle's dequantised rows (value(code) * scale in fp64); the kernel
rounds each dequantised value to bf16 once, inside the benchmark spec's tolerance
(max-abs 2e-2, rel-L2 5e-3; lse 2e-3)."""
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


def _hard_rows(n, width, seed):
    """bf16 rows with the cases a quantiser can get wrong: magnitudes over many
    binades, all-zero groups, signed zeros, values that land on E4M3 ties."""
    gen = torch.Generator().manual_seed(seed)
    x = torch.randn((n, width), generator=gen) * torch.exp(torch.empty((n, 1)).uniform_(-12, 12, generator=gen))
    x[::7, :128] = 0.0                       # an all-zero group
    x[3::11, 5] = -0.0                       # signed zeros next to non-zero values
    x[5::13, :] = 0.0
    x[5::13, 0] = -0.0                       # a row whose first group is -0 and zeros only
    # exact ties: group absmax 448 * 2^-4, other values halfway between E4M3 neighbours
    t = (torch.arange(64) % 15 + 8).float() * 2.0 ** -3 + 2.0 ** -4   # (1 + m/8) + 1/16 on the 2^0 binade
    x[1::9, :64] = (t * 2.0 ** -4)[None, :]
    x[1::9, 64] = 448 * 2.0 ** -4
    return x.to(torch.bfloat16)


@pytest.mark.parametrize("n", [1, 5, 4099])
def test_latent_quant_is_bit_exact(K, n):
    x = _hard_rows(n, 576, 100 + n)
    got = K.latent_quant_fp8(x.cuda())
    torch.cuda.synchronize()
    ref = oracle.latent_pack_fp8(W.bf16_bits(x))
    np.testing.assert_array_equal(got.cpu().numpy(), ref)


@pytest.mark.parametrize("n", [1, 2, 3, 4097])
def test_idx_key_quant_is_bit_exact(K, n):
    x = _hard_rows(n, 128, 200 + n)
    codes, scales = K.idx_key_quant_fp8(x.cuda())
    torch.cuda.synchronize()
    rc, rs = oracle.quant_fp8(W.bf16_bits(x))
    np.testing.assert_array_equal(codes.cpu().numpy(), rc)
    np.testing.assert_array_equal(scales.cpu().numpy().view(np.uint32), rs[:, 0].view(np.uint32))


def _check_fp8_sparse(out, lse, q, packed_rows, idx, Dv, scale, what):
    """(a) Against the oracle on the exactly dequantised rows (value(code) * scale in
    fp64): outputs within the benchmark spec's tolerance; lse within 2e-3 plus the largest
    score change that rounding each dequantised key value to bf16 (relative error
    <= 2^-9) can cause, 2^-9 * scale * max_t sum_i |q_i khat_ti|.
    (b) Against the oracle on the rows the kernel multiplies -- each dequantised value
    rounded to fp32, then to bf16 -- with the plain tolerance, lse 2e-3 included."""
    idx_np = idx.numpy()
    lat = oracle.latent_unpack_fp8(packed_rows)                    # [B, L, 576] fp64
    qd = oracle.bf16_bits_to_f64(W.bf16_bits(q))                   # [B, Hq, 576]
    ro, rl = oracle.attn_sparse(qd, lat, idx_np, Dv, scale)
    sel = np.where(idx_np[..., None] >= 0, np.abs(lat[np.arange(lat.shape[0])[:, None], np.maximum(idx_np, 0)]), 0)
    worst = np.einsum("bhi,bti->bht", np.abs(qd), sel).max(axis=-1)  # [B, Hq]
    assert_attn_close(out, ro, lse, rl, what, lse_tol=2.0 ** -9 * scale * worst + 2e-3)
    lat_bf = torch.from_numpy(lat.astype(np.float32)).to(torch.bfloat16)
    ro2, rl2 = oracle.attn_sparse(W.bf16_bits(q), W.bf16_bits(lat_bf), idx_np, Dv, scale)
    assert_attn_close(out, ro2, lse, rl2, what + " on the bf16-rounded dequantised rows")


@pytest.mark.parametrize("Hq,L,k", [(128, 3000, 700), (64, 600, 2048), (128, 5000, 256), (128, 2100, 2048),
                                    (128, 300, 128), (64, 50, 1), (128, 1000, 129)])
def test_sparse_attention_fp8(K, Hq, L, k):
    wl = W.DSA_128K
    B = 2
    gen = W.generator(1900 + Hq + L + k)
    q = W.normal_bf16((B, Hq, wl.Dk), gen)
    lat = W.normal_bf16((B, L, wl.Dk), gen)
    idx = torch.stack([torch.randperm(L, generator=gen)[:k] if k <= L else
                       torch.cat([torch.randperm(L, generator=gen), torch.full((k - L,), -1)])
                       for _ in range(B)]).to(torch.int32)
    idx[1, ::7] = -1
    packed = K.latent_quant_fp8(lat.cuda())
    out, lse = K.attn_decode_sparse_fp8(q.cuda(), packed, idx.cuda(), wl.Dv, wl.sparse_scale)
    torch.cuda.synchronize()
    _check_fp8_sparse(out, lse, q, packed.cpu().numpy(), idx, wl.Dv, wl.sparse_scale, f"fp8 sparse Hq={Hq} k={k}")


def test_sparse_attention_fp8_full_size(K):
    """B=8, 128 heads, 2048 of 131072 packed FP8 rows (656 bytes each)."""
    wl = W.DSA_128K
    dev = torch.device("cuda")
    gen = W.generator(W.SEED_BASE + wl.index + 300, dev)
    q = W.normal_bf16((wl.B, wl.Hq, wl.Dk), gen, dev)
    lat = W.normal_bf16((wl.B, wl.L, wl.Dk), gen, dev)
    packed = K.latent_quant_fp8(lat)
    del lat
    cpu_gen = W.generator(4343)
    idx = torch.stack([torch.randperm(wl.L, generator=cpu_gen)[:wl.k] for _ in range(wl.B)]).to(torch.int32)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    out, lse = K.attn_decode_sparse_fp8(q, packed, idx.to(dev), wl.Dv, wl.sparse_scale, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    rows = torch.stack([packed[b, idx[b].long().to(dev)] for b in range(wl.B)]).cpu().numpy()
    local = torch.arange(wl.k, dtype=torch.int32).repeat(wl.B, 1)
    _check_fp8_sparse(out, lse, q.cpu(), rows, local, wl.Dv, wl.sparse_scale, "fp8 sparse full size")


def test_sparse_fp8_bad_index_and_empty_row(K):
    wl = W.DSA_128K
    B, Hq, L, k = 2, 128, 400, 300
    gen = W.generator(23)
    q = W.normal_bf16((B, Hq, wl.Dk), gen)
    lat = W.normal_bf16((B, L, wl.Dk), gen)
    idx = torch.stack([torch.randperm(L, generator=gen)[:k] for _ in range(B)]).to(torch.int32)
    idx[0] = -1                      # row 0: nothing selected
    bad = idx.clone()
    bad[1, 3] = L + 5                # out of range: skipped and flagged
    bad[1, 8] = -9
    packed = K.latent_quant_fp8(lat.cuda())
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, lse = K.attn_decode_sparse_fp8(q.cuda(), packed, bad.cuda(), wl.Dv, wl.sparse_scale, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) & K.STATUS_BAD_INDEX
    assert torch.all(out[0] == 0) and torch.all(torch.isneginf(lse[0]))
    ok = idx[1:].clone()
    ok[0, 3] = -1
    ok[0, 8] = -1
    _check_fp8_sparse(out[1:], lse[1:], q[1:], packed[1:].cpu().numpy(), ok, wl.Dv, wl.sparse_scale, "fp8 bad index")


# ---- the lightning indexer in fp8 (query heads and keys as E4M3) ------------------------

def _fp8_score_bound(q_bits, w, kd):
    """fp32 error bound of the kernel's scores: exact products of the codes, the
    128-term dot in fp32, the 64-term weighted head sum and the scales (|d| <= 2^-16 *
    sum_j w_j * sum_i |qhat_ji khat_ti|, as for bf16 operands, plus the products'
    rounding); qhat = the query heads as the kernel quantises them."""
    qc, qs = oracle.quant_fp8(q_bits)
    q = oracle.dequant_fp8(qc, qs)
    absdot = np.einsum("bji,bti->btj", np.abs(q), np.abs(kd))
    return 2.0 ** -16 * np.einsum("btj,bj->bt", absdot, w.astype(np.float64)) + 1e-30


def _index_order(idx):
    out = np.full_like(idx, -1)
    for b in range(idx.shape[0]):
        v = np.sort(idx[b][idx[b] >= 0])
        out[b, :len(v)] = v
    return out


@pytest.mark.parametrize("L,k,lens", [(1000, 64, [1000, 777, 5]), (4096, 2048, [4096, 4000, 2049]),
                                      (300, 2048, [300, 1, 0])])
def test_fp8_indexer_and_topk_small(K, L, k, lens):
    wl = W.DSA_128K
    lens_t = torch.tensor(lens, dtype=torch.int32)
    inp = W.dsa_inputs(wl, B=len(lens), L=L, seed=131 + L + k, with_latent=False)
    q_idx, w = inp["q_idx"].cuda(), inp["w"].cuda()
    codes, scales = K.idx_key_quant_fp8(inp["k_idx"].cuda())
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    idx, scores = K.dsa_index_topk_fp8(q_idx, w, codes, scales, k, seq_lens=lens_t.cuda(), dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    idx, scores = idx.cpu().numpy(), scores.cpu().numpy()
    qb, wn = W.bf16_bits(inp["q_idx"]), inp["w"].numpy()
    cn, sn = codes.cpu().numpy(), scales.cpu().numpy()
    ref = oracle.dsa_scores_fp8(qb, wn, cn, sn, lens_t.numpy())
    fin = np.isfinite(ref)
    assert np.array_equal(np.isfinite(scores), fin)
    bound = _fp8_score_bound(qb, wn, oracle.dequant_fp8(cn, sn[..., None]))
    with np.errstate(invalid="ignore"):
        err = np.abs(scores.astype(np.float64) - ref)
    assert np.all(err[fin] <= bound[fin] + 2.0 ** -22 * np.abs(ref[fin]))
    np.testing.assert_array_equal(idx, _index_order(oracle.topk(scores, k, lens=lens_t.numpy())))


def test_fp8_indexer_full_size(K):
    """B=8, L=131072, k=2048 on FP8 keys: selection bit-exact on the kernel's scores for
    every row; scores against the oracle on sampled tokens."""
    wl = W.DSA_128K
    dev = torch.device("cuda")
    gen = W.generator(W.SEED_BASE + wl.index + 400, dev)
    q_idx = W.normal_bf16((wl.B, wl.HI, wl.dI), gen, dev)
    w = W.uniform_f32((wl.B, wl.HI), gen, dev)
    codes, scales = K.idx_key_quant_fp8(W.normal_bf16((wl.B, wl.L, wl.dI), gen, dev))
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    idx, scores = K.dsa_index_topk_fp8(q_idx, w, codes, scales, wl.k, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    idx, scores = idx.cpu().numpy(), scores.cpu().numpy()
    np.testing.assert_array_equal(idx, _index_order(oracle.topk(scores, wl.k)))
    rng = np.random.default_rng(9)
    sample = np.sort(rng.choice(wl.L, 3000, replace=False))
    st_ = torch.from_numpy(sample).to(dev)
    cn, sn = codes[:, st_].cpu().numpy(), scales[:, st_].cpu().numpy()
    qb, wn = W.bf16_bits(q_idx), w.cpu().numpy()
    ref = oracle.dsa_scores_fp8(qb, wn, cn, sn, np.full(wl.B, len(sample), np.int32))
    bound = _fp8_score_bound(qb, wn, oracle.dequant_fp8(cn, sn[..., None]))
    got = scores[:, sample].astype(np.float64)
    assert np.all(np.abs(got - ref) <= bound + 2.0 ** -22 * np.abs(ref))
