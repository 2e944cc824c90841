"""GPU parity of attn_prefill_causal (tcgen05 causal attention) against the
fp64 oracle, through the C ABI: ragged prompt lengths around the 128/256-row
tile edges, every group size, the full B=2 x 8192 x 32-head configuration on
sampled rows (first/last rows of tiles and blocks included), and the chain raw
q/k -> RoPE -> prefill."""
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


def _inputs(B, T, H, Hk, seed, d=128):
    gen = W.generator(seed)
    return (W.normal_bf16((B, T, H, d), gen), W.normal_bf16((B, Hk, T, d), gen),
            W.normal_bf16((B, Hk, T, d), gen))


def _run(K, q, k, v, scale):
    out, lse = K.attn_prefill_causal(q.cuda(), k.cuda(), v.cuda(), scale)
    torch.cuda.synchronize()
    return out, lse


@pytest.mark.parametrize("T", [1, 2, 127, 128, 129, 255, 256, 257, 300, 513])
def test_lengths_around_tile_edges(K, T):
    B, H, Hk = 2, 4, 2
    q, k, v = _inputs(B, T, H, Hk, 100 + T)
    out, lse = _run(K, q, k, v, 128 ** -0.5)
    ro, rl = oracle.attn_prefill(W.bf16_bits(q), W.bf16_bits(k), W.bf16_bits(v), 128 ** -0.5)
    assert_attn_close(out, ro, lse, rl, f"T={T}")


@pytest.mark.parametrize("H,Hk", [(4, 4), (8, 1), (16, 2), (64, 1), (32, 1)])
def test_group_sizes(K, H, Hk):
    B, T = 1, 384
    q, k, v = _inputs(B, T, H, Hk, 7 * H + Hk)
    out, lse = _run(K, q, k, v, 0.09)
    ro, rl = oracle.attn_prefill(W.bf16_bits(q), W.bf16_bits(k), W.bf16_bits(v), 0.09)
    assert_attn_close(out, ro, lse, rl, f"H={H} Hk={Hk}")


def test_large_logits_rescale_path(K):
    # a large scale makes the running max jump between tiles (the O rescale path)
    B, T, H, Hk = 1, 1024, 2, 1
    q, k, v = _inputs(B, T, H, Hk, 5)
    out, lse = _run(K, q, k, v, 1.0)
    ro, rl = oracle.attn_prefill(W.bf16_bits(q), W.bf16_bits(k), W.bf16_bits(v), 1.0)
    assert_attn_close(out, ro, lse, rl, "scale 1.0")


def test_full_size_sampled_rows(K):
    """B=2, T=8192, H=32, Hk=8, d=128, drawn on the device; the oracle checks
    sampled (batch, head, row) outputs one by one."""
    wl = W.PREFILL_8K
    dev = torch.device("cuda")
    gen = W.generator(W.SEED_BASE + wl.index + 100, dev)
    q = W.normal_bf16((wl.B, wl.T, wl.H, wl.d), gen, dev)
    k = W.normal_bf16((wl.B, wl.Hk, wl.T, wl.d), gen, dev)
    v = W.normal_bf16((wl.B, wl.Hk, wl.T, wl.d), gen, dev)
    out, lse = K.attn_prefill_causal(q, k, v, wl.scale)
    torch.cuda.synchronize()
    rng = np.random.default_rng(11)
    rows = [0, 1, 127, 128, 255, 256, 4095, 4096, 8063, 8064, 8191] + list(rng.integers(0, wl.T, 21))
    sel = [(int(rng.integers(wl.B)), int(rng.integers(wl.H)), int(i)) for i in rows]
    sel += [(wl.B - 1, wl.H - 1, wl.T - 1), (0, 0, 0)]
    qb, kb, vb = W.bf16_bits(q), W.bf16_bits(k), W.bf16_bits(v)
    ro, rl = oracle.attn_prefill(qb, kb, vb, wl.scale, sel=sel)
    got = torch.stack([out[b, i, h] for b, h, i in sel])
    got_l = torch.stack([lse[b, h, i] for b, h, i in sel])
    assert_attn_close(got, ro, got_l, rl, "prefill full size")


def test_chain_rope_then_prefill(K):
    wl = W.PREFILL_8K
    B, T = 1, 640
    inp = W.prefill_inputs(wl, B=B, T=T)
    r = wl.rope
    p = K.rope_params(wl.d, base=r.base)
    cos, sin = K.rope_table_build(p, T)
    qg, kg = inp["q"].cuda(), inp["k"].cuda()
    pos = inp["pos"].cuda()
    K.rope_apply_qk(qg, pos, kg, pos, cos, sin, q_layout="bthd", k_layout="bhtd")
    out, lse = K.attn_prefill_causal(qg, kg, inp["v"].cuda(), wl.scale)
    torch.cuda.synchronize()
    c, s = oracle.rope_table(wl.d, r.base, T)
    qr = oracle.rope_apply(W.bf16_bits(inp["q"]), inp["pos"].numpy(), c, s)
    kr = oracle.rope_apply(W.bf16_bits(inp["k"]), inp["pos"].numpy(), c, s, layout="bhtd")
    vr = oracle.bf16_bits_to_f64(W.bf16_bits(inp["v"]))
    ro, rl = oracle.attn_prefill(qr, kr, vr, wl.scale)
    qn = np.linalg.norm(qr, axis=-1).transpose(0, 2, 1)  # [B, H, T] like lse
    kmax = np.linalg.norm(kr, axis=-1).max(axis=-1)       # [B, Hk]
    kmax_h = np.repeat(kmax, wl.H // wl.Hk, axis=1)[:, :, None]
    assert_attn_close(out, ro, lse, rl, "chain prefill", lse_tol=chain_lse_tol(qn, kmax_h, wl.scale))
    # the attention step alone on the GPU-rotated q and k: the plain lse tolerance
    ro2, rl2 = oracle.attn_prefill(W.bf16_bits(qg.cpu()), W.bf16_bits(kg.cpu()), W.bf16_bits(inp["v"]), wl.scale)
    assert_attn_close(out, ro2, lse, rl2, "chain prefill on the GPU-rotated q/k")


def test_deterministic(K):
    q, k, v = _inputs(1, 700, 8, 2, 3)
    a = _run(K, q, k, v, 0.1)
    b = _run(K, q, k, v, 0.1)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


@pytest.mark.parametrize("T,n_sink,window", [(700, 4, 200), (513, 0, 128), (1000, 16, 300), (300, 3, 1),
                                             (900, 130, 256), (385, 0, 129)])
def test_window_prefill_against_oracle(K, T, n_sink, window):
    """Row i sees keys j <= i with j > i - window or j < n_sink: sampled rows (every
    third, plus the 128-row tile edges) against the row-by-row windowed decode."""
    B, H, Hk = 1, 4, 2
    q, k, v = _inputs(B, T, H, Hk, 300 + T + window)
    out, lse = K.attn_prefill_causal_window(q.cuda(), k.cuda(), v.cuda(), 128 ** -0.5, n_sink, window)
    torch.cuda.synchronize()
    rows = sorted(set(range(0, T, 3)) | {r for r in (127, 128, 255, 256, 383, 384, 511, 512) if r < T} | {T - 1})
    sel = [(0, h, i) for h in (0, 3) for i in rows]
    ro, rl = oracle.attn_prefill_window(W.bf16_bits(q), W.bf16_bits(k), W.bf16_bits(v), 128 ** -0.5, n_sink, window,
                                        sel)
    got = torch.stack([out[b, i, h] for b, h, i in sel])
    got_l = torch.stack([lse[b, h, i] for b, h, i in sel])
    assert_attn_close(got, ro, got_l, rl, f"window prefill T={T} s={n_sink} w={window}")


def test_window_longer_than_prompt_is_plain_causal(K):
    q, k, v = _inputs(2, 600, 8, 2, 41)
    a = K.attn_prefill_causal_window(q.cuda(), k.cuda(), v.cuda(), 0.1, 0, 600)
    b = K.attn_prefill_causal(q.cuda(), k.cuda(), v.cuda(), 0.1)
    torch.cuda.synchronize()
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])
