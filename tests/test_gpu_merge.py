"""GPU parity of attn_merge_lse (decode results over disjoint key sets merged into
the decode over their union), alone against the oracle's softmax merge, and as the
last step of a sequence-sharded decode emulated on one GPU: the cache cut into
slices, attn_decode_gqa on each slice, the parts merged, against the oracle's
decode over the whole cache."""
import numpy as np
import pytest
import torch

import oracle
from mqa_kv_cache_b200 import shard
from mqa_kv_cache_b200 import workloads as W
from tests.gpu_util import assert_attn_close, to_np_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def K():
    from mqa_kv_cache_b200 import kvattn
    return kvattn


@pytest.mark.parametrize("n,d", [(1, 128), (3, 64), (8, 128), (40, 128)])
def test_merge_against_oracle(K, n, d):
    B, H = 3, 16
    gen = W.generator(700 + n + d)
    o_parts = W.normal_bf16((n, B, H, d), gen)
    lse = torch.randn((n, B, H), generator=W.generator(701 + n)) * 4.0
    lse[0, 0, :] = -float("inf")             # an empty part
    lse[:, 1, 3] = -float("inf")             # a head whose every part is empty
    out, lse_out = K.attn_merge_lse(o_parts.cuda(), lse.float().cuda())
    torch.cuda.synchronize()
    ob = oracle.bf16_bits_to_f64(W.bf16_bits(o_parts))
    ln = lse.double().numpy()
    got, gl = to_np_f64(out), lse_out.cpu().numpy()
    for b in range(B):
        for h in range(H):
            if np.all(np.isneginf(ln[:, b, h])):
                assert np.all(got[b, h] == 0) and np.isneginf(gl[b, h])
                continue
            ro, rl = oracle.softmax_merge(ob[:, b, h], ln[:, b, h])
            assert np.max(np.abs(got[b, h] - ro)) <= 2e-2 and abs(gl[b, h] - rl) <= 1e-4 * max(1.0, abs(rl))


@pytest.mark.parametrize("n_shards,H,Hk", [(2, 32, 8), (4, 64, 1), (8, 8, 8)])
def test_sharded_decode_emulated(K, n_shards, H, Hk):
    """Slice r of the cache holds positions r * S .. (r + 1) * S - 1; each slice is decoded on
    its own (as rank r would) and the parts merged; some rows end inside the first slices."""
    B, d, T = 4, 128, 2048
    S = T // n_shards
    gen = W.generator(710 + n_shards)
    q = W.normal_bf16((B, H, d), gen)
    k = W.normal_bf16((B, Hk, T, d), gen)
    v = W.normal_bf16((B, Hk, T, d), gen)
    lens = torch.tensor([T, S // 2, T - 5, 0], dtype=torch.int32)
    outs, lses = [], []
    for r in range(n_shards):
        ks = k[:, :, r * S:(r + 1) * S].contiguous().cuda()
        vs = v[:, :, r * S:(r + 1) * S].contiguous().cuda()
        o, l = K.attn_decode_gqa(q.cuda(), ks, vs, shard.shard_lengths(lens, r, S).cuda(), d ** -0.5)
        outs.append(o)
        lses.append(l)
    out, lse = K.attn_merge_lse(torch.stack(outs), torch.stack(lses))
    full_o, full_l = K.attn_decode_gqa(q.cuda(), k.cuda(), v.cuda(), lens.cuda(), d ** -0.5)
    torch.cuda.synchronize()
    ro, rl = oracle.attn_decode(W.bf16_bits(q), W.bf16_bits(k), W.bf16_bits(v), lens.numpy(), d ** -0.5)
    assert_attn_close(out, ro, lse, rl, f"sharded n={n_shards}")
    assert torch.all(out[3] == 0) and torch.all(torch.isneginf(lse[3]))
    # against the one-call decode: the same result up to the bf16 rounding of the parts
    assert (out.float() - full_o.float()).abs().max().item() <= 2e-2
