"""The lightning indexer sharded over L, emulated on one GPU: the keys of every row
are cut into n slices; each slice runs dsa_index_topk on its own keys (its lengths
from shard_lengths), dsa_topk_candidates turns its selection into (score, global
index) pairs, the parts are concatenated in slice order (what the all-gather of
shard.gather_candidates produces), and dsa_topk_merge selects from them.  The result
must equal dsa_index_topk over the whole rows bit for bit -- the scores of a token do
not depend on the slicing -- including ties that straddle slice boundaries.  The
exchange itself is tested with two gloo ranks on CPU (test_shard_dist.py)."""
import numpy as np
import pytest
import torch

import oracle
from mqa_kv_cache_b200 import shard
from mqa_kv_cache_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def K():
    from mqa_kv_cache_b200 import kvattn
    return kvattn


def _sharded(K, q_idx, w, k_idx, k, n, lens):
    B, L, _ = k_idx.shape
    S = L // n
    cs, ci = [], []
    for r in range(n):
        my = shard.shard_lengths(lens, r, S)
        idx, scores = K.dsa_index_topk(q_idx, w, k_idx[:, r * S:(r + 1) * S].contiguous(), k, seq_lens=my)
        c_s, c_i = K.dsa_topk_candidates(scores, idx, r * S)
        cs.append(c_s)
        ci.append(c_i)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = K.dsa_topk_merge(torch.stack(cs), torch.stack(ci), dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    return out


@pytest.mark.parametrize("n,L,k", [(2, 4096, 64), (4, 8192, 2048), (2, 6000, 2048), (8, 131072, 2048)])
def test_sharded_topk_equals_unsharded(K, n, L, k):
    wl = W.DSA_128K
    B = 4
    inp = W.dsa_inputs(wl, B=B, L=L, seed=600 + n + L, with_latent=False)
    q_idx, w, k_idx = inp["q_idx"].cuda(), inp["w"].cuda(), inp["k_idx"].cuda()
    S = L // n
    # equal scores on both sides of every slice boundary: duplicated key rows
    for r in range(1, n):
        k_idx[:, r * S:r * S + 40] = k_idx[:, r * S - 40:r * S]
    lens = torch.tensor([L, L - S // 2, S + 7, 3 * k // 4 + 1], dtype=torch.int32).clamp(max=L).cuda()
    want, scores = K.dsa_index_topk(q_idx, w, k_idx, k, seq_lens=lens)
    got = _sharded(K, q_idx, w, k_idx, k, n, lens)
    assert torch.equal(got, want)
    # and the unsharded selection is the oracle's on the kernel's scores (ties to the lower index)
    ref = oracle.topk(scores.cpu().numpy(), k, lens=lens.cpu().numpy())
    sel = want.cpu().numpy()
    for b in range(B):
        np.testing.assert_array_equal(sel[b][sel[b] >= 0], np.sort(ref[b][ref[b] >= 0]))


def test_merge_takes_all_when_fewer_valid_than_k(K):
    cs = torch.tensor([[[3.0, 1.0, -np.inf]], [[2.0, -np.inf, -np.inf]]], dtype=torch.float32, device="cuda")
    ci = torch.tensor([[[4, 9, -1]], [[17, -1, -1]]], dtype=torch.int32, device="cuda")
    out = K.dsa_topk_merge(cs, ci)
    torch.cuda.synchronize()
    assert out.cpu().tolist() == [[4, 9, 17]]
    out = K.dsa_topk_merge(cs[:, :, :2].contiguous(), ci[:, :, :2].contiguous())
    torch.cuda.synchronize()
    assert out.cpu().tolist() == [[4, 17]]  # 3.0 and 2.0 beat 1.0
