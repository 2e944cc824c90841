"""The exchange step of a sequence-sharded decode, on CPU: two gloo ranks each
decode their slice of one cache with the fp64 oracle, gather_parts all-gathers the
(out, lse) pairs in rank order, and the oracle's softmax merge of the parts equals
the oracle's decode over the whole cache (the merge kernel itself is tested on
the GPU in test_gpu_merge.py)."""
import os
import socket
import sys
from datetime import timedelta

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs():
    rng = np.random.default_rng(5)
    B, H, Hk, d, T = 3, 4, 2, 16, 40
    q, k, v = rng.standard_normal((B, H, d)), rng.standard_normal((B, Hk, T, d)), rng.standard_normal((B, Hk, T, d))
    lens = np.array([40, 13, 27], np.int32)  # row 1 ends inside slice 0: slice 1 sees nothing of it
    return q, k, v, lens


def _worker(rank, world, port, out_dir):
    sys.path.insert(0, ROOT)
    import oracle
    from mqa_kv_cache_b200 import shard
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=timedelta(seconds=60))
    try:
        q, k, v, lens = _inputs()
        shard_len = k.shape[2] // world
        my = shard.shard_lengths(torch.from_numpy(lens), rank, shard_len).numpy()
        sl = slice(rank * shard_len, (rank + 1) * shard_len)
        o, l = oracle.attn_decode(q, np.ascontiguousarray(k[:, :, sl]), np.ascontiguousarray(v[:, :, sl]), my, 0.3)
        o_parts, l_parts = shard.gather_parts(torch.from_numpy(o), torch.from_numpy(l))
        np.save(os.path.join(out_dir, f"parts{rank}.npy"), o_parts.numpy())
        np.save(os.path.join(out_dir, f"lse{rank}.npy"), l_parts.numpy())
        np.save(os.path.join(out_dir, f"my{rank}.npy"), my)
    finally:
        dist.destroy_process_group()


def test_two_ranks_gather_and_merge(tmp_path):
    import oracle
    world = 2
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    q, k, v, lens = _inputs()
    full_o, full_l = oracle.attn_decode(q, k, v, lens, 0.3)
    parts = [np.load(tmp_path / f"parts{r}.npy") for r in range(world)]
    lses = [np.load(tmp_path / f"lse{r}.npy") for r in range(world)]
    assert np.array_equal(parts[0], parts[1]) and np.array_equal(lses[0], lses[1])  # every rank gathers the same
    assert list(np.load(tmp_path / "my0.npy")) == [20, 13, 20]
    assert list(np.load(tmp_path / "my1.npy")) == [20, 0, 7]
    B, H = lens.shape[0], q.shape[1]
    for b in range(B):
        for h in range(H):
            o, l = oracle.softmax_merge(parts[0][:, b, h], lses[0][:, b, h])
            np.testing.assert_allclose(o, full_o[b, h], rtol=1e-12, atol=1e-12)
            np.testing.assert_allclose(l, full_l[b, h], rtol=1e-12)


def test_shard_lengths_partition_every_row():
    """The slices' lengths add up to the row's length (capped at the slices' total) and
    each slice's rows are a prefix of it."""
    from mqa_kv_cache_b200 import shard
    lens = torch.tensor([0, 1, 99, 100, 101, 250, 400], dtype=torch.int32)
    S, n = 100, 4
    parts = torch.stack([shard.shard_lengths(lens, r, S) for r in range(n)])
    assert parts.dtype == torch.int32
    assert torch.equal(parts.sum(0), lens.clamp(max=S * n))
    assert torch.all((parts >= 0) & (parts <= S))
    # a slice is full before the next one holds anything
    for r in range(n - 1):
        assert torch.all((parts[r + 1] == 0) | (parts[r] == S))


def _index_inputs():
    rng = np.random.default_rng(9)
    B, HI, dI, L = 3, 8, 16, 96
    q = rng.standard_normal((B, HI, dI))
    w = rng.uniform(0, 1, (B, HI)).astype(np.float32)
    kk = rng.standard_normal((B, L, dI))
    kk[:, 50:60] = kk[:, 10:20]       # equal scores on both sides of the slice boundary (48)
    lens = np.array([96, 30, 61], np.int32)
    to_bits = lambda x: torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).view(torch.uint16).numpy()
    return to_bits(q), w, to_bits(kk), lens


def _index_worker(rank, world, port, out_dir, k):
    sys.path.insert(0, ROOT)
    import oracle
    from mqa_kv_cache_b200 import shard
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=timedelta(seconds=60))
    try:
        q, w, kk, lens = _index_inputs()
        S = kk.shape[1] // world
        my = shard.shard_lengths(torch.from_numpy(lens), rank, S).numpy()
        sc = oracle.dsa_scores(q, w, np.ascontiguousarray(kk[:, rank * S:(rank + 1) * S]), my)
        loc = oracle.topk(sc, k, lens=my)                                   # [B, k] local, -1 padded
        cs = np.where(loc >= 0, np.take_along_axis(sc, np.maximum(loc, 0), 1), -np.inf).astype(np.float32)
        ci = np.where(loc >= 0, loc + rank * S, -1).astype(np.int32)
        cs_all, ci_all = shard.gather_candidates(torch.from_numpy(cs), torch.from_numpy(ci))
        np.save(os.path.join(out_dir, f"cs{rank}.npy"), cs_all.numpy())
        np.save(os.path.join(out_dir, f"ci{rank}.npy"), ci_all.numpy())
    finally:
        dist.destroy_process_group()


def test_two_ranks_indexer_candidates_give_the_global_topk(tmp_path):
    """Each rank keeps the top-k of its key slice; the union of the gathered candidates
    holds the global top-k, ties across the slice boundary included."""
    import oracle
    world, k = 2, 12
    mp.start_processes(_index_worker, args=(world, _free_port(), str(tmp_path), k), nprocs=world, join=True,
                       start_method="spawn")
    q, w, kk, lens = _index_inputs()
    cs = [np.load(tmp_path / f"cs{r}.npy") for r in range(world)]
    ci = [np.load(tmp_path / f"ci{r}.npy") for r in range(world)]
    assert np.array_equal(cs[0], cs[1]) and np.array_equal(ci[0], ci[1])
    assert cs[0].shape == (world, 3, k)
    full = oracle.dsa_scores(q, w, kk, lens)
    want = oracle.topk(full, k, lens=lens)
    B, L = full.shape
    for b in range(B):
        union = np.full(L, -np.inf)
        for p in range(world):
            sel = ci[0][p, b] >= 0
            assert np.all(ci[0][p, b][sel] // (L // world) == p)            # part p holds slice p's indices
            union[ci[0][p, b][sel]] = cs[0][p, b][sel]
        n_valid = int(lens[b])
        got = oracle.topk(union[None], k, lens=np.array([L], np.int32))[0]
        got = got[:min(k, n_valid)]
        np.testing.assert_array_equal(got, want[b][:min(k, n_valid)])
