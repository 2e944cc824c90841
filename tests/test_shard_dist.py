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
