"""Host side of bench.py's multi-rank path, on CPU: two gloo ranks take the
same barrier and reductions the NCCL ranks take on GPUs (weak scaling: bytes
summed over ranks, step time = max over ranks), every rank draws its own
batch, and the reference arm runs on rank 0 alone."""
import json
import os
import socket
import subprocess
import sys
from datetime import timedelta

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    sys.path.insert(0, ROOT)
    import bench
    from mqa_kv_cache_b200 import workloads as W
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=timedelta(seconds=60))
    try:
        dev = torch.device("cpu")
        w = W.LLAMA3_8B_DECODE
        seed = bench.rank_seed(w, rank)
        lens = W.lengths(w.B, w.T_lo, w.T_hi, seed)
        local_bytes = bench.decode_bytes(w, lens)
        local_ms = 1.0 + 0.25 * rank
        bench.barrier(world)
        total, ms = bench.whole_job(local_bytes, local_ms, world, dev)
        bench.barrier(world)
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump({"seed": seed, "lens": lens.tolist(), "local_bytes": local_bytes, "total": total,
                       "ms": ms}, f)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_weak_scaling(tmp_path):
    world = 2
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    r = [json.load(open(tmp_path / f"rank{i}.json")) for i in range(world)]
    # each rank its own batch
    assert r[0]["seed"] != r[1]["seed"]
    assert r[0]["lens"] != r[1]["lens"]
    # every rank sees the same whole-job figures: bytes summed, time maxed
    for x in r:
        assert x["total"] == r[0]["local_bytes"] + r[1]["local_bytes"]
        assert x["ms"] == 1.25


def test_single_rank_reductions_are_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.whole_job(123, 4.5, 1, torch.device("cpu")) == (123.0, 4.5)


def test_decode_bytes_counts_each_row_once():
    sys.path.insert(0, ROOT)
    import bench
    from mqa_kv_cache_b200 import workloads as W
    w = W.TINY_GQA
    lens = torch.tensor([3, 5] + [1] * (w.B - 2), dtype=torch.int32)
    kv = int(lens.sum()) * w.Hk * w.d * 2 * 2      # K and V rows, bf16
    q_out = 2 * w.B * w.H * w.d * 2                 # q read, out written, bf16
    assert bench.decode_bytes(w, lens) == kv + q_out + w.B * w.H * 4


def test_reference_arm_runs_on_rank0_only():
    env = dict(os.environ, RANK="1", LOCAL_RANK="1", WORLD_SIZE="2")
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "2",
                        "--warmup", "3"], env=env, capture_output=True, text=True, timeout=120, cwd=ROOT)
    assert p.returncode == 0, p.stderr
    assert p.stdout.strip() == ""
