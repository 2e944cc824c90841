"""Failure detection on the GPU without a fault.

Every pipeline wait in the kernels is bounded; when one runs out the kernel
stops using its pipeline, sets KVATTN_STATUS_TIMEOUT in dev_status and returns,
and the context stays usable.  kvattn_test_decode_stall makes such a wait run
out on purpose: the decode's first CTA never issues the loads of one tile (a
barrier phase that nothing completes), with each wait limited to a few
milliseconds.  No load is issued and abandoned, nothing faults or traps.  The
tests check the status bit, that the call returns quickly, and that after the
workspace's counter region is cleared the next normal call is correct."""
import time

import pytest
import torch

import oracle
from mqa_kv_cache_b200 import workloads as W
from tests.gpu_util import assert_attn_close

pytestmark = pytest.mark.gpu

ZERO_BYTES = 64 << 10  # KVATTN_DECODE_WS_ZERO_BYTES
LIMIT_NS = 2_000_000   # 2 ms per wait while the stall is set


@pytest.fixture(scope="module")
def K():
    from mqa_kv_cache_b200 import kvattn
    return kvattn


def _inputs(B, H, Hk, d, T, seed):
    gen = W.generator(seed)
    q = W.normal_bf16((B, H, d), gen)
    k = W.normal_bf16((B, Hk, T, d), gen)
    v = W.normal_bf16((B, Hk, T, d), gen)
    lens = torch.randint(T // 2, T + 1, (B,), generator=torch.Generator().manual_seed(seed), dtype=torch.int32)
    return q, k, v, lens


@pytest.mark.parametrize("B,H,Hk,d,T", [(2, 16, 2, 128, 3000), (3, 8, 1, 64, 5000)])
def test_stalled_decode_reports_timeout_then_recovers(K, B, H, Hk, d, T):
    q, k, v, lens = _inputs(B, H, Hk, d, T, 900 + d)
    qg, kg, vg, lg = q.cuda(), k.cuda(), v.cuda(), lens.cuda()
    scale = d ** -0.5
    ws = K.workspace(K.attn_decode_gqa_workspace_bytes(B, H, Hk, d, T))
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    K.kvattn_test_decode_stall(0, LIMIT_NS)
    try:
        t0 = time.perf_counter()
        K.attn_decode_gqa(qg, kg, vg, lg, scale, ws=ws, dev_status=st)
        torch.cuda.synchronize()
        elapsed = time.perf_counter() - t0
    finally:
        K.kvattn_test_decode_stall(-1, 0)
    assert int(st.item()) & K.STATUS_TIMEOUT, "the stalled call must report a timeout"
    assert elapsed < 2.0, f"a stalled call took {elapsed:.3f} s with 2 ms waits"
    # the context is usable; clear the counters the aborted call may have left, run again
    ws[:ZERO_BYTES].zero_()
    st.zero_()
    out, lse = K.attn_decode_gqa(qg, kg, vg, lg, scale, ws=ws, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert int(ws[:ZERO_BYTES].count_nonzero()) == 0
    ro, rl = oracle.attn_decode(W.bf16_bits(q), W.bf16_bits(k), W.bf16_bits(v), lens.numpy(), scale)
    assert_attn_close(out, ro, lse, rl, f"after a stall B={B} H={H} Hk={Hk} d={d}")


def test_stall_setting_is_checked_and_off_by_default(K):
    with pytest.raises(K.KvattnError):
        K.kvattn_test_decode_stall(-2, 0)
    with pytest.raises(K.KvattnError):
        K.kvattn_test_decode_stall(0, -1)
    # without a stall the same call reports nothing
    q, k, v, lens = _inputs(2, 16, 2, 128, 3000, 905)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    K.attn_decode_gqa(q.cuda(), k.cuda(), v.cuda(), lens.cuda(), 128 ** -0.5, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
