"""GPU parity of rope_table_build and rope_apply_qk against the fp64 oracle,
through the C ABI."""
import numpy as np
import pytest
import torch

import oracle
from mqa_kv_cache_b200 import workloads as W
from tests.gpu_util import bf16_ulp, to_np_f64

pytestmark = pytest.mark.gpu

MODES = [
    (W.ROPE_NONE, dict(base=10000.0)),
    (W.ROPE_NONE, dict(base=500000.0)),
    (W.ROPE_PI, dict(base=10000.0, s=4.0)),
    (W.ROPE_NTK, dict(base=10000.0, s=8.0)),
    (W.ROPE_YARN, dict(base=10000.0, s=4.0, L_train=8192.0, alpha=1.0, beta=32.0)),
    (W.ROPE_DYN_NTK, dict(base=500000.0, L_train=4096.0, L_cur=20000.0)),
]


@pytest.fixture(scope="module")
def K():
    from mqa_kv_cache_b200 import kvattn
    return kvattn


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("mode,kw", MODES)
def test_table_matches_oracle(K, d, mode, kw):
    max_pos = 32769
    p = K.rope_params(d, scaling=mode, **kw)
    cos, sin = K.rope_table_build(p, max_pos)
    torch.cuda.synchronize()
    okw = {k: v for k, v in kw.items() if k != "base"}
    c_ref, s_ref = oracle.rope_table(d, kw["base"], max_pos, mode, **okw)
    theta, pos_div, mag = oracle.rope_freqs(d, kw["base"], mode, **okw)
    ang = (np.arange(max_pos, dtype=np.float64)[:, None] / pos_div) * theta[None, :]
    for got, ref in ((cos, c_ref), (sin, s_ref)):
        g = got.cpu().numpy().astype(np.float64)
        # One fp32 ulp for the final rounding, plus the angle's own evaluation
        # error: two fp64 evaluations of m * theta_i agree to a few ulps of the
        # angle (2^-48 |angle| covers 16 ulps), and cos/sin pass an absolute
        # angle error through unchanged (it dominates where cos or sin ~ 0).
        tol = np.abs(ref) * 2.0 ** -23 + mag * (np.abs(ang) + 1.0) * 2.0 ** -48
        bad = np.abs(g - ref) > tol
        assert not bad.any(), f"{bad.sum()} entries off, worst {np.abs(g - ref).max():.3e}"


def _exact_rotation(x_bits, pos, d, mode, kw, pair_style, layout):
    okw = {k: v for k, v in kw.items() if k != "base"}
    c, s = oracle.rope_table(d, kw["base"], int(pos.max()) + 1, mode, **okw)
    return oracle.rope_apply(x_bits, pos, c, s, pair_style=pair_style, layout=layout), c, s


def _assert_rotation_close(got, x_bits, exact, mag):
    """bf16 output within one bf16 ulp of the exact rotation, plus the fp32
    rounding of the table and of the two products."""
    x = oracle.bf16_bits_to_f64(x_bits)
    d = x.shape[-1]
    # |x_a| + |x_b| of each element's pair bounds the fp32 error of the products
    a = np.abs(x)
    err = np.abs(got - exact)
    tol = bf16_ulp(exact) + 2.0 ** -20 * mag * (a + a.max(axis=-1, keepdims=True))
    assert np.all(err <= tol), f"worst excess {(err - tol).max():.3e}"
    assert d > 0


@pytest.mark.parametrize("pair_style", [0, 1])
@pytest.mark.parametrize("mode,kw", [MODES[0], MODES[1], MODES[4]])
def test_apply_prefill_layout(K, pair_style, mode, kw):
    B, T, H, d = 2, 77, 8, 128
    gen = W.generator(101)
    x = W.normal_bf16((B, T, H, d), gen)
    pos = torch.randint(0, 40000, (B, T), generator=gen, dtype=torch.int32)
    bits = W.bf16_bits(x)
    exact, _, _ = _exact_rotation(bits, pos.numpy(), d, mode, kw, pair_style, "bthd")
    p = K.rope_params(d, scaling=mode, pair_style=pair_style, **kw)
    cos, sin = K.rope_table_build(p, int(pos.max()) + 1)
    xg = x.cuda()
    K.rope_apply_qk(xg, pos.cuda(), None, None, cos, sin, q_layout="bthd", pair_style=pair_style)
    torch.cuda.synchronize()
    mag = 0.1 * np.log(kw.get("s", 1.0)) + 1.0 if mode == W.ROPE_YARN else 1.0
    _assert_rotation_close(to_np_f64(xg), bits, exact, mag)


def test_apply_decode_q_and_cache_k_together(K):
    B, H, Hk, T, d = 3, 16, 4, 50, 64
    gen = W.generator(7)
    q = W.normal_bf16((B, H, d), gen)
    k = W.normal_bf16((B, Hk, T, d), gen)
    q_pos = torch.tensor([[50], [7], [49]], dtype=torch.int32)
    k_pos = torch.arange(T, dtype=torch.int32).repeat(B, 1)
    kw = dict(base=10000.0, s=4.0, L_train=8192.0, alpha=1.0, beta=32.0)
    p = K.rope_params(d, scaling=W.ROPE_YARN, **kw)
    cos, sin = K.rope_table_build(p, 64)
    qg, kg = q.cuda(), k.cuda()
    K.rope_apply_qk(qg, q_pos.cuda(), kg, k_pos.cuda(), cos, sin, q_layout="bhd", k_layout="bhtd")
    torch.cuda.synchronize()
    mag = 0.1 * np.log(4.0) + 1.0
    eq, _, _ = _exact_rotation(W.bf16_bits(q)[:, None], q_pos.numpy(), d, W.ROPE_YARN, kw, 0, "bthd")
    _assert_rotation_close(to_np_f64(qg), W.bf16_bits(q), eq[:, 0], mag)
    ek, _, _ = _exact_rotation(W.bf16_bits(k), k_pos.numpy(), d, W.ROPE_YARN, kw, 0, "bhtd")
    _assert_rotation_close(to_np_f64(kg), W.bf16_bits(k), ek, mag)


def test_apply_strided_view_and_v_untouched(K):
    # k and v interleaved in one buffer [B, T, 2, Hk, d]; only the k half is passed
    B, T, Hk, d = 2, 33, 2, 128
    gen = W.generator(9)
    kv = W.normal_bf16((B, T, 2, Hk, d), gen).cuda()
    before = kv.clone()
    pos = torch.arange(T, dtype=torch.int32).repeat(B, 1).cuda()
    p = K.rope_params(d, base=500000.0)
    cos, sin = K.rope_table_build(p, T)
    K.rope_apply_qk(None, None, kv[:, :, 0], pos, cos, sin, k_layout="bthd")
    torch.cuda.synchronize()
    assert torch.equal(kv[:, :, 1], before[:, :, 1])
    exact, _, _ = _exact_rotation(W.bf16_bits(before[:, :, 0]), pos.cpu().numpy(), d, W.ROPE_NONE,
                                  dict(base=500000.0), 0, "bthd")
    _assert_rotation_close(to_np_f64(kv[:, :, 0]), W.bf16_bits(before[:, :, 0]), exact, 1.0)


def test_bad_position_is_skipped_and_flagged(K):
    d = 64
    x = W.normal_bf16((1, 3, 2, d), W.generator(3)).cuda()
    before = x.clone()
    pos = torch.tensor([[0, 99, 1]], dtype=torch.int32).cuda()
    cos, sin = K.rope_table_build(K.rope_params(d, base=10000.0), 10)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    K.rope_apply_qk(x, pos, None, None, cos, sin, q_layout="bthd", dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) & K.STATUS_BAD_POSITION
    assert torch.equal(x[0, 1], before[0, 1])
    assert torch.equal(x[0, 0], before[0, 0])  # position 0 is the identity
    assert not torch.equal(x[0, 2], before[0, 2])
