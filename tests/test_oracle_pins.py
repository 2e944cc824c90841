"""Pins for the fp64 CPU oracle: values printed on the pages, closed forms,
invariants the pages state, and brute force on tiny inputs.  None of these
re-types the oracle's own formulas; each is chosen so that a plausible slip in
the oracle (a dropped term, a wrong sign or index, a transposed operand, an
off-by-one mask) fails at least one of them.  CPU only.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle
from mqa_kv_cache_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _bf16_bits(shape, seed):
    g = W.generator(seed)
    return W.bf16_bits(W.normal_bf16(shape, g))


# --------------------------------------------------------------------------
# KV-cache accounting: printed values ("注意力变体与 MoE"; "注意力机制进化史";
# "Agentic RL 入门3" §2.3.5).
# --------------------------------------------------------------------------

def _golden_rows(tag):
    rows = []
    with open(os.path.join(GOLDEN, "kv_cache_bytes.txt")) as f:
        for line in f:
            parts = line.split()
            if parts and parts[0] == tag:
                rows.append(parts[1:])
    assert rows, tag
    return rows


def test_kv_bytes_printed_llama2_70b_shape():
    for L, kv, hd, by, kib, gib in _golden_rows("kv"):
        b = oracle.kv_cache_bytes_per_token(int(L), int(kv), int(hd), int(by))
        assert b / 1024 == float(kib)
        assert f"{b * 32768 * 16 / 2 ** 30:.1f}" == gib


def test_kv_bytes_printed_mla_v3():
    (L, h, hd, dc, dr, by, mha_kib, mla_kib, ratio), = _golden_rows("mla")
    mha = oracle.kv_cache_bytes_per_token(int(L), int(h), int(hd), int(by))
    mla = oracle.latent_cache_bytes_per_token(int(L), int(dc), int(dr), int(by))
    assert f"{mha / 1024:.0f}" == mha_kib
    assert f"{mla / 1024:.1f}" == mla_kib
    assert f"{mha / mla:.1f}" == ratio


def test_kv_dims_table():
    for name, kv, hd, width in _golden_rows("dims"):
        assert oracle.kv_cache_bytes_per_token(1, int(kv), int(hd), 1) == int(width), name
    (name, dc, dr, width), = _golden_rows("dims_latent")
    assert oracle.latent_cache_bytes_per_token(1, int(dc), int(dr), 1) == int(width)


def test_kv_bytes_printed_llama2_7b():
    (L, h, hd, by, per_tok, n, total), = _golden_rows("p5")
    b = oracle.kv_cache_bytes_per_token(int(L), int(h), int(hd), int(by))
    assert b == int(per_tok)
    assert b * int(n) == int(total)


# --------------------------------------------------------------------------
# RoPE frequencies ("Agentic RL 入门3" §1.1, §1.2 ①-④)
# --------------------------------------------------------------------------

ALL_MODES = [
    (oracle.NONE, {}),
    (oracle.PI, dict(s=4.0)),
    (oracle.NTK, dict(s=4.0)),
    (oracle.YARN, dict(s=4.0, L_train=8192.0)),
    (oracle.DYN_NTK, dict(L_train=4096.0, L_cur=10000.0)),
]


def test_theta_closed_forms():
    th, pos_div, mag = oracle.rope_freqs(128, 10000.0)
    assert th[0] == 1.0  # i starts at 0: theta_0 = base^0
    # 10000^(-1/64), evaluated to 40 digits with decimal arithmetic
    assert th[1] == pytest.approx(0.8659643233600653523531691834, rel=1e-15)
    assert th[-1] == pytest.approx(10000.0 ** (-126 / 128), rel=1e-14)
    assert pos_div == 1.0 and mag == 1.0
    assert np.all(np.diff(th) < 0)


def test_ntk_base_identity():
    # b' = b s^(d/(d-2)) is the base that maps the slowest pair exactly onto
    # the PI frequency theta/s while leaving theta_0 = 1: (b')^(-(d-2)/d) =
    # b^(-(d-2)/d) / s.  A wrong exponent breaks this identity.
    for d, base, s in [(128, 10000.0, 4.0), (64, 500000.0, 8.0), (128, 1e6, 2.0)]:
        plain, _, _ = oracle.rope_freqs(d, base)
        ntk, pos_div, mag = oracle.rope_freqs(d, base, oracle.NTK, s=s)
        assert ntk[0] == 1.0
        assert ntk[-1] == pytest.approx(plain[-1] / s, rel=1e-13)
        assert pos_div == 1.0 and mag == 1.0
        assert np.all(ntk <= plain)
    # d = 128, base 10000, s = 4: b' = 40889.94243... (40-digit decimal evaluation)
    ntk, _, _ = oracle.rope_freqs(128, 10000.0, oracle.NTK, s=4.0)
    assert ntk[1] == pytest.approx(40889.94243248621641308 ** (-2 / 128), rel=1e-14)


def test_pi_divides_positions_only():
    th_pi, pos_div, mag = oracle.rope_freqs(64, 10000.0, oracle.PI, s=4.0)
    th, _, _ = oracle.rope_freqs(64, 10000.0)
    np.testing.assert_array_equal(th_pi, th)
    assert pos_div == 4.0 and mag == 1.0
    c_pi, s_pi = oracle.rope_table(64, 10000.0, 41, oracle.PI, s=4.0)
    c, s = oracle.rope_table(64, 10000.0, 11)
    # PI row 4j is the plain row j (m/s = j exactly)
    np.testing.assert_allclose(c_pi[::4], c, rtol=0, atol=1e-15)
    np.testing.assert_allclose(s_pi[::4], s, rtol=0, atol=1e-15)


def test_yarn_ramp_band_edges_cfg3_shape():
    # d = 128, base 10000, L_train = 8192, alpha = 1, beta = 32:
    # r_i = 8192 * 10000^(-2i/128) / (2 pi); r_25 = 35.703 > 32, r_26 = 30.918,
    # r_49 = 1.1290, r_50 = 0.97771 <= 1 (40-digit decimal evaluation).
    g = oracle.yarn_gamma(128, 10000.0, 8192.0, 1.0, 32.0)
    assert np.all(g[:26] == 1.0)
    assert np.all(g[50:] == 0.0)
    assert g[26] == pytest.approx(0.96509374840355728580638, rel=1e-12)
    assert g[49] == pytest.approx(0.00416264326876862976372, rel=1e-10)
    assert np.all(np.diff(g) <= 0)


def test_yarn_frequencies_and_temperature():
    d, base, s, Lt = 128, 10000.0, 4.0, 8192.0
    th, _, _ = oracle.rope_freqs(d, base)
    ty, pos_div, mag = oracle.rope_freqs(d, base, oracle.YARN, s=s, L_train=Lt)
    g = oracle.yarn_gamma(d, base, Lt)
    # gamma = 1: unchanged; gamma = 0: exactly PI's theta/s; in between: between the two
    np.testing.assert_array_equal(ty[g == 1.0], th[g == 1.0])
    np.testing.assert_allclose(ty[g == 0.0], th[g == 0.0] / s, rtol=1e-15)
    mid = (g > 0) & (g < 1)
    assert np.all((ty[mid] < th[mid]) & (ty[mid] > th[mid] / s))
    assert pos_div == 1.0
    # sqrt(1/t) = 0.1 ln s + 1 at s = 4 (40-digit decimal evaluation)
    assert mag == pytest.approx(1.138629436111989061883446424, rel=1e-15)
    c, sn = oracle.rope_table(d, base, 3, oracle.YARN, s=s, L_train=Lt)
    np.testing.assert_allclose(c[0], mag, rtol=1e-15)  # cos(0) * mag
    np.testing.assert_array_equal(sn[0], 0.0)


def test_yarn_frequency_values_in_the_ramp():
    # theta^Y_i for d = 128, base 10000, s = 4, L_train = 8192, alpha 1, beta 32,
    # at two pairs inside the ramp (40-digit decimal evaluation of the page's
    # definitions): i = 26 (gamma 0.96509...) and i = 40 (gamma 0.10074...).
    ty, _, _ = oracle.rope_freqs(128, 10000.0, oracle.YARN, s=4.0, L_train=8192.0)
    assert ty[26] == pytest.approx(0.02309291880262394439893578, rel=1e-13)
    assert ty[40] == pytest.approx(0.001029497526604667895278467, rel=1e-13)


def test_dynamic_ntk_reduces_to_plain_below_training_length():
    th, _, _ = oracle.rope_freqs(128, 10000.0)
    dyn, _, _ = oracle.rope_freqs(128, 10000.0, oracle.DYN_NTK, L_train=4096.0, L_cur=1000.0)
    np.testing.assert_array_equal(dyn, th)
    dyn2, _, _ = oracle.rope_freqs(128, 10000.0, oracle.DYN_NTK, L_train=4096.0, L_cur=16384.0)
    ntk, _, _ = oracle.rope_freqs(128, 10000.0, oracle.NTK, s=4.0)
    np.testing.assert_array_equal(dyn2, ntk)


@pytest.mark.parametrize("mode", [oracle.PI, oracle.NTK, oracle.YARN])
def test_scalings_at_s1_are_plain(mode):
    kw = dict(s=1.0, L_train=4096.0)
    c0, s0 = oracle.rope_table(64, 10000.0, 300)
    c1, s1 = oracle.rope_table(64, 10000.0, 300, mode, **kw)
    np.testing.assert_allclose(c1, c0, rtol=0, atol=1e-13)
    np.testing.assert_allclose(s1, s0, rtol=0, atol=1e-13)


# --------------------------------------------------------------------------
# RoPE rotation ("Agentic RL 入门3" §1.1)
# --------------------------------------------------------------------------

def _rot(x, m, d, pair_style=0, mode=oracle.NONE, **kw):
    """Rotate fp64 vectors x [n, d] at position m with the oracle."""
    c, s = oracle.rope_table(d, 10000.0, m + 1, mode, **kw)
    xx = np.ascontiguousarray(np.asarray(x, np.float64).reshape(1, 1, -1, d))
    pos = np.array([[m]], np.int32)
    return oracle.rope_apply(xx, pos, c, s, pair_style=pair_style)[0, 0]


def test_rotation_direction_and_identity_at_zero():
    d = 8
    e0 = np.zeros((1, d))
    e0[0, 0] = 1.0
    # theta_0 = 1, m = 1: R(1,1) (1, 0)^T = (cos 1, sin 1)
    y = _rot(e0, 1, d)
    assert y[0, 0] == pytest.approx(0.5403023058681397174009366, abs=1e-15)
    assert y[0, 1] == pytest.approx(0.8414709848078965066525023, abs=1e-15)
    assert np.all(y[0, 2:] == 0.0)
    e1 = np.zeros((1, d))
    e1[0, 1] = 1.0
    y = _rot(e1, 1, d)  # R (0, 1)^T = (-sin 1, cos 1)
    assert y[0, 0] == pytest.approx(-0.8414709848078965066525023, abs=1e-15)
    assert y[0, 1] == pytest.approx(0.5403023058681397174009366, abs=1e-15)
    x = np.random.default_rng(1).standard_normal((3, d))
    np.testing.assert_array_equal(_rot(x, 0, d), x)


@pytest.mark.parametrize("mode,kw", ALL_MODES)
@pytest.mark.parametrize("pair_style", [0, 1])
def test_relative_position_property(mode, kw, pair_style):
    # R_m^T R_n = R_{n-m}: rot(q, m) . rot(k, n) depends only on n - m
    d = 64
    rng = np.random.default_rng(7)
    q = rng.standard_normal((1, d))
    k = rng.standard_normal((1, d))
    _, _, mag = oracle.rope_freqs(d, 10000.0, mode, **kw)
    for m, n in [(0, 5), (17, 3), (1000, 1234)]:
        ref = float(_rot(q, m, d, pair_style, mode, **kw)[0] @ _rot(k, n, d, pair_style, mode, **kw)[0])
        for c in (1, 1000, 30000):
            got = float(_rot(q, m + c, d, pair_style, mode, **kw)[0] @
                        _rot(k, n + c, d, pair_style, mode, **kw)[0])
            assert got == pytest.approx(ref, rel=1e-9, abs=1e-9)
        # and at m = n it is the plain dot product times mag^2 (= 1/t under YaRN)
    same = float(_rot(q, 321, d, pair_style, mode, **kw)[0] @ _rot(k, 321, d, pair_style, mode, **kw)[0])
    assert same == pytest.approx(mag * mag * float(q[0] @ k[0]), rel=1e-12)


@pytest.mark.parametrize("mode,kw", ALL_MODES)
def test_rotation_preserves_norm_times_mag(mode, kw):
    d = 128
    x = np.random.default_rng(3).standard_normal((5, d))
    _, _, mag = oracle.rope_freqs(d, 10000.0, mode, **kw)
    y = _rot(x, 4321, d, 0, mode, **kw)
    np.testing.assert_allclose(np.linalg.norm(y, axis=1), mag * np.linalg.norm(x, axis=1), rtol=1e-13)


def test_pair_styles_are_a_permutation_of_each_other():
    d = 16
    x = np.random.default_rng(5).standard_normal((2, d))
    perm = np.empty(d, int)  # adjacent slot (2i, 2i+1) <- half-split slot (i, i + d/2)
    perm[0::2] = np.arange(d // 2)
    perm[1::2] = np.arange(d // 2) + d // 2
    y_half = _rot(x, 77, d, pair_style=1)
    y_adj = _rot(x[:, perm], 77, d, pair_style=0)
    np.testing.assert_allclose(y_adj, y_half[:, perm], rtol=0, atol=1e-15)


def test_rope_apply_layouts_and_bf16_widening():
    d, B, T, H = 32, 2, 5, 3
    bits = _bf16_bits((B, T, H, d), 11)
    pos = np.array([[0, 1, 2, 3, 4], [9, 8, 7, 6, 5]], np.int32)
    c, s = oracle.rope_table(d, 500000.0, 10)
    y1 = oracle.rope_apply(bits, pos, c, s)
    y2 = oracle.rope_apply(oracle.bf16_bits_to_f64(bits), pos, c, s)
    np.testing.assert_array_equal(y1, y2)
    y3 = oracle.rope_apply(np.ascontiguousarray(bits.transpose(0, 2, 1, 3)), pos, c, s, layout="bhtd")
    np.testing.assert_array_equal(y3, y1.transpose(0, 2, 1, 3))
    # position 0 rows are untouched
    np.testing.assert_array_equal(y1[0, 0], oracle.bf16_bits_to_f64(bits[0, 0]))


# --------------------------------------------------------------------------
# Attention ("注意力变体与 MoE" attention(); "attention" GroupQueryAttention)
# --------------------------------------------------------------------------

def _f64(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def test_single_key_returns_its_value():
    q, k, v = _f64((1, 2, 16), 1), _f64((1, 1, 4, 16), 2), _f64((1, 1, 4, 16), 3)
    out, lse = oracle.attn_decode(q, k, v, np.array([1], np.int32), 0.25)
    np.testing.assert_array_equal(out[0, 0], v[0, 0, 0])
    assert lse[0, 0] == pytest.approx(0.25 * float(q[0, 0] @ k[0, 0, 0]), rel=1e-15)


def test_zero_query_gives_uniform_weights():
    q = np.zeros((1, 1, 8))
    k, v = _f64((1, 1, 10, 8), 2), _f64((1, 1, 10, 8), 3)
    out, lse = oracle.attn_decode(q, k, v, np.array([7], np.int32), 1.0)
    np.testing.assert_allclose(out[0, 0], v[0, 0, :7].mean(0), rtol=1e-14)
    assert lse[0, 0] == pytest.approx(math.log(7.0), rel=1e-15)


def test_two_keys_weights_quarter_three_quarters():
    # scores (0, ln 3) -> softmax (1/4, 3/4): pins the exponential base and the scale
    q = np.zeros((1, 1, 4))
    q[0, 0, 0] = 1.0
    k = np.zeros((1, 1, 2, 4))
    k[0, 0, 1, 0] = 2.0
    v = _f64((1, 1, 2, 4), 9)
    scale = math.log(3.0) / 2.0
    out, lse = oracle.attn_decode(q, k, v, np.array([2], np.int32), scale)
    np.testing.assert_allclose(out[0, 0], 0.25 * v[0, 0, 0] + 0.75 * v[0, 0, 1], rtol=1e-14)
    assert lse[0, 0] == pytest.approx(math.log(4.0), rel=1e-14)


def test_softmax_weights_sum_to_one():
    # with every value row equal to ones, the output is the sum of the weights
    q, k = _f64((2, 4, 16), 4), _f64((2, 2, 50, 16), 5)
    v = np.ones((2, 2, 50, 16))
    out, _ = oracle.attn_decode(q, k, v, np.array([50, 13], np.int32), 0.7)
    np.testing.assert_allclose(out, 1.0, rtol=0, atol=1e-14)


def test_gqa_equals_mha_on_repeat_interleaved_kv():
    B, H, Hk, T, d = 2, 8, 2, 33, 16
    q, k, v = _bf16_bits((B, H, d), 1), _bf16_bits((B, Hk, T, d), 2), _bf16_bits((B, Hk, T, d), 3)
    lens = np.array([33, 20], np.int32)
    g = H // Hk
    out_g, lse_g = oracle.attn_decode(q, k, v, lens, 0.25)
    out_m, lse_m = oracle.attn_decode(q, np.repeat(k, g, axis=1), np.repeat(v, g, axis=1), lens, 0.25)
    np.testing.assert_array_equal(out_g, out_m)
    np.testing.assert_array_equal(lse_g, lse_m)
    # and a head-interleaved mapping (h % Hk) would differ
    k_wrong = np.tile(k, (1, g, 1, 1))
    out_w, _ = oracle.attn_decode(q, k_wrong, np.tile(v, (1, g, 1, 1)), lens, 0.25)
    assert not np.allclose(out_w, out_g)


def test_mha_is_independent_per_head():
    B, H, T, d = 1, 4, 21, 8
    q, k, v = _bf16_bits((B, H, d), 1), _bf16_bits((B, H, T, d), 2), _bf16_bits((B, H, T, d), 3)
    lens = np.array([21], np.int32)
    out, lse = oracle.attn_decode(q, k, v, lens, 0.3)
    for h in range(H):
        o1, l1 = oracle.attn_decode(q[:, h:h + 1], k[:, h:h + 1], v[:, h:h + 1], lens, 0.3)
        np.testing.assert_array_equal(o1[0, 0], out[0, h])
        assert l1[0, 0] == lse[0, h]


def test_rows_past_length_are_ignored_and_empty_cache():
    q, k, v = _f64((1, 2, 8), 1), _f64((1, 1, 12, 8), 2), _f64((1, 1, 12, 8), 3)
    lens = np.array([5], np.int32)
    o1, l1 = oracle.attn_decode(q, k, v, lens, 0.5)
    k2, v2 = k.copy(), v.copy()
    k2[:, :, 5:] = 1e6
    v2[:, :, 5:] = np.nan
    o2, l2 = oracle.attn_decode(q, k2, v2, lens, 0.5)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)
    o3, l3 = oracle.attn_decode(q, k, v, np.array([0], np.int32), 0.5)
    assert np.all(o3 == 0.0) and np.all(np.isneginf(l3))


def test_split_keys_merge_identity():
    # softmax over a union of key sets = lse-weighted mix of the parts
    T, d = 40, 8
    q, k, v = _f64((1, 1, d), 1), _f64((1, 1, T, d), 2), _f64((1, 1, T, d), 3)
    full, full_lse = oracle.attn_decode(q, k, v, np.array([T], np.int32), 0.4)
    for n in (1, 2, 3, 7, 40):
        cuts = np.linspace(0, T, n + 1).astype(int)
        os_, ls_ = [], []
        for a, b in zip(cuts[:-1], cuts[1:]):
            o, l = oracle.attn_decode(q, np.ascontiguousarray(k[:, :, a:b]), np.ascontiguousarray(v[:, :, a:b]),
                                      np.array([b - a], np.int32), 0.4)
            os_.append(o[0, 0])
            ls_.append(l[0, 0])
        m, ml = oracle.softmax_merge(np.array(os_), np.array(ls_))
        np.testing.assert_allclose(m, full[0, 0], rtol=1e-13, atol=1e-15)
        assert ml == pytest.approx(full_lse[0, 0], rel=1e-14)
    # an empty part contributes nothing
    m, ml = oracle.softmax_merge(np.array([full[0, 0], np.zeros(d)]), np.array([full_lse[0, 0], -np.inf]))
    np.testing.assert_array_equal(m, full[0, 0])


def test_selected_heads_match_full_call():
    B, H, Hk, T, d = 2, 4, 1, 9, 8
    q, k, v = _bf16_bits((B, H, d), 1), _bf16_bits((B, Hk, T, d), 2), _bf16_bits((B, Hk, T, d), 3)
    lens = np.array([9, 4], np.int32)
    out, lse = oracle.attn_decode(q, k, v, lens, 0.3)
    sel = [(1, 3), (0, 0), (1, 1)]
    o, l = oracle.attn_decode(q, k, v, lens, 0.3, sel=sel)
    for i, (b, h) in enumerate(sel):
        np.testing.assert_array_equal(o[i], out[b, h])
        assert l[i] == lse[b, h]


def test_prefill_causal_row0_and_future_independence():
    B, T, H, Hk, d = 1, 12, 4, 2, 8
    q, k, v = _f64((B, T, H, d), 1), _f64((B, Hk, T, d), 2), _f64((B, Hk, T, d), 3)
    out, lse = oracle.attn_prefill(q, k, v, 0.35)
    # row 0 sees only key 0
    for h in range(H):
        np.testing.assert_array_equal(out[0, 0, h], v[0, h // 2, 0])
    # perturbing keys/values at j > i leaves row i unchanged
    i = 6
    k2, v2 = k.copy(), v.copy()
    k2[:, :, i + 1:] += 5.0
    v2[:, :, i + 1:] = np.nan
    out2, lse2 = oracle.attn_prefill(q, k2, v2, 0.35)
    np.testing.assert_array_equal(out2[:, :i + 1], out[:, :i + 1])
    np.testing.assert_array_equal(lse2[:, :, :i + 1], lse[:, :, :i + 1])
    # but perturbing key i itself does change row i (the diagonal is visible)
    k3 = k.copy()
    k3[:, :, i] += 5.0
    out3, _ = oracle.attn_prefill(q, k3, v, 0.35)
    assert not np.allclose(out3[:, i], out[:, i])


def test_prefill_row_equals_decode_over_prefix():
    B, T, H, Hk, d = 2, 10, 4, 2, 8
    q, k, v = _bf16_bits((B, T, H, d), 1), _bf16_bits((B, Hk, T, d), 2), _bf16_bits((B, Hk, T, d), 3)
    out, lse = oracle.attn_prefill(q, k, v, 0.3)
    for i in (0, 4, 9):
        o, l = oracle.attn_decode(np.ascontiguousarray(q[:, i]), k, v, np.array([i + 1] * B, np.int32), 0.3)
        np.testing.assert_array_equal(o, out[:, i])
        np.testing.assert_array_equal(l, lse[:, :, i])
    o, l = oracle.attn_prefill(q, k, v, 0.3, sel=[(1, 3, 7), (0, 0, 0)])
    np.testing.assert_array_equal(o[0], out[1, 7, 3])
    np.testing.assert_array_equal(o[1], out[0, 0, 0])


def _textbook_attention(q, k, v, scale, mask):
    """A second, independent statement of grouped-query attention in fp64 torch
    ("注意力变体与 MoE", attention(); "attention", GroupQueryAttention): K/V heads
    repeated g times along the head axis (query head h reads KV head h // g),
    scores = scale q k^T, masked entries -inf, softmax over keys, weights @ V.
    q [B, H, Tq, d]; k, v [B, Hk, Tk, d]; mask [B, Tq, Tk] True = hidden.
    A cross-check of the C oracle on tiny shapes, not a pin."""
    g = q.shape[1] // k.shape[1]
    kr = torch.repeat_interleave(k, g, dim=1)
    vr = torch.repeat_interleave(v, g, dim=1)
    s = torch.einsum("bhqd,bhkd->bhqk", q, kr) * scale
    s = s.masked_fill(mask[:, None], float("-inf"))
    lse = torch.logsumexp(s, dim=-1)
    return torch.einsum("bhqk,bhkd->bhqd", torch.softmax(s, dim=-1), vr), lse


def test_decode_matches_a_textbook_statement():
    B, H, Hk, T, d = 3, 8, 2, 40, 16
    q, k, v = _bf16_bits((B, H, d), 11), _bf16_bits((B, Hk, T, d), 12), _bf16_bits((B, Hk, T, d), 13)
    lens = np.array([40, 17, 1], np.int32)
    out, lse = oracle.attn_decode(q, k, v, lens, 0.25)
    f = lambda bits: torch.from_numpy(oracle.bf16_bits_to_f64(bits))
    mask = torch.arange(T)[None, None, :] >= torch.from_numpy(lens)[:, None, None]
    ro, rl = _textbook_attention(f(q)[:, :, None], f(k), f(v), 0.25, mask)
    np.testing.assert_allclose(out, ro[:, :, 0].numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, rl[:, :, 0].numpy(), rtol=0, atol=1e-12)


def test_prefill_matches_a_textbook_statement():
    B, T, H, Hk, d = 2, 24, 4, 1, 8
    q, k, v = _bf16_bits((B, T, H, d), 14), _bf16_bits((B, Hk, T, d), 15), _bf16_bits((B, Hk, T, d), 16)
    out, lse = oracle.attn_prefill(q, k, v, 0.3)
    f = lambda bits: torch.from_numpy(oracle.bf16_bits_to_f64(bits))
    causal = torch.triu(torch.ones(T, T, dtype=torch.bool), diagonal=1).expand(B, T, T)
    ro, rl = _textbook_attention(f(q).permute(0, 2, 1, 3), f(k), f(v), 0.3, causal)
    np.testing.assert_allclose(out, ro.permute(0, 2, 1, 3).numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, rl.numpy(), rtol=0, atol=1e-12)


# --------------------------------------------------------------------------
# Lightning indexer and top-k ("Agentic RL 入门3" §2.2 (1)(2); "attention" DSA ①)
# --------------------------------------------------------------------------

def _bits_of(x):
    return W.bf16_bits(torch.tensor(np.asarray(x, np.float32)).to(torch.bfloat16))


def test_indexer_closed_forms():
    HI, dI, L = 3, 4, 5
    q = np.zeros((1, HI, dI), np.float32)
    q[0, 0] = [1, 2, 0, 0]
    q[0, 1] = [0, 0, 1, -1]
    q[0, 2] = [1, 1, 1, 1]
    k = np.zeros((1, L, dI), np.float32)
    k[0, 0] = [1, 2, 0, 0]     # dots: 5, 0, 3
    k[0, 1] = [-1, -2, 0, 0]   # dots: -5, 0, -3 -> ReLU 0
    k[0, 2] = [0, 0, 2, -2]    # dots: 0, 4, 0
    k[0, 3] = [0, 0, -2, 2]    # dots: 0, -4, 0
    k[0, 4] = [1, 0, 0, 0]     # dots: 1, 0, 1
    w = np.array([[0.5, 2.0, 0.25]], np.float32)
    s = oracle.dsa_scores(_bits_of(q), w, _bits_of(k), np.array([L], np.int32))
    np.testing.assert_array_equal(s[0], [0.5 * 5 + 0.25 * 3, 0.0, 2.0 * 4, 0.0, 0.5 * 1 + 0.25 * 1])
    s = oracle.dsa_scores(_bits_of(q), w, _bits_of(k), np.array([3], np.int32))
    assert np.all(np.isneginf(s[0, 3:]))


def _topk_brute(scores, k):
    """rank(j) = #{i : s_i > s_j or (s_i == s_j and i < j)}; keep rank < k."""
    n = len(scores)
    ranks = [sum(1 for i in range(n) if scores[i] > scores[j] or (scores[i] == scores[j] and i < j))
             for j in range(n)]
    out = [-1] * k
    for j, r in enumerate(ranks):
        if r < k:
            out[r] = j
    return out


@pytest.mark.parametrize("seed", range(6))
def test_topk_brute_force_tiny(seed):
    rng = np.random.default_rng(seed)
    n = int(rng.integers(1, 64))
    k = int(rng.integers(1, 17))
    kind = seed % 3
    if kind == 0:
        s = rng.standard_normal(n)
    elif kind == 1:
        s = rng.integers(-3, 4, n).astype(np.float64)  # many ties
    else:
        s = rng.choice([0.0, -0.0, 1.0, -1.0], n)  # signed zeros tie
    got = oracle.topk(s[None], k)[0]
    assert list(got) == _topk_brute(list(s), k)


def test_topk_lengths_padding_and_nan():
    s = np.array([[3.0, 1.0, 2.0, 9.0, 9.0, 0.5]])
    assert list(oracle.topk(s, 4, lens=np.array([6], np.int32))[0]) == [3, 4, 0, 2]
    assert list(oracle.topk(s, 4, lens=np.array([2], np.int32))[0]) == [0, 1, -1, -1]
    with pytest.raises(ValueError):
        oracle.topk(np.array([[1.0, np.nan]]), 1)


def test_sparse_attention_all_rows_equals_mqa():
    B, Hq, Dk, Dv, L = 2, 4, 24, 16, 10
    q, C = _bf16_bits((B, Hq, Dk), 1), _bf16_bits((B, L, Dk), 2)
    idx = np.tile(np.arange(L, dtype=np.int32), (B, 1))
    out, lse = oracle.attn_sparse(q, C, idx, Dv, 0.2)
    # MQA over the latent rows with K = V = the full row, then keep the first Dv columns
    kv = np.ascontiguousarray(C[:, None])
    o_full, l_full = oracle.attn_decode(q, kv, kv, np.array([L] * B, np.int32), 0.2)
    np.testing.assert_array_equal(out, o_full[:, :, :Dv])
    np.testing.assert_array_equal(lse, l_full)


def test_sparse_attention_equals_masked_dense():
    # selecting rows S = dense attention with -inf on every row outside S
    B, Hq, Dk, Dv, L = 1, 3, 16, 8, 30
    q, C = _bf16_bits((B, Hq, Dk), 3), _bf16_bits((B, L, Dk), 4)
    sel = np.array([[25, 3, 17, 4, -1, 9, -1]], np.int32)
    out, lse = oracle.attn_sparse(q, C, sel, Dv, 0.5)
    rows = [r for r in sel[0] if r >= 0]
    kv = np.ascontiguousarray(C[:, rows][:, None])
    o_d, l_d = oracle.attn_decode(q, kv, kv, np.array([len(rows)], np.int32), 0.5)
    np.testing.assert_allclose(out, o_d[:, :, :Dv], rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(lse, l_d, rtol=1e-14)
    # order of the selected set does not matter
    perm = np.array([[9, -1, 4, 17, 25, -1, 3]], np.int32)
    out2, _ = oracle.attn_sparse(q, C, perm, Dv, 0.5)
    np.testing.assert_allclose(out2, out, rtol=1e-13, atol=1e-15)


# ---- sliding window with attention sinks ----------------------------------------

def test_window_positions_small_cases():
    assert oracle.window_positions(10, 2, 3) == [0, 1, 7, 8, 9]
    assert oracle.window_positions(3, 4, 2) == [0, 1, 2]      # everything fits
    assert oracle.window_positions(5, 0, 2) == [3, 4]         # no sinks
    assert oracle.window_positions(6, 2, 4) == [0, 1, 2, 3, 4, 5]  # sinks and window meet
    assert oracle.window_positions(7, 2, 4) == [0, 1, 3, 4, 5, 6]
    assert oracle.window_positions(0, 3, 5) == []


def _rand(shape, rng):
    return rng.standard_normal(shape)


def test_window_decode_against_masked_softmax():
    """The windowed decode equals softmax over all rows with -inf outside the row set,
    written out here in numpy (brute force, fp64)."""
    rng = np.random.default_rng(3)
    B, H, Hk, d, T = 3, 4, 2, 8, 40
    q, k, v = _rand((B, H, d), rng), _rand((B, Hk, T, d), rng), _rand((B, Hk, T, d), rng)
    lens = np.array([40, 9, 23], np.int32)
    s_, w_, scale = 3, 7, 0.3
    out, lse = oracle.attn_decode_window(q, k, v, lens, scale, s_, w_)
    for b in range(B):
        keep = np.zeros(T, bool)
        keep[:min(s_, lens[b])] = True
        keep[max(s_, lens[b] - w_):lens[b]] = True
        for h in range(H):
            sc = scale * k[b, h // (H // Hk)] @ q[b, h]
            sc[~keep] = -np.inf
            p = np.exp(sc - sc.max())
            np.testing.assert_allclose(out[b, h], (p / p.sum()) @ v[b, h // (H // Hk)], rtol=1e-12, atol=1e-12)
            np.testing.assert_allclose(lse[b, h], sc.max() + np.log(p.sum()), rtol=1e-12)


def test_window_decode_special_cases():
    rng = np.random.default_rng(4)
    B, H, Hk, d, T = 2, 2, 1, 16, 30
    q, k, v = _rand((B, H, d), rng), _rand((B, Hk, T, d), rng), _rand((B, Hk, T, d), rng)
    lens = np.array([30, 12], np.int32)
    full, full_l = oracle.attn_decode(q, k, v, lens, 0.25)
    # a window (plus sinks) covering every cached token is the plain decode
    for s_, w_ in ((0, 30), (5, 25), (2, 100)):
        o, l = oracle.attn_decode_window(q, k, v, lens, 0.25, s_, w_)
        np.testing.assert_array_equal(o, full)
        np.testing.assert_array_equal(l, full_l)
    # window 1, no sinks: the last cached token's value
    o, l = oracle.attn_decode_window(q, k, v, lens, 0.25, 0, 1)
    for b in range(B):
        np.testing.assert_allclose(o[b], np.repeat(v[b, :, lens[b] - 1], H, axis=0), rtol=1e-14)
        np.testing.assert_allclose(l[b], 0.25 * (q[b] @ k[b, 0, lens[b] - 1]), rtol=1e-12)
    # an empty cache attends to nothing
    o, l = oracle.attn_decode_window(q, k, v, np.array([0, 0], np.int32), 0.25, 2, 3)
    assert np.all(o == 0) and np.all(np.isneginf(l))


def test_prefill_window_special_cases():
    rng = np.random.default_rng(5)
    B, T, H, Hk, d = 1, 24, 2, 1, 8
    q, k, v = _rand((B, T, H, d), rng), _rand((B, Hk, T, d), rng), _rand((B, Hk, T, d), rng)
    sel = [(0, h, i) for h in range(H) for i in (0, 1, 7, 23)]
    full, full_l = oracle.attn_prefill(q, k, v, 0.5, sel=sel)
    # a window as long as the prompt is the plain causal prefill
    o, l = oracle.attn_prefill_window(q, k, v, 0.5, 0, T, sel)
    np.testing.assert_allclose(o, full, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(l, full_l, rtol=1e-12)
    # window 1, no sinks: every row sees only its own token
    o, l = oracle.attn_prefill_window(q, k, v, 0.5, 0, 1, sel)
    for n, (b, h, i) in enumerate(sel):
        np.testing.assert_allclose(o[n], v[b, 0, i], rtol=1e-14)
    # window 1 with 2 sinks: row 7 sees tokens 0, 1 and 7 only
    o, l = oracle.attn_prefill_window(q, k, v, 0.5, 2, 1, [(0, 0, 7)])
    sc = 0.5 * (k[0, 0, [0, 1, 7]] @ q[0, 7, 0])
    p = np.exp(sc - sc.max())
    np.testing.assert_allclose(o[0], (p / p.sum()) @ v[0, 0, [0, 1, 7]], rtol=1e-12)


# ---- block-level indexer ("attention" page, "Qwen Sparse Attention (QSA)") -----------

def _qsa_tables(d, n):
    theta, _, _ = oracle.rope_freqs(d, 10000.0)
    c, s = oracle.rope_table(d, 10000.0, n)
    return theta, c, s


def test_qsa_block_key_closed_form():
    """A group of four equal keys u gives RMS-normalised u rotated by the angle
    4j * theta_i at pair i: written with np.cos / np.sin from the frequencies, not
    from the table, so a wrong rotation position (4j + 3, or j) fails."""
    rng = np.random.default_rng(11)
    d, eps = 16, 1e-6
    theta, c, s = _qsa_tables(d, 64)
    u = rng.standard_normal((5, d))
    k = np.repeat(u, 4, axis=0)[None]                  # blocks 0..4, four equal rows each
    kb = oracle.qsa_block_keys(k, np.array([20]), c, s, eps)
    for j in range(5):
        n = u[j] / math.sqrt((u[j] ** 2).mean() + eps)
        ang = 4 * j * theta
        x, y = n[0::2], n[1::2]
        np.testing.assert_allclose(kb[0, j, 0::2], x * np.cos(ang) - y * np.sin(ang), rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(kb[0, j, 1::2], y * np.cos(ang) + x * np.sin(ang), rtol=1e-12, atol=1e-12)


def test_qsa_block_key_is_the_mean_not_the_sum():
    """Zero-sum offsets inside a group leave the block key unchanged, and with a
    large eps the normalised magnitude is sqrt(d) * rms / sqrt(rms^2 + eps) of the
    MEAN (a sum would carry rms 4x larger)."""
    rng = np.random.default_rng(12)
    d, eps = 8, 0.5
    _, c, s = _qsa_tables(d, 16)
    u = 0.1 * rng.standard_normal(d)
    delta = rng.standard_normal((4, d))
    delta -= delta.mean(axis=0)
    k1 = np.repeat(u[None], 4, axis=0)[None]
    k2 = (u[None] + delta)[None]
    a = oracle.qsa_block_keys(k1, np.array([4]), c, s, eps)
    b = oracle.qsa_block_keys(k2, np.array([4]), c, s, eps)
    np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-14)
    rms = math.sqrt((u ** 2).mean())
    np.testing.assert_allclose(np.linalg.norm(a[0, 0]), math.sqrt(d) * rms / math.sqrt(rms * rms + eps), rtol=1e-12)


def test_qsa_incomplete_group_makes_no_block():
    rng = np.random.default_rng(13)
    d = 8
    _, c, s = _qsa_tables(d, 32)
    k = rng.standard_normal((1, 12, d))
    kb = oracle.qsa_block_keys(k, np.array([10]), c, s, 1e-6)
    assert kb.shape == (1, 3, d)
    assert np.all(kb[0, 2] == 0)                     # tokens 8, 9: no complete group
    k2 = k.copy()
    k2[0, 8:] = 1e3                                 # changing them changes no block key
    np.testing.assert_array_equal(oracle.qsa_block_keys(k2, np.array([10]), c, s, 1e-6), kb)


def test_qsa_scores_match_the_token_indexer_on_block_keys():
    """Block scores are the lightning-indexer scores with blocks for tokens: the
    numpy restatement agrees with the C indexer on bf16 block keys."""
    gen = W.generator(14)
    B, HI, dI, NB = 2, 4, 16, 30
    q = W.bf16_bits(W.normal_bf16((B, HI, dI), gen))
    kb = W.bf16_bits(W.normal_bf16((B, NB, dI), gen))
    w = np.random.default_rng(14).uniform(0, 1, (B, HI)).astype(np.float32)
    lens = np.array([4 * NB + 3, 4 * 7 + 1], np.int32)
    sc = oracle.qsa_scores(q, w, kb, lens)
    ref = oracle.dsa_scores(q, w, kb, np.array([NB, 7], np.int32))
    np.testing.assert_allclose(sc, ref, rtol=1e-13, atol=0)
    assert np.all(np.isneginf(sc[1, 7:]))


def test_qsa_relu_drops_negative_heads():
    q = np.array([[[1.0, 0.0], [0.0, 1.0]]])         # two indexer heads
    kb = np.array([[[2.0, -3.0], [-1.0, -1.0]]])
    w = np.array([[0.5, 2.0]])
    sc = oracle.qsa_scores(q, w, kb, np.array([8]))
    np.testing.assert_array_equal(sc, [[1.0, 0.0]])


def test_qsa_expand_worked_example():
    """Ten tokens: blocks 0 (0-3) and 1 (4-7) complete, tokens 8, 9 the tail.
    With one block kept and block 1 the better, the set is 4..7 plus 8, 9."""
    q = np.array([[[1.0, 0.0]]])
    kb = np.array([[[0.1, 0.0], [0.9, 0.0]]])
    tok, cnt = oracle.qsa_select(q, np.array([[1.0]]), kb, np.array([10]), n_top=1)
    assert cnt[0] == 6
    assert list(tok[0]) == [4, 5, 6, 7, 8, 9, -1]


def test_qsa_budget_is_4k_plus_tail():
    """512 blocks of 4 give 2048 tokens, plus 0..3 trailing ones: 2048..2051."""
    rng = np.random.default_rng(15)
    for L in (4 * 600, 4 * 600 + 1, 4 * 600 + 3, 4 * 512, 4 * 100 + 2):
        sel = rng.permutation(L // 4)[:512]
        tok, cnt = oracle.qsa_expand(sel[None], np.array([L]), 512)
        nb = L // 4
        assert cnt[0] == 4 * min(nb, 512) + L % 4 <= 2051
        t = tok[0, :cnt[0]]
        assert np.all(np.diff(t) > 0) and t[-1] < L and np.all(tok[0, cnt[0]:] == -1)
        assert set(t[t >= 4 * nb]) == set(range(4 * nb, L))


def test_qsa_ties_go_to_the_lower_block():
    q = np.array([[[1.0]]])
    kb = np.array([[[1.0], [2.0], [2.0], [2.0], [0.5]]])
    tok, cnt = oracle.qsa_select(q, np.array([[1.0]]), kb, np.array([20]), n_top=2)
    assert list(tok[0, :cnt[0]]) == [4, 5, 6, 7, 8, 9, 10, 11]


def test_qsa_short_sequence_attends_to_everything():
    """With at most n_top complete groups every token is selected, so the sparse
    GQA decode is the plain decode."""
    rng = np.random.default_rng(16)
    B, H, Hk, d, T = 2, 4, 2, 8, 30
    q, k, v = rng.standard_normal((B, H, d)), rng.standard_normal((B, Hk, T, d)), rng.standard_normal((B, Hk, T, d))
    lens = np.array([30, 13], np.int32)
    qi = rng.standard_normal((B, 3, d))
    kb = rng.standard_normal((B, T // 4, d))
    tok, cnt = oracle.qsa_select(qi, rng.uniform(0, 1, (B, 3)), kb, lens, n_top=8)
    assert list(cnt) == [30, 13]
    o, l = oracle.attn_decode_gqa_sparse(q, k, v, tok, cnt, 0.3)
    ro, rl = oracle.attn_decode(q, k, v, lens, 0.3)
    np.testing.assert_allclose(o, ro, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(l, rl, rtol=1e-13)


def test_sparse_gqa_against_masked_softmax():
    """Over any token list the sparse decode is softmax with -inf outside the list
    (brute force in numpy); one listed token returns its value row."""
    rng = np.random.default_rng(17)
    B, H, Hk, d, T = 2, 6, 3, 8, 25
    q, k, v = rng.standard_normal((B, H, d)), rng.standard_normal((B, Hk, T, d)), rng.standard_normal((B, Hk, T, d))
    tok = np.full((B, 10), -1, np.int32)
    tok[0, :5] = [0, 3, 4, 17, 24]
    tok[1, :1] = [9]
    cnt = np.array([5, 1], np.int32)
    o, l = oracle.attn_decode_gqa_sparse(q, k, v, tok, cnt, 0.4)
    for b in range(B):
        keep = np.zeros(T, bool)
        keep[tok[b, :cnt[b]]] = True
        for h in range(H):
            sc = 0.4 * k[b, h // 2] @ q[b, h]
            sc[~keep] = -np.inf
            p = np.exp(sc - sc.max())
            np.testing.assert_allclose(o[b, h], (p / p.sum()) @ v[b, h // 2], rtol=1e-12, atol=1e-13)
            np.testing.assert_allclose(l[b, h], sc.max() + np.log(p.sum()), rtol=1e-12)
    np.testing.assert_allclose(o[1], v[1, np.arange(H) // 2, 9], rtol=1e-14)
    # -1 entries are unused slots: the same list with holes gives the same result
    tok2 = np.full((B, 12), -1, np.int32)
    tok2[0, :8] = [-1, 0, 3, -1, 4, 17, -1, 24]
    tok2[1, :3] = [-1, 9, -1]
    o2, l2 = oracle.attn_decode_gqa_sparse(q, k, v, tok2, np.array([8, 3], np.int32), 0.4)
    np.testing.assert_array_equal(o2, o)
    np.testing.assert_array_equal(l2, l)
