"""Pins of the oracle's FP8 (E4M3) cache quantiser, CPU only.

The pages fix the byte budget ("稀疏注意力：省了什么，没省什么", 改进一: 656 bytes per
token and layer for the FP8 latent + scales + bf16 RoPE part, about 132 for an
indexer key, 48,068 over 61 layers against V3's 70,272) but no rounding rule; the
oracle reads it as one fp32 scale per 128 values, s = absmax / 448, E4M3
round-to-nearest-even of x / s in fp32, saturating.  These tests pin that
quantiser to things other than itself:
  * the byte budget printed on the page (tests/golden/fp8_cache_bytes.txt);
  * the E4M3 format's closed forms (largest finite 448, smallest normal 2^-6,
    smallest subnormal 2^-9, 1.0 = 0x38) and its 254 finite values being
    exactly the values torch's float8_e4m3fn dtype represents;
  * round-to-nearest-even against torch's fp32 -> float8_e4m3fn conversion
    (a library routine) on random values, midpoints and the subnormal range;
  * exact round trip of inputs that are E4M3 values times a power of two;
  * the error bound: |dequant - x| <= (half an E4M3 spacing at x/s + the fp32
    division's rounding) * s;
  * the absmax element mapping to +-448, an all-zero group giving scale 0;
  * the FP8 indexer scores equal the indexer formula on the dequantised query
    heads and keys (the indexer's product runs on E4M3 operands), and with
    lossless operands equal the bf16 oracle's scores exactly.
"""
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "fp8_cache_bytes.txt")


def _rows(tag):
    out = []
    for line in open(GOLDEN):
        f = line.split()
        if f and f[0] == tag:
            out.append([float(x) for x in f[1:]])
    return out


def _bits(x):
    """float32 array that is bf16-representable -> bf16 bit patterns."""
    x = np.ascontiguousarray(x, np.float32)
    u = x.view(np.uint32)
    assert np.all((u & 0xFFFF) == 0), "not bf16-representable"
    return (u >> 16).astype(np.uint16)


def _to_bf16_bits(x):
    return torch.tensor(np.asarray(x, np.float32)).to(torch.bfloat16).view(torch.uint16).numpy()


def test_page_byte_budget():
    (row, key, layers, total, v3), = _rows("v32")
    (d_I, k, d_c, d_nope, d_rope), = _rows("dims")
    assert oracle.latent_fp8_row_bytes() == row == 656
    assert oracle.idx_key_fp8_bytes(int(d_I)) == key == 132
    assert layers * (oracle.latent_fp8_row_bytes() + oracle.idx_key_fp8_bytes(int(d_I))) == total
    # V3's bf16 latent: 576 two-byte values per layer, 61 layers
    assert oracle.latent_cache_bytes_per_token(int(layers), int(d_nope), int(d_rope), 2) == v3
    x = np.zeros((3, int(d_c)), np.uint16)
    assert oracle.latent_pack_fp8(x).shape == (3, 656)


def test_e4m3_closed_forms():
    v = oracle.e4m3_value(np.array([0x7E, 0x08, 0x07, 0x01, 0x38, 0x3C, 0x40, 0xB8, 0x00, 0x80], np.uint8))
    assert list(v[:8]) == [448.0, 2.0 ** -6, 7 * 2.0 ** -9, 2.0 ** -9, 1.0, 1.5, 2.0, -1.0]
    assert v[8] == 0.0 and v[9] == 0.0 and np.signbit(v[9])
    assert np.isnan(oracle.e4m3_value(np.array([0x7F, 0xFF], np.uint8))).all()


def test_e4m3_values_match_the_torch_dtype():
    codes = np.arange(256, dtype=np.uint8)
    ours = oracle.e4m3_value(codes)
    theirs = torch.tensor(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    fin = ~np.isnan(theirs)
    assert np.array_equal(np.isnan(ours), ~fin)
    assert np.array_equal(ours[fin], theirs[fin])
    assert fin.sum() == 254


def test_round_to_nearest_even_matches_torch_conversion():
    rng = np.random.default_rng(5)
    vals = oracle.e4m3_value(np.arange(0, 0x7F, dtype=np.uint8))  # 0 .. 448
    mids = (vals[:-1] + vals[1:]) / 2                             # every tie
    y = np.concatenate([
        rng.standard_normal(20000) * 50, rng.uniform(-464, 464, 20000),
        rng.uniform(-2 ** -5, 2 ** -5, 20000),                     # subnormal range
        mids, -mids, vals, -vals, np.nextafter(mids, 0), np.nextafter(mids, 1000)]).astype(np.float32)
    y = y[np.abs(y) < 464]  # torch's conversion does not saturate above the last midpoint
    ours = oracle.e4m3_round(y)
    theirs = torch.tensor(y).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, theirs)


def test_saturation_above_the_largest_value():
    y = np.array([464.0, 479.0, 480.0, 1e6, np.inf, -500.0, -np.inf], np.float32)
    c = oracle.e4m3_round(y)
    assert list(c) == [0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0xFE, 0xFE]


def test_lossless_round_trip_for_e4m3_values_times_a_power_of_two():
    rng = np.random.default_rng(7)
    codes = rng.integers(0, 0x7F, size=(40, 128)).astype(np.uint8)
    codes[:, 3] = 0x7E                                  # each group holds +-448: absmax = 448 * 2^e
    codes |= (rng.integers(0, 2, size=codes.shape) << 7).astype(np.uint8)
    e = rng.integers(-20, 10, size=(40, 1))
    x = oracle.e4m3_value(codes) * 2.0 ** e
    xb = _bits(x.astype(np.float32))
    c2, s2 = oracle.quant_fp8(xb)
    assert np.array_equal(s2[:, 0], (2.0 ** e[:, 0]).astype(np.float32))
    back = oracle.dequant_fp8(c2, s2)
    assert np.array_equal(back, x)


def test_error_bound_and_absmax_code():
    rng = np.random.default_rng(11)
    x = rng.standard_normal((64, 512)) * np.exp(rng.uniform(-8, 8, size=(64, 1)))
    xb = _to_bf16_bits(x)
    xf = oracle.bf16_bits_to_f64(xb)
    codes, scales = oracle.quant_fp8(xb)
    deq = oracle.dequant_fp8(codes, scales)
    s = np.repeat(scales.astype(np.float64), 128, axis=1)
    y = xf / s
    e = np.floor(np.log2(np.maximum(np.abs(y), 2.0 ** -6)))
    half_spacing = 2.0 ** (e - 3) / 2                    # 3 mantissa bits; subnormal spacing 2^-9
    bound = (half_spacing + np.abs(y) * 2.0 ** -24) * s
    assert np.all(np.abs(deq - xf) <= bound)
    # the largest magnitude of each group lands on +-448
    vals = np.abs(oracle.e4m3_value(codes)).reshape(64, 4, 128)
    assert np.all(vals.max(axis=-1) == 448.0)
    # scale = absmax / 448 in fp32
    amax = np.abs(xf).reshape(64, 4, 128).max(axis=-1).astype(np.float32)
    assert np.array_equal(scales, (amax / np.float32(448.0)).astype(np.float32))


def test_zero_group_and_layout():
    rng = np.random.default_rng(13)
    lat = _to_bf16_bits(rng.standard_normal((5, 576)))
    lat[2, 128:256] = 0                                   # one all-zero group
    packed = oracle.latent_pack_fp8(lat)
    codes, scales = oracle.quant_fp8(lat[:, :512])
    assert np.array_equal(packed[:, :512], codes)
    assert np.array_equal(packed[:, 512:528].copy().view(np.float32), scales)
    assert np.array_equal(packed[:, 528:].copy().view(np.uint16), lat[:, 512:])  # bf16 RoPE part as is
    assert scales[2, 1] == 0 and not packed[2, 128:256].any()
    un = oracle.latent_unpack_fp8(packed)
    assert np.array_equal(un[:, 512:], oracle.bf16_bits_to_f64(lat[:, 512:]))
    assert np.all(un[2, 128:256] == 0)
    assert np.array_equal(un[:, :512], oracle.dequant_fp8(codes, scales))


def test_fp8_indexer_scores_are_the_indexer_on_dequantised_operands():
    rng = np.random.default_rng(17)
    B, HI, dI, L = 2, 8, 128, 40
    q = _to_bf16_bits(rng.standard_normal((B, HI, dI)))
    w = rng.uniform(0, 1, (B, HI)).astype(np.float32)
    k = _to_bf16_bits(rng.standard_normal((B, L, dI)))
    lens = np.array([L, 23], np.int32)
    codes, ks = oracle.quant_fp8(k)
    got = oracle.dsa_scores_fp8(q, w, codes, ks[..., 0], lens)
    # the same formula in numpy, on the dequantised keys and the dequantised query heads
    kd = oracle.dequant_fp8(codes, ks)
    qc, qs = oracle.quant_fp8(q)
    qd = oracle.dequant_fp8(qc, qs)
    ref = np.einsum("bj,btj->bt", w.astype(np.float64), np.maximum(np.einsum("bjd,btd->btj", qd, kd), 0.0))
    for b in range(B):
        assert np.allclose(got[b, :lens[b]], ref[b, :lens[b]], rtol=1e-12, atol=1e-12)
        assert np.all(np.isneginf(got[b, lens[b]:]))
    # the query is quantised: with its bf16 values the scores differ
    ref_bf16_q = np.einsum("bj,btj->bt", w.astype(np.float64),
                           np.maximum(np.einsum("bjd,btd->btj", oracle.bf16_bits_to_f64(q), kd), 0.0))
    assert not np.allclose(got[0], ref_bf16_q[0], rtol=1e-6)
    # lossless operands (E4M3 values times a power of two): the bf16 oracle's scores exactly
    kc = rng.integers(0, 0x7F, size=(B, L, dI)).astype(np.uint8)
    kc[..., 0] = 0x7E
    kb = _bits((oracle.e4m3_value(kc) * 2.0 ** -4).astype(np.float32))
    qcl = rng.integers(0, 0xFF, size=(B, HI, dI)).astype(np.uint8) & 0xF7  # no NaN codes
    qcl[..., 5] = 0x7E
    qb = _bits((oracle.e4m3_value(qcl) * 2.0 ** 3).astype(np.float32))
    c2, s2 = oracle.quant_fp8(kb)
    assert np.array_equal(oracle.dsa_scores_fp8(qb, w, c2, s2[..., 0], lens), oracle.dsa_scores(qb, w, kb, lens))
