"""fp64 CPU oracle for RoPE + grouped-query KV-cache attention, the
lightning-indexer sparse path and the block-level (4-token group) indexer.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / reference leg of ``bench.py`` may import this package.
The CUDA product path never imports it, and it imports nothing from the
product package: the two are independent statements of the same method.

All arrays are numpy.  bf16 inputs are passed as ``np.uint16`` bit patterns
(widened exactly inside the C code); fp64 inputs as ``np.float64``.  Results
are fp64.  Each wrapper names the C function it calls; the C file cites the
passage of the pages each one restates.
"""
import ctypes

import numpy as np

from . import build as _build

NONE, PI, NTK, YARN, DYN_NTK = 0, 1, 2, 3, 4

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        i32, i64, dbl, vp = ctypes.c_int, ctypes.c_int64, ctypes.c_double, ctypes.c_void_p
        L.oracle_rope_freqs.argtypes = [i32, dbl, i32, dbl, dbl, dbl, dbl, dbl, vp, vp, vp]
        L.oracle_yarn_gamma.argtypes = [i32, dbl, dbl, dbl, dbl, vp]
        L.oracle_rope_table.argtypes = [i32, dbl, i32, dbl, dbl, dbl, dbl, dbl, i32, vp, vp]
        L.oracle_rope_apply.argtypes = [i32, vp, i32, i32, i32, i64, i64, i64, vp, vp, vp, i32, i32,
                                        i32, vp]
        L.oracle_attn_decode.argtypes = [i32, vp, vp, vp, vp, i32, i32, i32, i32, i32, dbl, i32, vp,
                                         vp, vp, i32]
        L.oracle_attn_prefill.argtypes = [i32, vp, vp, vp, i32, i32, i32, i32, i32, dbl, i32, vp,
                                          vp, vp, i32]
        L.oracle_softmax_merge.argtypes = [i32, i32, vp, vp, vp, vp]
        L.oracle_dsa_scores.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, vp, i32]
        L.oracle_topk.argtypes = [vp, i32, i32, vp]
        L.oracle_topk_rows.argtypes = [vp, vp, i32, i32, i32, vp, i32]
        L.oracle_attn_sparse.argtypes = [i32, vp, vp, vp, i32, i32, i32, i32, i32, i32, dbl, vp, vp,
                                         i32]
        L.oracle_kv_cache_bytes_per_token.argtypes = [i32, i32, i32, i32]
        L.oracle_kv_cache_bytes_per_token.restype = i64
        L.oracle_latent_cache_bytes_per_token.argtypes = [i32, i32, i32, i32]
        L.oracle_latent_cache_bytes_per_token.restype = i64
        L.oracle_max_threads.restype = i32
        L.oracle_e4m3_value.argtypes = [vp, i64, vp]
        L.oracle_e4m3_round.argtypes = [vp, i64, vp]
        L.oracle_quant_fp8_groups.argtypes = [vp, i64, i32, vp, vp]
        L.oracle_dequant_fp8_groups.argtypes = [vp, vp, i64, i32, vp]
        L.oracle_latent_pack_fp8.argtypes = [vp, i64, vp]
        L.oracle_latent_unpack_fp8.argtypes = [vp, i64, vp]
        L.oracle_latent_fp8_row_bytes.restype = i32
        L.oracle_idx_key_fp8_bytes.argtypes = [i32]
        L.oracle_idx_key_fp8_bytes.restype = i32
        L.oracle_dsa_scores_fp8.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, vp, i32]
        _lib = L
    return _lib


def max_threads() -> int:
    return lib().oracle_max_threads()


def _p(a):
    return a.ctypes.data_as(ctypes.c_void_p)


def _src(x):
    """(dtype flag, contiguous array) for a bf16-bits or fp64 input."""
    x = np.ascontiguousarray(x)
    if x.dtype == np.uint16:
        return 0, x
    if x.dtype == np.float64:
        return 1, x
    raise TypeError(f"oracle inputs are uint16 (bf16 bits) or float64, got {x.dtype}")


def _check(rc, fn):
    if rc != 0:
        raise ValueError(f"{fn} rejected its arguments (rc={rc})")


def rope_freqs(d, base, scaling=NONE, s=1.0, L_train=0.0, alpha=1.0, beta=32.0, L_cur=0.0):
    """-> (theta [d/2], position divisor, cos/sin magnitude).  oracle_rope_freqs."""
    theta = np.zeros(d // 2, np.float64)
    pos_div = np.zeros(1, np.float64)
    mag = np.zeros(1, np.float64)
    _check(lib().oracle_rope_freqs(d, base, scaling, s, L_train, alpha, beta, L_cur, _p(theta),
                                   _p(pos_div), _p(mag)), "oracle_rope_freqs")
    return theta, float(pos_div[0]), float(mag[0])


def yarn_gamma(d, base, L_train, alpha=1.0, beta=32.0):
    g = np.zeros(d // 2, np.float64)
    _check(lib().oracle_yarn_gamma(d, base, L_train, alpha, beta, _p(g)), "oracle_yarn_gamma")
    return g


def rope_table(d, base, max_pos, scaling=NONE, s=1.0, L_train=0.0, alpha=1.0, beta=32.0, L_cur=0.0):
    """-> (cos, sin), each [max_pos, d/2] fp64.  oracle_rope_table."""
    c = np.zeros((max_pos, d // 2), np.float64)
    sn = np.zeros((max_pos, d // 2), np.float64)
    _check(lib().oracle_rope_table(d, base, scaling, s, L_train, alpha, beta, L_cur, max_pos, _p(c),
                                   _p(sn)), "oracle_rope_table")
    return c, sn


def rope_apply(x, pos, cos, sin, pair_style=0, layout="bthd"):
    """Rotate head vectors.  x: [B, T, H, d] (layout 'bthd') or [B, H, T, d]
    (layout 'bhtd'); pos: [B, T] int32.  Returns fp64 in the same layout."""
    flag, x = _src(x)
    if layout == "bthd":
        B, T, H, d = x.shape
        sb, st, sh = T * H * d, H * d, d
    elif layout == "bhtd":
        B, H, T, d = x.shape
        sb, st, sh = H * T * d, d, T * d
    else:
        raise ValueError(layout)
    pos = np.ascontiguousarray(pos, dtype=np.int32).reshape(B, T)
    cos = np.ascontiguousarray(cos, np.float64)
    sin = np.ascontiguousarray(sin, np.float64)
    y = np.zeros((B, T, H, d), np.float64)
    _check(lib().oracle_rope_apply(flag, _p(x), B, T, H, sb, st, sh, _p(pos), _p(cos), _p(sin),
                                   cos.shape[0], d, pair_style, _p(y)), "oracle_rope_apply")
    return y if layout == "bthd" else np.ascontiguousarray(y.transpose(0, 2, 1, 3))


def attn_decode(q, k, v, seq_lens, scale, sel=None, nthreads=0):
    """q [B,H,d], k/v [B,Hk,T_max,d] -> (out, lse).  sel: optional [(b,h), ...]."""
    fq, q = _src(q)
    fk, k = _src(k)
    fv, v = _src(v)
    if not (fq == fk == fv):
        raise TypeError("q, k, v must share a dtype")
    B, H, d = q.shape
    _, Hk, T_max, _ = k.shape
    lens = np.ascontiguousarray(seq_lens, np.int32)
    if sel is None:
        out = np.zeros((B, H, d), np.float64)
        lse = np.zeros((B, H), np.float64)
        n_sel, selp = 0, None
    else:
        s = np.ascontiguousarray(np.asarray(sel, np.int32).reshape(-1, 2))
        n_sel, selp = s.shape[0], _p(s)
        out = np.zeros((n_sel, d), np.float64)
        lse = np.zeros(n_sel, np.float64)
    _check(lib().oracle_attn_decode(fq, _p(q), _p(k), _p(v), _p(lens), B, H, Hk, d, T_max, scale,
                                    n_sel, selp, _p(out), _p(lse), nthreads), "oracle_attn_decode")
    return out, lse


def window_positions(length, n_sink, window):
    """Token positions a query at position `length` attends to under a sliding
    window with attention sinks ("Agentic RL 入门3" §1: the last w keys, the first
    s tokens kept; the band i - w < j <= i of the "attention" page, with the query's
    own token not yet in the cache): tokens 0 .. n_sink-1 and the last `window`
    of the `length` cached tokens, each once, in increasing order."""
    sinks = list(range(min(n_sink, length)))
    return sinks + list(range(max(n_sink, length - window), length))


def attn_decode_window(q, k, v, seq_lens, scale, n_sink, window):
    """Decode over a linear cache (row t holds token t) restricted to the window
    and the sinks: the plain decode definition over the gathered rows of each
    sequence.  q [B,H,d], k/v [B,Hk,T,d] (bf16 bits or float64) -> (out, lse)."""
    B, H, d = np.shape(q)
    Hk = np.shape(k)[1]
    out = np.zeros((B, H, d), np.float64)
    lse = np.zeros((B, H), np.float64)
    for b in range(B):
        idx = window_positions(int(seq_lens[b]), n_sink, window)
        n = len(idx)
        kb = np.asarray(k)[b:b + 1][:, :, idx] if n else np.asarray(k)[b:b + 1][:, :, :1]
        vb = np.asarray(v)[b:b + 1][:, :, idx] if n else np.asarray(v)[b:b + 1][:, :, :1]
        o, l = attn_decode(np.asarray(q)[b:b + 1], np.ascontiguousarray(kb), np.ascontiguousarray(vb),
                           np.array([n], np.int32), scale)
        out[b], lse[b] = o[0], l[0]
    return out, lse


def attn_prefill_window(q, k, v, scale, n_sink, window, sel):
    """Causal prefill with a sliding window and sinks, row by row: row i of a prompt
    is the decode of q_i over the prefix 0 .. i (its own token included, so the
    band is i - window < j <= i) restricted to the sinks and the window.
    q [B,T,H,d], k/v [B,Hk,T,d]; sel = [(b, h, i), ...] -> (out [n, d], lse [n])."""
    q, k, v = np.asarray(q), np.asarray(k), np.asarray(v)
    d = q.shape[-1]
    out = np.zeros((len(sel), d), np.float64)
    lse = np.zeros(len(sel), np.float64)
    for n, (b, h, i) in enumerate(sel):
        o, l = attn_decode_window(q[b:b + 1, i], np.ascontiguousarray(k[b:b + 1, :, :i + 1]),
                                  np.ascontiguousarray(v[b:b + 1, :, :i + 1]), np.array([i + 1], np.int32), scale,
                                  n_sink, window)
        out[n], lse[n] = o[0, h], l[0, h]
    return out, lse


def attn_prefill(q, k, v, scale, sel=None, nthreads=0):
    """q [B,T,H,d], k/v [B,Hk,T,d] -> (out [B,T,H,d], lse [B,H,T]) or, with
    sel = [(b,h,i), ...], (out [n,d], lse [n])."""
    fq, q = _src(q)
    fk, k = _src(k)
    fv, v = _src(v)
    if not (fq == fk == fv):
        raise TypeError("q, k, v must share a dtype")
    B, T, H, d = q.shape
    Hk = k.shape[1]
    if sel is None:
        out = np.zeros((B, T, H, d), np.float64)
        lse = np.zeros((B, H, T), np.float64)
        n_sel, selp = 0, None
    else:
        s = np.ascontiguousarray(np.asarray(sel, np.int32).reshape(-1, 3))
        n_sel, selp = s.shape[0], _p(s)
        out = np.zeros((n_sel, d), np.float64)
        lse = np.zeros(n_sel, np.float64)
    _check(lib().oracle_attn_prefill(fq, _p(q), _p(k), _p(v), B, T, H, Hk, d, scale, n_sel, selp,
                                     _p(out), _p(lse), nthreads), "oracle_attn_prefill")
    return out, lse


def softmax_merge(o, lse):
    o = np.ascontiguousarray(o, np.float64)
    lse = np.ascontiguousarray(lse, np.float64)
    n, d = o.shape
    out = np.zeros(d, np.float64)
    ol = np.zeros(1, np.float64)
    _check(lib().oracle_softmax_merge(n, d, _p(o), _p(lse), _p(out), _p(ol)), "oracle_softmax_merge")
    return out, float(ol[0])


def dsa_scores(q_idx, w, k_idx, lens, nthreads=0):
    """q_idx [B,H_I,d_I] uint16, w [B,H_I] float32, k_idx [B,L_max,d_I] uint16
    -> scores [B, L_max] fp64 (-inf past each length)."""
    q_idx = np.ascontiguousarray(q_idx, np.uint16)
    k_idx = np.ascontiguousarray(k_idx, np.uint16)
    w = np.ascontiguousarray(w, np.float32)
    B, HI, dI = q_idx.shape
    L_max = k_idx.shape[1]
    lens = np.ascontiguousarray(lens, np.int32)
    sc = np.zeros((B, L_max), np.float64)
    _check(lib().oracle_dsa_scores(_p(q_idx), _p(w), _p(k_idx), _p(lens), B, HI, dI, L_max, _p(sc),
                                   nthreads), "oracle_dsa_scores")
    return sc


def topk(scores, k, lens=None, nthreads=0):
    """Row-wise top-k of scores [B, L_max] (fp32 or fp64, widened exactly):
    (score desc, index asc), -1 padded.  -> int32 [B, k]."""
    sc = np.ascontiguousarray(np.asarray(scores).astype(np.float64))
    if sc.ndim == 1:
        sc = sc[None]
    B, L_max = sc.shape
    lens = np.full(B, L_max, np.int32) if lens is None else np.ascontiguousarray(lens, np.int32)
    idx = np.zeros((B, k), np.int32)
    _check(lib().oracle_topk_rows(_p(sc), _p(lens), B, L_max, k, _p(idx), nthreads),
           "oracle_topk_rows")
    return idx


def attn_sparse(q, latent, idx, Dv, scale, nthreads=0):
    """q [B,Hq,Dk], latent [B,L_max,Dk], idx [B,k] int32 (-1 skipped)
    -> (out [B,Hq,Dv], lse [B,Hq])."""
    fq, q = _src(q)
    fc, latent = _src(latent)
    if fq != fc:
        raise TypeError("q and latent must share a dtype")
    B, Hq, Dk = q.shape
    L_max = latent.shape[1]
    idx = np.ascontiguousarray(idx, np.int32)
    k = idx.shape[1]
    out = np.zeros((B, Hq, Dv), np.float64)
    lse = np.zeros((B, Hq), np.float64)
    _check(lib().oracle_attn_sparse(fq, _p(q), _p(latent), _p(idx), B, Hq, Dk, Dv, L_max, k, scale,
                                    _p(out), _p(lse), nthreads), "oracle_attn_sparse")
    return out, lse


def kv_cache_bytes_per_token(n_layer, n_kv_head, d_head, bytes_per_elem=2):
    return int(lib().oracle_kv_cache_bytes_per_token(n_layer, n_kv_head, d_head, bytes_per_elem))


def latent_cache_bytes_per_token(n_layer, d_c, d_rope, bytes_per_elem=2):
    return int(lib().oracle_latent_cache_bytes_per_token(n_layer, d_c, d_rope, bytes_per_elem))


def bf16_bits_to_f64(bits):
    """Exact widening of bf16 bit patterns (uint16) to float64."""
    bits = np.ascontiguousarray(bits, np.uint16)
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)



# ---------------------------------------------------------------------------
# Block-level indexer ("attention" page, "Qwen Sparse Attention (QSA)" §3 ①–④)
#
# The visible prefix of a sequence of length L is cut into groups of 4 tokens;
# each complete group becomes one block key: the mean of its 4 indexer keys,
# normalised, then rotated at the position of the group's first token.  Blocks
# are scored like the lightning indexer (a weighted sum over indexer heads of
# ReLU(q . key)), the best n_top blocks are taken, every selected block is
# unpacked back into its 4 token positions and the 0..3 tokens of the trailing
# incomplete group are appended unconditionally; standard GQA attention then runs
# over those tokens of the full-precision cache.
#
# Readings where the section leaves a step open:
# * "normalise" = RMS normalisation without a learned gain,
#   x / sqrt(mean(x^2) + eps) (the pages name RMS-style normalisation as their
#   stabiliser elsewhere; no gain vector is given);
# * the rotation is the model's RoPE table over all d_I dimensions at position 4j
#   (the group's first token), with the same pair layout as every other rotation;
# * the head weights w_j of the lightning indexer are kept (w_j = 1 gives the
#   plain head sum of the section's sketch);
# * one selection per sequence serves every KV head (the indexer has no KV-head
#   axis);
# * ties between block scores go to the lower block index, as in the top-k.
# ---------------------------------------------------------------------------
QSA_BLOCK = 4


def qsa_block_keys(k_idx, lens, cos, sin, eps, pair_style=0):
    """k_idx [B, L_max, d_I] (bf16 bits or float64), lens [B] -> block keys
    [B, L_max // 4, d_I] fp64; rows j >= lens[b] // 4 are zero (no block)."""
    _, k = _src(k_idx)
    k = bf16_bits_to_f64(k) if k.dtype == np.uint16 else k
    B, L_max, d = k.shape
    nb_max = L_max // QSA_BLOCK
    out = np.zeros((B, nb_max, d), np.float64)
    for b in range(B):
        nb = int(lens[b]) // QSA_BLOCK
        if nb == 0:
            continue
        groups = k[b, :nb * QSA_BLOCK].reshape(nb, QSA_BLOCK, d)
        mean = groups.sum(axis=1) / QSA_BLOCK
        rms = np.sqrt((mean * mean).sum(axis=1) / d + eps)
        normed = mean / rms[:, None]
        pos = (np.arange(nb, dtype=np.int32) * QSA_BLOCK)[None]
        out[b, :nb] = rope_apply(normed[None, :, None, :], pos, cos, sin, pair_style)[0, :, 0, :]
    return out


def qsa_scores(q_idx, w, block_keys, lens):
    """Block scores s_j = sum_h w_h ReLU(q_h . key_j) over the complete blocks
    j < lens[b] // 4; -inf elsewhere.  q_idx [B, H_I, d_I], w [B, H_I],
    block_keys [B, NB, d_I] (bf16 bits or float64) -> [B, NB] fp64."""
    q = np.asarray(q_idx)
    q = bf16_bits_to_f64(q) if q.dtype == np.uint16 else q.astype(np.float64)
    kb = np.asarray(block_keys)
    kb = bf16_bits_to_f64(kb) if kb.dtype == np.uint16 else kb.astype(np.float64)
    w = np.asarray(w, np.float64)
    B, NB, _ = kb.shape
    sc = np.full((B, NB), -np.inf)
    for b in range(B):
        nb = min(int(lens[b]) // QSA_BLOCK, NB)
        dots = kb[b, :nb] @ q[b].T                      # [nb, H_I]
        sc[b, :nb] = np.maximum(dots, 0.0) @ w[b]
    return sc


def qsa_expand(block_sel, lens, n_top):
    """Selected blocks [B, n_top] (any order, -1 padded) -> (token positions
    [B, 4 * n_top + 3] int32 in increasing order, -1 padded; counts [B]): every
    selected block j gives 4j .. 4j+3, then the trailing tokens 4 * (L // 4) ..
    L - 1 of the incomplete group."""
    block_sel = np.asarray(block_sel, np.int64)
    B = block_sel.shape[0]
    width = QSA_BLOCK * n_top + QSA_BLOCK - 1
    tok = np.full((B, width), -1, np.int32)
    cnt = np.zeros(B, np.int32)
    for b in range(B):
        L = int(lens[b])
        blocks = sorted(int(j) for j in block_sel[b] if j >= 0)
        toks = [QSA_BLOCK * j + r for j in blocks for r in range(QSA_BLOCK)]
        toks += list(range(QSA_BLOCK * (L // QSA_BLOCK), L))
        tok[b, :len(toks)] = toks
        cnt[b] = len(toks)
    return tok, cnt


def qsa_select(q_idx, w, block_keys, lens, n_top, scores=None):
    """Score the complete blocks, keep the best n_top, expand with the tail.
    With `scores` given (the kernel's own fp32 block scores), the selection is
    taken on those, so that both sides decide in the same precision."""
    nb_max = np.shape(block_keys)[1]
    sc = qsa_scores(q_idx, w, block_keys, lens) if scores is None else np.asarray(scores, np.float64)
    nb = np.array([min(int(x) // QSA_BLOCK, nb_max) for x in lens], np.int32)
    sel = topk(sc, n_top, lens=nb)
    return qsa_expand(sel, lens, n_top)


def attn_decode_gqa_sparse(q, k, v, tok_idx, tok_count, scale):
    """GQA decode over the listed tokens of a linear cache: the plain decode
    definition over the gathered rows of each sequence (the first tok_count[b]
    entries of tok_idx[b]; an entry -1 marks an unused slot, as in the sparse
    latent decode, and is skipped).  q [B,H,d], k/v [B,Hk,T,d] -> (out, lse)."""
    B, H, d = np.shape(q)
    out = np.zeros((B, H, d), np.float64)
    lse = np.zeros((B, H), np.float64)
    k, v, q = np.asarray(k), np.asarray(v), np.asarray(q)
    for b in range(B):
        idx = [int(t) for t in tok_idx[b][:int(tok_count[b])] if t >= 0]
        n = len(idx)
        kb = k[b:b + 1][:, :, idx] if n else k[b:b + 1][:, :, :1]
        vb = v[b:b + 1][:, :, idx] if n else v[b:b + 1][:, :, :1]
        o, l = attn_decode(q[b:b + 1], np.ascontiguousarray(kb), np.ascontiguousarray(vb),
                           np.array([n], np.int32), scale)
        out[b], lse[b] = o[0], l[0]
    return out, lse


# ---------------------------------------------------------------------------
# FP8 (E4M3) latent cache and indexer keys ("稀疏注意力：省了什么，没省什么",
# 改进一: 656 bytes per token and layer = FP8 latent + scales + bf16 RoPE part,
# and an indexer key of about 132 bytes).  Reading: one fp32 scale per group of
# 128 values, s = absmax / 448, code = E4M3 round-to-nearest-even of x / s in
# fp32, saturating; the 64 RoPE values of a latent row stay bf16.  See oracle.c.
# ---------------------------------------------------------------------------
LATENT_FP8_ROW_BYTES = 656
FP8_GROUP = 128


def e4m3_value(codes):
    """E4M3 codes (uint8) -> their values (fp64; NaN for the NaN codes)."""
    c = np.ascontiguousarray(codes, np.uint8)
    out = np.zeros(c.shape, np.float64)
    _check(lib().oracle_e4m3_value(_p(c), c.size, _p(out)), "oracle_e4m3_value")
    return out


def e4m3_round(y):
    """fp32 values -> E4M3 codes (round to nearest even, saturating)."""
    y = np.ascontiguousarray(y, np.float32)
    out = np.zeros(y.shape, np.uint8)
    _check(lib().oracle_e4m3_round(_p(y), y.size, _p(out)), "oracle_e4m3_round")
    return out


def quant_fp8(x_bits, group=FP8_GROUP):
    """bf16 bits [..., n] (n a multiple of group) -> (codes uint8 [..., n],
    scales float32 [..., n // group])."""
    x = np.ascontiguousarray(x_bits, np.uint16)
    n = x.shape[-1]
    if n % group:
        raise ValueError("last dimension must be a multiple of the group")
    codes = np.zeros(x.shape, np.uint8)
    scales = np.zeros(x.shape[:-1] + (n // group,), np.float32)
    _check(lib().oracle_quant_fp8_groups(_p(x), x.size // group, group, _p(codes), _p(scales)),
           "oracle_quant_fp8_groups")
    return codes, scales


def dequant_fp8(codes, scales, group=FP8_GROUP):
    """(codes [..., n], scales [..., n // group]) -> values fp64 [..., n]."""
    c = np.ascontiguousarray(codes, np.uint8)
    sc = np.ascontiguousarray(scales, np.float32)
    out = np.zeros(c.shape, np.float64)
    _check(lib().oracle_dequant_fp8_groups(_p(c), _p(sc), c.size // group, group, _p(out)),
           "oracle_dequant_fp8_groups")
    return out


def latent_pack_fp8(latent_bits):
    """Latent rows [..., 576] (bf16 bits) -> packed FP8 rows [..., 656] uint8."""
    x = np.ascontiguousarray(latent_bits, np.uint16)
    if x.shape[-1] != 576:
        raise ValueError("latent rows are 576 wide")
    n = x.size // 576
    out = np.zeros(x.shape[:-1] + (LATENT_FP8_ROW_BYTES,), np.uint8)
    _check(lib().oracle_latent_pack_fp8(_p(x), n, _p(out)), "oracle_latent_pack_fp8")
    return out


def latent_unpack_fp8(packed):
    """Packed FP8 rows [..., 656] -> dequantised latent rows [..., 576] fp64."""
    p = np.ascontiguousarray(packed, np.uint8)
    if p.shape[-1] != LATENT_FP8_ROW_BYTES:
        raise ValueError("packed rows are 656 bytes")
    n = p.size // LATENT_FP8_ROW_BYTES
    out = np.zeros(p.shape[:-1] + (576,), np.float64)
    _check(lib().oracle_latent_unpack_fp8(_p(p), n, _p(out)), "oracle_latent_unpack_fp8")
    return out


def latent_fp8_row_bytes():
    return int(lib().oracle_latent_fp8_row_bytes())


def idx_key_fp8_bytes(d_I=128):
    return int(lib().oracle_idx_key_fp8_bytes(d_I))


def dsa_scores_fp8(q_idx, w, codes, kscale, lens, nthreads=0):
    """Indexer scores in fp8: the query heads q_idx [B,H_I,d_I] (bf16 bits) are quantised
    to E4M3 like the keys, and s = sum_j w_j ReLU(qhat_j . khat_t) on the dequantised
    operands.  w [B,H_I] float32, codes [B,L_max,d_I] uint8, kscale [B,L_max] float32
    -> scores [B, L_max] fp64."""
    q_idx = np.ascontiguousarray(q_idx, np.uint16)
    codes = np.ascontiguousarray(codes, np.uint8)
    kscale = np.ascontiguousarray(kscale, np.float32)
    w = np.ascontiguousarray(w, np.float32)
    B, HI, dI = q_idx.shape
    L_max = codes.shape[1]
    lens = np.ascontiguousarray(lens, np.int32)
    sc = np.zeros((B, L_max), np.float64)
    _check(lib().oracle_dsa_scores_fp8(_p(q_idx), _p(w), _p(codes), _p(kscale), _p(lens), B, HI, dI, L_max,
                                       _p(sc), nthreads), "oracle_dsa_scores_fp8")
    return sc
