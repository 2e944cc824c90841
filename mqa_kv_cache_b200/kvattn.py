"""Thin Python binding of libkvattn.so (the C ABI declared in include/kvattn.h).

Argument marshalling only: every step of the computation runs in the CUDA
library.  PyTorch provides device memory and the current stream; tensors must
be CUDA tensors of the documented dtype and layout.  There is no CPU
fallback: if the shared library is missing this module raises ImportError.
Function names match the C entry points.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libkvattn.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is not built; run `python -m mqa_kv_cache_b200.build`")

_lib = ctypes.CDLL(LIB_PATH)

_i32, _i64, _f32, _vp, _sz = ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_void_p, ctypes.c_size_t


class RopeParams(ctypes.Structure):
    _fields_ = [("head_dim", ctypes.c_int), ("scaling", ctypes.c_int), ("pair_style", ctypes.c_int),
                ("reserved", ctypes.c_int), ("base", ctypes.c_double), ("s", ctypes.c_double),
                ("L_train", ctypes.c_double), ("alpha", ctypes.c_double), ("beta", ctypes.c_double),
                ("L_cur", ctypes.c_double)]


_lib.kvattn_last_error_string.restype = ctypes.c_char_p
_lib.kvattn_version.restype = ctypes.c_char_p
_lib.rope_table_build.argtypes = [ctypes.POINTER(RopeParams), _i32, _vp, _vp, _vp]
_lib.rope_apply_qk.argtypes = [_vp, _i32, _i32, _i32, _i64, _i64, _i64, _vp,
                               _vp, _i32, _i32, _i32, _i64, _i64, _i64, _vp,
                               _vp, _vp, _i32, _i32, _i32, _vp, _vp]
_lib.attn_decode_gqa_workspace_bytes.argtypes = [_i32, _i32, _i32, _i32, _i32]
_lib.attn_decode_gqa_workspace_bytes.restype = _sz
_lib.attn_decode_gqa.argtypes = [_vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _f32, _vp, _vp, _vp, _sz,
                                 _vp, _vp]
_lib.attn_decode_gqa_rope.argtypes = [_vp, _vp, _vp, _vp, _i32, _i32, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32,
                                      _f32, _vp, _vp, _vp, _sz, _vp, _vp]
_lib.kv_append_rope.argtypes = [_vp, _vp, _vp, _i32, _i32, _i32, _vp, _vp, _i32, _vp, _vp, _i32, _i32, _vp, _vp]
_lib.kv_append_rope_ring.argtypes = [_vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _vp, _vp, _i32, _vp, _vp, _i32, _i32,
                                     _vp, _vp]
_lib.attn_decode_gqa_rope_window.argtypes = [_vp, _vp, _vp, _vp, _i32, _i32, _vp, _vp, _vp, _i32, _i32, _i32, _i32,
                                             _i32, _i32, _i32, _f32, _vp, _vp, _vp, _sz, _vp, _vp]
_lib.attn_decode_gqa_noalloc.argtypes = [_vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _f32, _vp, _vp, _vp,
                                         _vp]
_lib.attn_prefill_causal.argtypes = [_vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _f32, _vp, _vp, _vp]
_lib.attn_prefill_causal_window.argtypes = [_vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _i32, _i32, _f32, _vp, _vp,
                                            _vp]
_lib.dsa_index_topk_workspace_bytes.argtypes = [_i32, _i32, _i32]
_lib.dsa_index_topk_workspace_bytes.restype = _sz
_lib.dsa_index_topk.argtypes = [_vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _vp, _vp, _vp, _sz, _vp, _vp]
_lib.attn_decode_sparse_workspace_bytes.argtypes = [_i32, _i32, _i32, _i32]
_lib.attn_decode_sparse_workspace_bytes.restype = _sz
_lib.attn_decode_sparse.argtypes = [_vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _i32, _f32, _vp, _vp, _vp, _sz,
                                    _vp, _vp]
_lib.qsa_block_keys.argtypes = [_vp, _vp, _vp, _i32, _i32, _i32, _i32, _vp, _vp, _i32, _i32, _f32, _vp, _vp, _vp]
_lib.qsa_select_workspace_bytes.argtypes = [_i32, _i32, _i32]
_lib.qsa_select_workspace_bytes.restype = _sz
_lib.qsa_select.argtypes = [_vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _vp, _vp, _vp, _vp, _sz, _vp, _vp]
_lib.attn_decode_gqa_sparse_workspace_bytes.argtypes = [_i32, _i32, _i32, _i32, _i32]
_lib.attn_decode_gqa_sparse_workspace_bytes.restype = _sz
_lib.attn_decode_gqa_sparse.argtypes = [_vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _i32, _f32, _vp, _vp,
                                        _vp, _sz, _vp, _vp]
_lib.attn_merge_lse.argtypes = [_vp, _vp, _i32, _i32, _i32, _i32, _vp, _vp, _vp]
_lib.attn_decode_sparse_fp8.argtypes = [_vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _i32, _f32, _vp, _vp, _vp, _sz,
                                        _vp, _vp]
_lib.latent_quant_fp8.argtypes = [_vp, ctypes.c_longlong, _vp, _vp]
_lib.dsa_topk_candidates.argtypes = [_vp, _vp, _i32, _i32, _i32, _i32, _vp, _vp, _vp]
_lib.dsa_topk_merge.argtypes = [_vp, _vp, _i32, _i32, _i32, _vp, _vp, _vp]
_lib.dsa_index_topk_fp8.argtypes = [_vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _vp, _vp, _vp, _sz, _vp,
                                    _vp]
_lib.idx_key_quant_fp8.argtypes = [_vp, ctypes.c_longlong, _vp, _vp, _vp]
_lib.kvattn_test_decode_stall.argtypes = [_i32, ctypes.c_longlong]
_lib.attn_decode_gqa_noalloc_reset.argtypes = [_vp]

ROPE_NONE, ROPE_PI, ROPE_NTK, ROPE_YARN, ROPE_DYN_NTK = 0, 1, 2, 3, 4
STATUS_BAD_POSITION, STATUS_BAD_LENGTH, STATUS_BAD_INDEX, STATUS_NAN_SCORE, STATUS_TIMEOUT = 1, 2, 4, 8, 16


class KvattnError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"kvattn error {code}: {msg}")
        self.code = code


def kvattn_test_decode_stall(drop_tile: int = -1, wait_limit_ns: int = 0):
    """kvattn_test_decode_stall: failure-detection testing only (see the header).
    (-1, 0) restores normal operation."""
    _check(_lib.kvattn_test_decode_stall(int(drop_tile), int(wait_limit_ns)))


def attn_decode_gqa_noalloc_reset():
    """Zero the counter region of the allocation-free decode's static scratch
    (on the current stream); needed only after a call that timed out."""
    _check(_lib.attn_decode_gqa_noalloc_reset(_stream()))


def library():
    """The loaded ctypes.CDLL (for direct C-ABI calls)."""
    return _lib


def version() -> str:
    return _lib.kvattn_version().decode()


def _check(rc: int):
    if rc != 0:
        raise KvattnError(rc, _lib.kvattn_last_error_string().decode())


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _need(t, dtype, name):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")


def _contig(t, name):
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def rope_params(head_dim, base, scaling=ROPE_NONE, s=1.0, L_train=0.0, alpha=1.0, beta=32.0, L_cur=0.0,
                pair_style=0) -> RopeParams:
    return RopeParams(head_dim, scaling, pair_style, 0, base, s, L_train, alpha, beta, L_cur)


def rope_table_build(params: RopeParams, max_pos: int, device=None):
    """-> (cos, sin) fp32 [max_pos, head_dim/2] on `device` (default: current)."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    half = params.head_dim // 2
    cos = torch.empty((max_pos, half), dtype=torch.float32, device=dev)
    sin = torch.empty((max_pos, half), dtype=torch.float32, device=dev)
    _check(_lib.rope_table_build(ctypes.byref(params), max_pos, _ptr(cos), _ptr(sin), _stream()))
    return cos, sin


def _view(x, layout):
    """(nb, nt, nh, sb, st, sh) of a head-vector tensor for rope_apply_qk."""
    if x.stride(-1) != 1:
        raise ValueError("innermost dimension must be contiguous")
    if layout == "bhd":      # [B, H, d], one token per batch entry
        B, H, _ = x.shape
        return B, 1, H, x.stride(0), 0, x.stride(1)
    if layout == "bthd":     # [B, T, H, d]
        B, T, H, _ = x.shape
        return B, T, H, x.stride(0), x.stride(1), x.stride(2)
    if layout == "bhtd":     # [B, H, T, d] (the cache layout)
        B, H, T, _ = x.shape
        return B, T, H, x.stride(0), x.stride(2), x.stride(1)
    raise ValueError(layout)


def rope_apply_qk(q, q_pos, k, k_pos, cos, sin, q_layout="bthd", k_layout="bhtd", pair_style=0,
                  dev_status=None):
    """Rotate q and/or k in place.  Positions are int32 CUDA tensors with one
    entry per (batch, token): q_pos [B, T_q] (T_q = 1 for 'bhd'), k_pos [B, T]."""
    _need(cos, torch.float32, "cos")
    _need(sin, torch.float32, "sin")
    head_dim = 2 * cos.shape[1]
    qv = (0, 0, 0, 0, 0, 0)
    kv = (0, 0, 0, 0, 0, 0)
    if q is not None:
        _need(q, torch.bfloat16, "q")
        _need(q_pos, torch.int32, "q_pos")
        _contig(q_pos, "q_pos")
        qv = _view(q, q_layout)
        if q_pos.numel() != qv[0] * qv[1]:
            raise ValueError("q_pos must hold one position per (batch, token)")
    if k is not None:
        _need(k, torch.bfloat16, "k")
        _need(k_pos, torch.int32, "k_pos")
        _contig(k_pos, "k_pos")
        kv = _view(k, k_layout)
        if k_pos.numel() != kv[0] * kv[1]:
            raise ValueError("k_pos must hold one position per (batch, token)")
    _check(_lib.rope_apply_qk(_ptr(q), *qv, _ptr(q_pos) if q is not None else None,
                              _ptr(k), *kv, _ptr(k_pos) if k is not None else None,
                              _ptr(cos), _ptr(sin), cos.shape[0], head_dim, pair_style, _ptr(dev_status),
                              _stream()))


def attn_decode_gqa_workspace_bytes(B, n_head, n_kv_head, head_dim, T_max) -> int:
    return int(_lib.attn_decode_gqa_workspace_bytes(B, n_head, n_kv_head, head_dim, T_max))


def workspace(nbytes: int, device=None):
    """A zero-filled, 256-byte aligned uint8 CUDA buffer of at least `nbytes`
    bytes (the decode workspace wants its counter region zero before first use)."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    return torch.zeros(max(int(nbytes), 256), dtype=torch.uint8, device=dev)


def attn_decode_gqa(q, k_cache, v_cache, seq_lens, scale, out=None, lse=None, ws=None, dev_status=None,
                    want_lse=True):
    """q [B, H, d] bf16, k_cache/v_cache [B, Hk, T_max, d] bf16, seq_lens int32 [B]
    -> (out [B, H, d] bf16, lse [B, H] fp32 or None)."""
    for t, n in ((q, "q"), (k_cache, "k_cache"), (v_cache, "v_cache")):
        _need(t, torch.bfloat16, n)
        _contig(t, n)
    _need(seq_lens, torch.int32, "seq_lens")
    _contig(seq_lens, "seq_lens")
    B, H, d = q.shape
    Bk, Hk, T_max, dk = k_cache.shape
    if (Bk, dk) != (B, d) or v_cache.shape != k_cache.shape or seq_lens.numel() != B:
        raise ValueError("inconsistent decode shapes")
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((B, H), dtype=torch.float32, device=q.device)
    need = attn_decode_gqa_workspace_bytes(B, H, Hk, d, T_max)
    if ws is None:
        ws = workspace(need, q.device)
    _check(_lib.attn_decode_gqa(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(seq_lens), B, H, Hk, d, T_max,
                                float(scale), _ptr(out), _ptr(lse), _ptr(ws), ws.numel(), _ptr(dev_status),
                                _stream()))
    return out, lse


def attn_decode_gqa_rope(q, q_pos, cos, sin, k_cache, v_cache, seq_lens, scale, pair_style=0, out=None, lse=None,
                         ws=None, dev_status=None, want_lse=True):
    """attn_decode_gqa with the queries rotated inside the kernel: q [B, H, d] raw
    (not modified), q_pos int32 [B] (or [B, 1]) their positions, cos/sin the
    rope_table_build tables [max_pos, d/2]."""
    for t, n in ((q, "q"), (k_cache, "k_cache"), (v_cache, "v_cache")):
        _need(t, torch.bfloat16, n)
        _contig(t, n)
    for t, n in ((seq_lens, "seq_lens"), (q_pos, "q_pos")):
        _need(t, torch.int32, n)
        _contig(t, n)
    _need(cos, torch.float32, "cos")
    _need(sin, torch.float32, "sin")
    B, H, d = q.shape
    Bk, Hk, T_max, dk = k_cache.shape
    if (Bk, dk) != (B, d) or v_cache.shape != k_cache.shape or seq_lens.numel() != B or q_pos.numel() != B:
        raise ValueError("inconsistent decode shapes")
    if cos.shape[1] * 2 != d or sin.shape != cos.shape:
        raise ValueError("tables must be [max_pos, d/2]")
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((B, H), dtype=torch.float32, device=q.device)
    need = attn_decode_gqa_workspace_bytes(B, H, Hk, d, T_max)
    if ws is None:
        ws = workspace(need, q.device)
    _check(_lib.attn_decode_gqa_rope(_ptr(q), _ptr(q_pos), _ptr(cos), _ptr(sin), cos.shape[0], pair_style,
                                     _ptr(k_cache), _ptr(v_cache), _ptr(seq_lens), B, H, Hk, d, T_max, float(scale),
                                     _ptr(out), _ptr(lse), _ptr(ws), ws.numel(), _ptr(dev_status), _stream()))
    return out, lse


def kv_append_rope(k_new, v_new, pos, k_cache, v_cache, cos, sin, pair_style=0, dev_status=None):
    """Write RoPE(k_new) and v_new ([B, Hk, d]) into slot pos[b] (int32 [B]) of the
    [B, Hk, T_max, d] caches."""
    for t, n in ((k_new, "k_new"), (v_new, "v_new"), (k_cache, "k_cache"), (v_cache, "v_cache")):
        _need(t, torch.bfloat16, n)
        _contig(t, n)
    _need(pos, torch.int32, "pos")
    _contig(pos, "pos")
    _need(cos, torch.float32, "cos")
    _need(sin, torch.float32, "sin")
    B, Hk, d = k_new.shape
    Bc, Hc, T_max, dc = k_cache.shape
    if (Bc, Hc, dc) != (B, Hk, d) or v_cache.shape != k_cache.shape or v_new.shape != k_new.shape or pos.numel() != B:
        raise ValueError("inconsistent append shapes")
    _check(_lib.kv_append_rope(_ptr(k_new), _ptr(v_new), _ptr(pos), B, Hk, d, _ptr(k_cache), _ptr(v_cache), T_max,
                               _ptr(cos), _ptr(sin), cos.shape[0], pair_style, _ptr(dev_status), _stream()))


def kv_append_rope_ring(k_new, v_new, pos, k_cache, v_cache, cos, sin, n_sink, window, pair_style=0, dev_status=None):
    """kv_append_rope into a rolling cache of n_sink + window slots (slot of position
    p >= n_sink: n_sink + (p - n_sink) % window)."""
    for t, n in ((k_new, "k_new"), (v_new, "v_new"), (k_cache, "k_cache"), (v_cache, "v_cache")):
        _need(t, torch.bfloat16, n)
        _contig(t, n)
    _need(pos, torch.int32, "pos")
    _contig(pos, "pos")
    B, Hk, d = k_new.shape
    Bc, Hc, T_max, dc = k_cache.shape
    if (Bc, Hc, dc) != (B, Hk, d) or v_cache.shape != k_cache.shape or v_new.shape != k_new.shape or pos.numel() != B:
        raise ValueError("inconsistent append shapes")
    _check(_lib.kv_append_rope_ring(_ptr(k_new), _ptr(v_new), _ptr(pos), int(n_sink), int(window), B, Hk, d,
                                    _ptr(k_cache), _ptr(v_cache), T_max, _ptr(cos), _ptr(sin), cos.shape[0],
                                    pair_style, _ptr(dev_status), _stream()))


def attn_decode_gqa_rope_window(q, q_pos, cos, sin, k_cache, v_cache, seq_lens, scale, n_sink, window, pair_style=0,
                                out=None, lse=None, ws=None, dev_status=None, want_lse=True):
    """attn_decode_gqa_rope over a rolling cache: seq_lens = tokens so far; attention over the
    min(seq_lens, n_sink + window) filled slots (the sinks and the last `window` tokens)."""
    for t, n in ((q, "q"), (k_cache, "k_cache"), (v_cache, "v_cache")):
        _need(t, torch.bfloat16, n)
        _contig(t, n)
    for t, n in ((seq_lens, "seq_lens"), (q_pos, "q_pos")):
        _need(t, torch.int32, n)
        _contig(t, n)
    B, H, d = q.shape
    _, Hk, T_max, _ = k_cache.shape
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((B, H), dtype=torch.float32, device=q.device)
    if ws is None:
        ws = workspace(attn_decode_gqa_workspace_bytes(B, H, Hk, d, T_max), q.device)
    _check(_lib.attn_decode_gqa_rope_window(_ptr(q), _ptr(q_pos), _ptr(cos), _ptr(sin), cos.shape[0], pair_style,
                                            _ptr(k_cache), _ptr(v_cache), _ptr(seq_lens), int(n_sink), int(window), B,
                                            H, Hk, d, T_max, float(scale), _ptr(out), _ptr(lse), _ptr(ws), ws.numel(),
                                            _ptr(dev_status), _stream()))
    return out, lse


def attn_decode_gqa_noalloc(q, k_cache, v_cache, seq_lens, scale, out=None, lse=None, dev_status=None,
                            want_lse=True):
    """attn_decode_gqa without a workspace: the library's static device scratch
    is used (shared by every call on the device; see include/kvattn.h)."""
    for t, n in ((q, "q"), (k_cache, "k_cache"), (v_cache, "v_cache")):
        _need(t, torch.bfloat16, n)
        _contig(t, n)
    _need(seq_lens, torch.int32, "seq_lens")
    B, H, d = q.shape
    _, Hk, T_max, _ = k_cache.shape
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((B, H), dtype=torch.float32, device=q.device)
    _check(_lib.attn_decode_gqa_noalloc(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(seq_lens), B, H, Hk, d, T_max,
                                        float(scale), _ptr(out), _ptr(lse), _ptr(dev_status), _stream()))
    return out, lse


def attn_prefill_causal(q, k, v, scale, out=None, lse=None, want_lse=True):
    """q [B, T, H, d] bf16, k/v [B, Hk, T, d] bf16 -> (out [B, T, H, d] bf16, lse [B, H, T] fp32)."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, torch.bfloat16, n)
        _contig(t, n)
    B, T, H, d = q.shape
    Hk = k.shape[1]
    if k.shape != (B, Hk, T, d) or v.shape != k.shape:
        raise ValueError("inconsistent prefill shapes")
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((B, H, T), dtype=torch.float32, device=q.device)
    _check(_lib.attn_prefill_causal(_ptr(q), _ptr(k), _ptr(v), B, T, H, Hk, d, float(scale), _ptr(out), _ptr(lse),
                                    _stream()))
    return out, lse


def attn_prefill_causal_window(q, k, v, scale, n_sink, window, out=None, lse=None, want_lse=True):
    """attn_prefill_causal where row i sees keys j <= i with j > i - window or j < n_sink."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, torch.bfloat16, n)
        _contig(t, n)
    B, T, H, d = q.shape
    Hk = k.shape[1]
    if k.shape != (B, Hk, T, d) or v.shape != k.shape:
        raise ValueError("inconsistent prefill shapes")
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((B, H, T), dtype=torch.float32, device=q.device)
    _check(_lib.attn_prefill_causal_window(_ptr(q), _ptr(k), _ptr(v), B, T, H, Hk, d, int(n_sink), int(window),
                                           float(scale), _ptr(out), _ptr(lse), _stream()))
    return out, lse


def dsa_index_topk_workspace_bytes(B, L_max, k) -> int:
    return int(_lib.dsa_index_topk_workspace_bytes(B, L_max, k))


def dsa_index_topk(q_idx, w, k_idx, k, seq_lens=None, topk_idx=None, scores_out=None, ws=None, dev_status=None,
                   want_scores=True):
    """q_idx [B, H_I, d_I] bf16, w [B, H_I] fp32, k_idx [B, L_max, d_I] bf16
    -> (topk_idx int32 [B, k], scores fp32 [B, L_max] or None)."""
    _need(q_idx, torch.bfloat16, "q_idx")
    _need(k_idx, torch.bfloat16, "k_idx")
    _need(w, torch.float32, "w")
    for t, n in ((q_idx, "q_idx"), (k_idx, "k_idx"), (w, "w")):
        _contig(t, n)
    B, HI, dI = q_idx.shape
    L_max = k_idx.shape[1]
    if seq_lens is not None:
        _need(seq_lens, torch.int32, "seq_lens")
    if topk_idx is None:
        topk_idx = torch.empty((B, k), dtype=torch.int32, device=q_idx.device)
    if scores_out is None and want_scores:
        scores_out = torch.empty((B, L_max), dtype=torch.float32, device=q_idx.device)
    if ws is None:
        ws = workspace(dsa_index_topk_workspace_bytes(B, L_max, k), q_idx.device)
    _check(_lib.dsa_index_topk(_ptr(q_idx), _ptr(w), _ptr(k_idx), _ptr(seq_lens), B, HI, dI, L_max, k,
                               _ptr(topk_idx), _ptr(scores_out), _ptr(ws), ws.numel(), _ptr(dev_status),
                               _stream()))
    return topk_idx, scores_out


def dsa_index_topk_fp8(q_idx, w, k_codes, k_scales, k, seq_lens=None, topk_idx=None, scores_out=None, ws=None,
                       dev_status=None, want_scores=True):
    """q_idx [B, 64, 128] bf16, w [B, 64] fp32, k_codes [B, L_max, 128] uint8 and
    k_scales [B, L_max] fp32 (idx_key_quant_fp8) -> (topk_idx int32 [B, k],
    scores fp32 [B, L_max] or None)."""
    _need(q_idx, torch.bfloat16, "q_idx")
    _need(k_codes, torch.uint8, "k_codes")
    _need(k_scales, torch.float32, "k_scales")
    _need(w, torch.float32, "w")
    for t, n in ((q_idx, "q_idx"), (k_codes, "k_codes"), (k_scales, "k_scales"), (w, "w")):
        _contig(t, n)
    B, HI, dI = q_idx.shape
    L_max = k_codes.shape[1]
    if tuple(k_scales.shape) != (B, L_max):
        raise ValueError("k_scales must be [B, L_max]")
    if seq_lens is not None:
        _need(seq_lens, torch.int32, "seq_lens")
    if topk_idx is None:
        topk_idx = torch.empty((B, k), dtype=torch.int32, device=q_idx.device)
    if scores_out is None and want_scores:
        scores_out = torch.empty((B, L_max), dtype=torch.float32, device=q_idx.device)
    if ws is None:
        ws = workspace(dsa_index_topk_workspace_bytes(B, L_max, k), q_idx.device)
    _check(_lib.dsa_index_topk_fp8(_ptr(q_idx), _ptr(w), _ptr(k_codes), _ptr(k_scales), _ptr(seq_lens), B, HI, dI,
                                   L_max, k, _ptr(topk_idx), _ptr(scores_out), _ptr(ws), ws.numel(),
                                   _ptr(dev_status), _stream()))
    return topk_idx, scores_out


def dsa_topk_candidates(scores, topk_idx, idx_offset, cand_scores=None, cand_idx=None):
    """One key slice's selection as (score, global index) pairs: scores [B, L_slice] fp32,
    topk_idx int32 [B, k] (local indices) -> (cand_scores fp32 [B, k], cand_idx int32 [B, k])."""
    _need(scores, torch.float32, "scores")
    _need(topk_idx, torch.int32, "topk_idx")
    _contig(scores, "scores")
    _contig(topk_idx, "topk_idx")
    B, L_slice = scores.shape
    k = topk_idx.shape[1]
    if cand_scores is None:
        cand_scores = torch.empty((B, k), dtype=torch.float32, device=scores.device)
    if cand_idx is None:
        cand_idx = torch.empty((B, k), dtype=torch.int32, device=scores.device)
    _check(_lib.dsa_topk_candidates(_ptr(scores), _ptr(topk_idx), B, L_slice, k, int(idx_offset), _ptr(cand_scores),
                                    _ptr(cand_idx), _stream()))
    return cand_scores, cand_idx


def dsa_topk_merge(cand_scores, cand_idx, topk_idx=None, dev_status=None):
    """The slices' candidates [n_parts, B, k] (slice order) -> topk_idx int32 [B, k]: the
    k best under (score desc, index asc), increasing index order, -1 padded."""
    _need(cand_scores, torch.float32, "cand_scores")
    _need(cand_idx, torch.int32, "cand_idx")
    _contig(cand_scores, "cand_scores")
    _contig(cand_idx, "cand_idx")
    n, B, k = cand_idx.shape
    if tuple(cand_scores.shape) != (n, B, k):
        raise ValueError("cand_scores and cand_idx shapes differ")
    if topk_idx is None:
        topk_idx = torch.empty((B, k), dtype=torch.int32, device=cand_idx.device)
    _check(_lib.dsa_topk_merge(_ptr(cand_scores), _ptr(cand_idx), n, B, k, _ptr(topk_idx), _ptr(dev_status),
                               _stream()))
    return topk_idx


def attn_decode_sparse_workspace_bytes(B, Hq, Dv, k) -> int:
    return int(_lib.attn_decode_sparse_workspace_bytes(B, Hq, Dv, k))


def attn_decode_sparse(q, latent, topk_idx, Dv, scale, out=None, lse=None, ws=None, dev_status=None,
                       want_lse=True):
    """q [B, Hq, Dk] bf16, latent [B, L_max, Dk] bf16, topk_idx int32 [B, k]
    -> (out [B, Hq, Dv] bf16, lse [B, Hq] fp32)."""
    _need(q, torch.bfloat16, "q")
    _need(latent, torch.bfloat16, "latent")
    _need(topk_idx, torch.int32, "topk_idx")
    for t, n in ((q, "q"), (latent, "latent"), (topk_idx, "topk_idx")):
        _contig(t, n)
    B, Hq, Dk = q.shape
    L_max = latent.shape[1]
    k = topk_idx.shape[1]
    if out is None:
        out = torch.empty((B, Hq, Dv), dtype=torch.bfloat16, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    if ws is None:
        ws = workspace(attn_decode_sparse_workspace_bytes(B, Hq, Dv, k), q.device)
    _check(_lib.attn_decode_sparse(_ptr(q), _ptr(latent), _ptr(topk_idx), B, Hq, Dk, Dv, L_max, k, float(scale),
                                   _ptr(out), _ptr(lse), _ptr(ws), ws.numel(), _ptr(dev_status), _stream()))
    return out, lse


def attn_decode_sparse_fp8(q, latent_fp8, topk_idx, Dv, scale, out=None, lse=None, ws=None, dev_status=None,
                           want_lse=True):
    """q [B, Hq, 576] bf16, latent_fp8 [B, L_max, 656] uint8 (latent_quant_fp8 rows),
    topk_idx int32 [B, k] -> (out [B, Hq, Dv] bf16, lse [B, Hq] fp32)."""
    _need(q, torch.bfloat16, "q")
    _need(latent_fp8, torch.uint8, "latent_fp8")
    _need(topk_idx, torch.int32, "topk_idx")
    for t, n in ((q, "q"), (latent_fp8, "latent_fp8"), (topk_idx, "topk_idx")):
        _contig(t, n)
    B, Hq, Dk = q.shape
    if latent_fp8.dim() != 3 or latent_fp8.shape[0] != B or latent_fp8.shape[2] != LATENT_FP8_ROW_BYTES:
        raise ValueError("latent_fp8 must be [B, L_max, 656]")
    L_max = latent_fp8.shape[1]
    k = topk_idx.shape[1]
    if out is None:
        out = torch.empty((B, Hq, Dv), dtype=torch.bfloat16, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    if ws is None:
        ws = workspace(attn_decode_sparse_workspace_bytes(B, Hq, Dv, k), q.device)
    _check(_lib.attn_decode_sparse_fp8(_ptr(q), _ptr(latent_fp8), _ptr(topk_idx), B, Hq, Dk, Dv, L_max, k,
                                       float(scale), _ptr(out), _ptr(lse), _ptr(ws), ws.numel(), _ptr(dev_status),
                                       _stream()))
    return out, lse


LATENT_FP8_ROW_BYTES = 656


def latent_quant_fp8(latent, packed=None):
    """latent [..., 576] bf16 (contiguous) -> packed FP8 rows [..., 656] uint8."""
    _need(latent, torch.bfloat16, "latent")
    _contig(latent, "latent")
    if latent.shape[-1] != 576:
        raise ValueError("latent rows are 576 wide")
    n = latent.numel() // 576
    if packed is None:
        packed = torch.empty(tuple(latent.shape[:-1]) + (LATENT_FP8_ROW_BYTES,), dtype=torch.uint8,
                             device=latent.device)
    _need(packed, torch.uint8, "packed")
    _contig(packed, "packed")
    if packed.numel() != n * LATENT_FP8_ROW_BYTES:
        raise ValueError("packed must hold 656 bytes per row")
    _check(_lib.latent_quant_fp8(_ptr(latent), n, _ptr(packed), _stream()))
    return packed


def idx_key_quant_fp8(k_idx, codes=None, scales=None):
    """k_idx [..., 128] bf16 (contiguous) -> (codes [..., 128] uint8, scales [...] fp32)."""
    _need(k_idx, torch.bfloat16, "k_idx")
    _contig(k_idx, "k_idx")
    if k_idx.shape[-1] != 128:
        raise ValueError("indexer keys are 128 wide")
    n = k_idx.numel() // 128
    if codes is None:
        codes = torch.empty(k_idx.shape, dtype=torch.uint8, device=k_idx.device)
    if scales is None:
        scales = torch.empty(k_idx.shape[:-1], dtype=torch.float32, device=k_idx.device)
    _need(codes, torch.uint8, "codes")
    _need(scales, torch.float32, "scales")
    if codes.numel() != n * 128 or scales.numel() != n:
        raise ValueError("codes / scales sizes")
    _check(_lib.idx_key_quant_fp8(_ptr(k_idx), n, _ptr(codes), _ptr(scales), _stream()))
    return codes, scales


QSA_BLOCK = 4


def qsa_block_keys(k_idx, seq_lens, cos, sin, block_keys=None, block_from=None, max_new=0, eps=1e-6, pair_style=0,
                   dev_status=None):
    """k_idx [B, L_max, 128] bf16 (L_max a multiple of 4), seq_lens int32 [B] (tokens)
    -> block_keys [B, L_max // 4, 128] bf16 (groups [block_from, min(len // 4,
    block_from + max_new)) written)."""
    _need(k_idx, torch.bfloat16, "k_idx")
    _contig(k_idx, "k_idx")
    _need(seq_lens, torch.int32, "seq_lens")
    B, L_max, dI = k_idx.shape
    if block_keys is None:
        block_keys = torch.zeros((B, L_max // QSA_BLOCK, dI), dtype=torch.bfloat16, device=k_idx.device)
    _need(block_keys, torch.bfloat16, "block_keys")
    if block_from is not None:
        _need(block_from, torch.int32, "block_from")
    _check(_lib.qsa_block_keys(_ptr(k_idx), _ptr(seq_lens), _ptr(block_from), int(max_new), B, dI, L_max, _ptr(cos),
                               _ptr(sin), cos.shape[0], pair_style, float(eps), _ptr(block_keys), _ptr(dev_status),
                               _stream()))
    return block_keys


def qsa_select_workspace_bytes(B, L_max, n_top) -> int:
    return int(_lib.qsa_select_workspace_bytes(B, L_max, n_top))


def qsa_select(q_idx, w, block_keys, seq_lens, n_top=512, tok_idx=None, tok_count=None, scores_out=None, ws=None,
               dev_status=None, want_scores=False):
    """q_idx [B, 64, 128] bf16, w [B, 64] fp32, block_keys [B, L_max // 4, 128] bf16,
    seq_lens int32 [B] -> (tok_idx int32 [B, 4 n_top + 3], tok_count int32 [B],
    group scores fp32 [B, L_max // 4] or None)."""
    _need(q_idx, torch.bfloat16, "q_idx")
    _need(block_keys, torch.bfloat16, "block_keys")
    _need(w, torch.float32, "w")
    _need(seq_lens, torch.int32, "seq_lens")
    for t, n in ((q_idx, "q_idx"), (block_keys, "block_keys"), (w, "w")):
        _contig(t, n)
    B, HI, dI = q_idx.shape
    L_max = block_keys.shape[1] * QSA_BLOCK
    dev = q_idx.device
    if tok_idx is None:
        tok_idx = torch.empty((B, QSA_BLOCK * n_top + QSA_BLOCK - 1), dtype=torch.int32, device=dev)
    if tok_count is None:
        tok_count = torch.empty(B, dtype=torch.int32, device=dev)
    if scores_out is None and want_scores:
        scores_out = torch.empty((B, L_max // QSA_BLOCK), dtype=torch.float32, device=dev)
    if ws is None:
        ws = workspace(qsa_select_workspace_bytes(B, L_max, n_top), dev)
    _check(_lib.qsa_select(_ptr(q_idx), _ptr(w), _ptr(block_keys), _ptr(seq_lens), B, HI, dI, L_max, n_top,
                           _ptr(tok_idx), _ptr(tok_count), _ptr(scores_out), _ptr(ws), ws.numel(), _ptr(dev_status),
                           _stream()))
    return tok_idx, tok_count, scores_out


def attn_decode_gqa_sparse_workspace_bytes(B, n_head, n_kv_head, head_dim, n_idx) -> int:
    return int(_lib.attn_decode_gqa_sparse_workspace_bytes(B, n_head, n_kv_head, head_dim, n_idx))


def attn_decode_gqa_sparse(q, k_cache, v_cache, tok_idx, scale, tok_count=None, out=None, lse=None, ws=None,
                           dev_status=None, want_lse=True):
    """q [B, H, d] bf16, k_cache/v_cache [B, Hk, T_max, d] bf16, tok_idx int32 [B, n_idx]
    (the first tok_count[b] entries used; -1 skipped) -> (out [B, H, d], lse [B, H])."""
    for t, n in ((q, "q"), (k_cache, "k_cache"), (v_cache, "v_cache"), (tok_idx, "tok_idx")):
        _contig(t, n)
    for t, n in ((q, "q"), (k_cache, "k_cache"), (v_cache, "v_cache")):
        _need(t, torch.bfloat16, n)
    _need(tok_idx, torch.int32, "tok_idx")
    if tok_count is not None:
        _need(tok_count, torch.int32, "tok_count")
    B, H, d = q.shape
    Bk, Hk, T_max, dk = k_cache.shape
    if (Bk, dk) != (B, d) or v_cache.shape != k_cache.shape or tok_idx.shape[0] != B:
        raise ValueError("inconsistent sparse decode shapes")
    n_idx = tok_idx.shape[1]
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((B, H), dtype=torch.float32, device=q.device)
    if ws is None:
        ws = workspace(attn_decode_gqa_sparse_workspace_bytes(B, H, Hk, d, n_idx), q.device)
    _check(_lib.attn_decode_gqa_sparse(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(tok_idx), _ptr(tok_count), n_idx, B,
                                       H, Hk, d, T_max, float(scale), _ptr(out), _ptr(lse), _ptr(ws), ws.numel(),
                                       _ptr(dev_status), _stream()))
    return out, lse


def attn_merge_lse(o_parts, lse_parts, out=None, lse=None, want_lse=True):
    """o_parts [n, B, H, d] bf16, lse_parts [n, B, H] fp32 (decode results over disjoint
    key sets) -> (out [B, H, d] bf16, lse [B, H] fp32 or None) over their union."""
    _need(o_parts, torch.bfloat16, "o_parts")
    _need(lse_parts, torch.float32, "lse_parts")
    _contig(o_parts, "o_parts")
    _contig(lse_parts, "lse_parts")
    n, B, H, d = o_parts.shape
    if lse_parts.shape != (n, B, H):
        raise ValueError("lse_parts must be [n, B, H]")
    if out is None:
        out = torch.empty((B, H, d), dtype=torch.bfloat16, device=o_parts.device)
    if lse is None and want_lse:
        lse = torch.empty((B, H), dtype=torch.float32, device=o_parts.device)
    _check(_lib.attn_merge_lse(_ptr(o_parts), _ptr(lse_parts), n, B, H, d, _ptr(out), _ptr(lse), _stream()))
    return out, lse
