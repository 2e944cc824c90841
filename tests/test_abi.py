"""The C-ABI library: it builds for sm_100a, loads, exports every function that
include/kvattn.h declares, and rejects bad arguments on the host before any
launch.  CPU only (no compute calls)."""
import ctypes
import os
import re
import subprocess

import pytest

from mqa_kv_cache_b200 import build as kbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "kvattn.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+char\s*\*|int|size_t)\s+(\w+)\s*\(", text, flags=re.M)))


@pytest.fixture(scope="module")
def lib():
    return ctypes.CDLL(kbuild.build())


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ("rope_table_build", "rope_apply_qk", "attn_decode_gqa", "attn_prefill_causal", "dsa_index_topk",
              "attn_decode_sparse"):
        assert n in names


def test_header_is_plain_c():
    subprocess.run(["gcc", "-fsyntax-only", "-std=c99", "-Wall", "-Werror", "-x", "c", HEADER], check=True)


def test_library_exports_every_declared_symbol(lib):
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


def test_built_for_sm100a_only():
    objs = os.path.join(os.path.dirname(kbuild.LIB), "_build")
    assert os.path.isdir(objs)
    assert "arch=compute_100a,code=sm_100a" in kbuild.ARCH


def _err(lib):
    lib.kvattn_last_error_string.restype = ctypes.c_char_p
    return lib.kvattn_last_error_string().decode()


def test_host_validation_rejects_before_launch(lib):
    vp = ctypes.c_void_p
    # NULL tensors
    rc = lib.attn_decode_gqa(None, None, None, None, 1, 8, 2, 64, 16, ctypes.c_float(0.125), None, None, None,
                             ctypes.c_size_t(0), None, None)
    assert rc == -1 and "NULL" in _err(lib)
    fake = vp(1 << 20)  # never dereferenced: validation fails first
    # group size not supported (n_head % n_kv_head != 0)
    rc = lib.attn_decode_gqa(fake, fake, fake, fake, 1, 6, 4, 64, 16, ctypes.c_float(0.125), fake, None, fake,
                             ctypes.c_size_t(1 << 20), None, None)
    assert rc == -3 and "multiple" in _err(lib)
    # unsupported head_dim
    rc = lib.attn_decode_gqa(fake, fake, fake, fake, 1, 8, 2, 96, 16, ctypes.c_float(0.125), fake, None, fake,
                             ctypes.c_size_t(1 << 20), None, None)
    assert rc == -4
    # misaligned pointer
    rc = lib.attn_decode_gqa(vp((1 << 20) + 2), fake, fake, fake, 1, 8, 2, 64, 16, ctypes.c_float(0.125), fake,
                             None, fake, ctypes.c_size_t(1 << 20), None, None)
    assert rc == -2


def test_rope_table_rejects_bad_params(lib):
    class P(ctypes.Structure):
        _fields_ = [("head_dim", ctypes.c_int), ("scaling", ctypes.c_int), ("pair_style", ctypes.c_int),
                    ("reserved", ctypes.c_int), ("base", ctypes.c_double), ("s", ctypes.c_double),
                    ("L_train", ctypes.c_double), ("alpha", ctypes.c_double), ("beta", ctypes.c_double),
                    ("L_cur", ctypes.c_double)]
    fake = ctypes.c_void_p(1 << 20)
    p = P(63, 0, 0, 0, 10000.0, 1.0, 0.0, 1.0, 32.0, 0.0)
    assert lib.rope_table_build(ctypes.byref(p), 16, fake, fake, None) == -3
    p = P(64, 3, 0, 0, 10000.0, 4.0, 8192.0, 32.0, 1.0, 0.0)  # beta <= alpha
    assert lib.rope_table_build(ctypes.byref(p), 16, fake, fake, None) == -3
    p = P(64, 9, 0, 0, 10000.0, 4.0, 8192.0, 1.0, 32.0, 0.0)
    assert lib.rope_table_build(ctypes.byref(p), 16, fake, fake, None) == -4
    p = P(64, 1, 0, 0, 10000.0, 0.5, 0.0, 1.0, 32.0, 0.0)  # PI with s < 1
    assert lib.rope_table_build(ctypes.byref(p), 16, fake, fake, None) == -3


def test_new_entry_points_reject_bad_arguments_on_the_host(lib):
    vp, i32, f32, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    fake = vp(1 << 20)  # never dereferenced: validation fails first
    # qsa_block_keys: NULL, width other than 128, L_max not a multiple of 4
    lib.qsa_block_keys.argtypes = [vp, vp, vp, i32, i32, i32, i32, vp, vp, i32, i32, f32, vp, vp, vp]
    assert lib.qsa_block_keys(None, fake, None, 0, 1, 128, 64, fake, fake, 64, 0, 1e-6, fake, None, None) == -1
    assert lib.qsa_block_keys(fake, fake, None, 0, 1, 64, 64, fake, fake, 64, 0, 1e-6, fake, None, None) == -4
    assert lib.qsa_block_keys(fake, fake, None, 0, 1, 128, 66, fake, fake, 64, 0, 1e-6, fake, None, None) == -3
    assert "multiple of 4" in _err(lib)
    # qsa_select: n_top outside 1..2048, wrong indexer shape, misaligned output
    lib.qsa_select.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, i32, vp, vp, vp, vp, sz, vp, vp]
    assert lib.qsa_select(fake, fake, fake, fake, 1, 64, 128, 64, 0, fake, fake, None, fake, 1 << 20, None, None) == -3
    assert lib.qsa_select(fake, fake, fake, fake, 1, 32, 128, 64, 8, fake, fake, None, fake, 1 << 20, None, None) == -4
    assert lib.qsa_select(fake, fake, fake, fake, 1, 64, 128, 64, 8, vp((1 << 20) + 4), fake, None, fake, 1 << 20,
                          None, None) == -2
    # attn_decode_gqa_sparse: NULL list, group above 32 at head_dim 128
    lib.attn_decode_gqa_sparse.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, f32, vp, vp, vp, sz, vp, vp]
    assert lib.attn_decode_gqa_sparse(fake, fake, fake, None, None, 8, 1, 8, 2, 128, 64, 0.1, fake, None, fake,
                                      1 << 20, None, None) == -1
    assert lib.attn_decode_gqa_sparse(fake, fake, fake, fake, None, 8, 1, 64, 1, 128, 64, 0.1, fake, None, fake,
                                      1 << 20, None, None) == -4
    # attn_merge_lse: no parts, unsupported head_dim
    lib.attn_merge_lse.argtypes = [vp, vp, i32, i32, i32, i32, vp, vp, vp]
    assert lib.attn_merge_lse(fake, fake, 0, 1, 8, 128, fake, None, None) == -3
    assert lib.attn_merge_lse(fake, fake, 2, 1, 8, 96, fake, None, None) == -4
