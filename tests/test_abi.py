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
