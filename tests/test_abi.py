"""The C-ABI library loads on a CPU-only host and exports what include/mk.h declares."""
import ctypes
import os
import re

import pytest

import decode_persistent_block_b200 as dpb
from decode_persistent_block_b200 import mk

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    src = open(os.path.join(ROOT, "include", "mk.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return set(re.findall(r"^\s*(?:int|void|size_t|const\s+char\s*\*)\s*\*?\s*(mk_\w+)\s*\(", src, flags=re.M))


@pytest.fixture(scope="module")
def lib():
    dpb.build()
    return mk.load()


def test_every_declared_symbol_is_exported_and_bound(lib):
    names = declared_functions()
    assert len(names) >= 18, names
    for n in names:
        assert hasattr(lib, n), n
    assert names == set(mk.SIGNATURES), names ^ set(mk.SIGNATURES)


def test_strerror_and_codes(lib):
    for code, name in mk.ERRORS.items():
        assert lib.mk_strerror(code) and lib.mk_strerror(code) != b"unknown error", name
    assert lib.mk_strerror(12345) == b"unknown error"
    hdr = open(os.path.join(ROOT, "include", "mk.h")).read()
    for code, name in mk.ERRORS.items():
        assert re.search(rf"#define {name} \({code}\)", hdr), name


def test_default_options(lib):
    o = mk.make_options()
    assert o.l2_prefetch == -1 and o.mode == mk.MODE_MEGAKERNEL and o.ring_stages == 0


def test_create_rejects_bad_arguments_without_a_gpu(lib):
    h = ctypes.c_void_p()
    assert lib.mk_create(None, None, None, None, ctypes.byref(h)) == mk.CODES["MK_ERR_INVALID_ARG"]
    cfg = mk.MkConfig(2, 256, 4, 2, 96, 768, 4096, 0, 0, 1e-5, 1e4, 32, 0)  # head_dim 96
    assert lib.mk_create(ctypes.byref(cfg), None, None, None, ctypes.byref(h)) == mk.CODES["MK_ERR_UNSUPPORTED"]
    cfg.head_dim = 64
    # weights missing
    assert lib.mk_create(ctypes.byref(cfg), None, None, None, ctypes.byref(h)) == mk.CODES["MK_ERR_INVALID_ARG"]
    w = mk.MkWeights()
    assert lib.mk_create(ctypes.byref(cfg), ctypes.byref(w), None, None, ctypes.byref(h)) == \
        mk.CODES["MK_ERR_INVALID_ARG"]
    # handle-taking calls reject NULL
    assert lib.mk_build_schedule(None) == mk.CODES["MK_ERR_INVALID_ARG"]
    assert lib.mk_decode_step(None, 0, 0, None, None) == mk.CODES["MK_ERR_INVALID_ARG"]
    assert lib.mk_reset(None) == mk.CODES["MK_ERR_INVALID_ARG"]
    lib.mk_destroy(None)
