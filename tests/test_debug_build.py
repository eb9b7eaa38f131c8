"""The DSA_DEBUG build (libdsa_debug.so): host-checked gather indices and
shared-memory canaries. CPU side: it builds, exports every symbol the header
declares and validates arguments as the release build does."""
import ctypes
import os
import re

import pytest

from indexed_sparse_attention_relu_b200 import binding as B
from indexed_sparse_attention_relu_b200 import build as build_mod

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def dlib():
    return ctypes.CDLL(build_mod.build(debug=True))


def test_debug_library_exports_the_header(dlib):
    text = re.sub(r"/\*.*?\*/", "", open(os.path.join(ROOT, "include", "dsa.h")).read(), flags=re.S)
    for name in sorted(set(re.findall(r"\b(dsa_[a-z0-9_]+)\s*\(", text))):
        assert hasattr(dlib, name), name
    assert build_mod.DEBUG_LIB.endswith("libdsa_debug.so")


def test_debug_library_validates_like_the_release_build(dlib):
    dlib.dsa_sparse_mla_attn.argtypes = [ctypes.POINTER(B.dsa_batch), ctypes.POINTER(B.dsa_mla_in), ctypes.c_void_p,
                                         ctypes.c_int32, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                         ctypes.c_size_t, ctypes.c_void_p]
    fake = 0x10000
    bt = B.dsa_batch(2, 2, 256, fake, fake, fake, None, 0, 0)
    mla = B.dsa_mla_in(128, 256, 64, 0.04, fake, fake, 0)   # d_latent 256: unsupported
    assert dlib.dsa_sparse_mla_attn(ctypes.byref(bt), ctypes.byref(mla), fake, 64, fake, None, None, 0, None) == \
        B.DSA_ERR_UNSUPPORTED_SHAPE
    empty = B.dsa_batch(2, 0, 256, fake, fake, fake, None, 0, 0)
    mla_ok = B.dsa_mla_in(128, 512, 64, 0.04, fake, fake, 0)
    # an empty batch returns before the (synchronising) index check
    assert dlib.dsa_sparse_mla_attn(ctypes.byref(empty), ctypes.byref(mla_ok), fake, 64, fake, None, None, 0,
                                    None) == B.DSA_OK
