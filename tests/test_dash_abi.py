"""Host-side checks of the router's C ABI (include/dash_route.h), no GPU: every
declared function is exported and invalid arguments are rejected before any
device work.  The fake pointers below are never dereferenced."""

import ctypes
import os
import re

import pytest

import differentiable_sparse_attention_b200 as dsa
from differentiable_sparse_attention_b200 import build as build_mod

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dash_route.h")
FAKE = ctypes.c_void_p(1 << 20)
MISALIGNED = ctypes.c_void_p((1 << 20) + 8)


@pytest.fixture(scope="module")
def lib():
    build_mod.build()
    return dsa._lib()


def declared():
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    return sorted(set(re.findall(r"\b(dash_route_\w+)\s*\(", text)))


def test_header_matches_binding_and_library(lib):
    assert set(declared()) == set(dsa.DASH_EXPORTED)
    for name in declared():
        assert getattr(lib, name) is not None


def call(lib, *, q=FAKE, B=1, Hq=4, Hkv=2, N=256, D=64, chunk=16, gamma=4.0, alpha=1.5,
         max_iter=4, wbar=FAKE, ws=FAKE, ws_bytes=None):
    if ws_bytes is None:
        ws_bytes = lib.dash_route_workspace_size(B, Hq, Hkv, N, D, chunk)
    return lib.dash_route_fwd(q, FAKE, B, Hq, Hkv, N, D, chunk, gamma, alpha, max_iter, wbar, FAKE,
                              FAKE, ws, ws_bytes, None)


def test_argument_validation(lib):
    assert call(lib, q=None) == dsa.E_NULL
    assert call(lib, ws=None) == dsa.E_NULL
    assert call(lib, wbar=None) == dsa.E_NULL
    assert call(lib, Hq=3) == dsa.E_SHAPE              # not a multiple of Hkv
    assert call(lib, Hkv=0) == dsa.E_SHAPE
    assert call(lib, N=257 * 16, chunk=16) == dsa.E_SHAPE   # 257 complete chunks > 256
    assert call(lib, chunk=0) == dsa.E_SHAPE
    assert call(lib, D=96) == dsa.E_UNSUPPORTED
    assert call(lib, alpha=1.0) == dsa.E_ALPHA
    assert call(lib, alpha=3.5) == dsa.E_ALPHA
    assert call(lib, gamma=0.0) == dsa.E_SHAPE
    assert call(lib, max_iter=17) == dsa.E_MAXITER
    assert call(lib, q=MISALIGNED) == dsa.E_ALIGN
    assert call(lib, ws_bytes=1) == dsa.E_WORKSPACE


def test_no_complete_chunk_is_a_no_op(lib):
    # N < chunk: empty outputs, accepted with NULL output pointers, nothing launched
    assert call(lib, N=10, chunk=16, wbar=None) == dsa.OK


def test_workspace_size(lib):
    small = lib.dash_route_workspace_size(1, 4, 2, 256, 64, 16)
    big = lib.dash_route_workspace_size(1, 4, 2, 4096, 64, 16)
    assert 0 < small < big
    assert lib.dash_route_workspace_size(1, 3, 2, 256, 64, 16) == 0
