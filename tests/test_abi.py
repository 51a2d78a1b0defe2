"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every function that include/entmax_attn.h declares, and rejects invalid
arguments before touching any device state.

Every call below fails validation before any CUDA call is made, so the fake
(but aligned, non-null) pointers are never dereferenced.
"""

import ctypes
import os
import re

import pytest

import differentiable_sparse_attention_b200 as dsa
from differentiable_sparse_attention_b200 import build as build_mod

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "entmax_attn.h")


@pytest.fixture(scope="module")
def lib():
    build_mod.build()
    return dsa._lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(entmax_attn_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    assert set(names) == set(dsa.EXPORTED)


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
        assert getattr(lib, name) is not None


def test_bounds_checked_build_exports_the_same_boundary():
    # the debug build (-DENTMAX_BOUNDS_CHECK) is the same C ABI
    path = build_mod.build(bounds_check=True)
    assert path.endswith("libentmax_attn_bounds.so")
    dbg = ctypes.CDLL(path)
    for name in declared_functions():
        assert getattr(dbg, name) is not None, name
    dbg.entmax_attn_error_string.restype = ctypes.c_char_p
    assert dbg.entmax_attn_error_string(0) == b"success"


FAKE = ctypes.c_void_p(1 << 20)          # 256-byte aligned, never dereferenced
MISALIGNED = ctypes.c_void_p((1 << 20) + 8)


def fwd(lib, *, q=FAKE, B=1, H=1, N=256, D=64, dtype=0, alpha=1.5, causal=1, block=128,
        max_iter=2, out=FAKE, ws=FAKE, ws_bytes=None):
    if ws_bytes is None:
        ws_bytes = lib.entmax_attn_workspace_size(B, H, N, D, block, causal) if N > 0 else 0
    return lib.entmax_attn_fwd(q, FAKE, FAKE, B, H, N, D, dtype, alpha, causal, block, max_iter,
                               out, FAKE, FAKE, None, ws, ws_bytes, None)


def test_forward_argument_validation(lib):
    assert fwd(lib, q=None) == dsa.E_NULL
    assert fwd(lib, out=None) == dsa.E_NULL
    assert fwd(lib, ws=None) == dsa.E_NULL
    assert fwd(lib, N=0) == dsa.E_SHAPE
    assert fwd(lib, N=262145) == dsa.E_SHAPE
    assert fwd(lib, B=0) == dsa.E_SHAPE
    assert fwd(lib, D=96) == dsa.E_UNSUPPORTED
    assert fwd(lib, block=32) == dsa.E_UNSUPPORTED
    assert fwd(lib, dtype=7) == dsa.E_UNSUPPORTED
    assert fwd(lib, dtype=1, D=128) == dsa.E_UNSUPPORTED   # fp32 path: head dim 64
    assert fwd(lib, alpha=1.0) == dsa.E_ALPHA
    assert fwd(lib, alpha=1.02) == dsa.E_ALPHA    # k = 1/(alpha - 1) above 20
    assert fwd(lib, alpha=3.5) == dsa.E_ALPHA
    assert fwd(lib, alpha=float("nan")) == dsa.E_ALPHA
    assert fwd(lib, dtype=1, alpha=1.7) == dsa.E_UNSUPPORTED   # fp32 path: 1.5 and 2 only
    assert fwd(lib, max_iter=-1) == dsa.E_MAXITER
    assert fwd(lib, max_iter=17) == dsa.E_MAXITER
    assert fwd(lib, q=MISALIGNED) == dsa.E_ALIGN
    assert fwd(lib, ws_bytes=1) == dsa.E_WORKSPACE


def test_backward_argument_validation(lib):
    def bwd(q=FAKE, D=64, block=128, alpha=1.5, ws_bytes=None, dq=FAKE):
        if ws_bytes is None:
            ws_bytes = lib.entmax_attn_workspace_size(1, 1, 256, 64, 128, 1)
        return lib.entmax_attn_bwd(q, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 1, 256, D, 0, alpha, 1,
                                   block, dq, FAKE, FAKE, FAKE, ws_bytes, None)
    assert bwd(q=None) == dsa.E_NULL
    assert bwd(dq=None) == dsa.E_NULL
    assert bwd(D=32) == dsa.E_UNSUPPORTED
    assert bwd(alpha=5.0) == dsa.E_ALPHA
    assert bwd(alpha=2.5) == dsa.E_ALPHA     # gradients: alpha <= 2 only
    assert bwd(alpha=1.75, q=None) == dsa.E_NULL   # generic alpha <= 2 is accepted
    assert bwd(q=MISALIGNED) == dsa.E_ALIGN
    assert bwd(ws_bytes=0) == dsa.E_WORKSPACE


def test_sizes(lib):
    assert dsa.mask_words(256, 64) == 1
    assert dsa.mask_words(4096, 128) == 1
    assert dsa.mask_words(131072, 128) == 32
    assert dsa.mask_words(300, 64) == 1
    assert lib.entmax_attn_mask_words(0, 128) == dsa.E_SHAPE
    assert lib.entmax_attn_mask_words(256, 96) == dsa.E_UNSUPPORTED
    small = dsa.workspace_size(1, 1, 256, 64, 128, True)
    big = dsa.workspace_size(1, 1, 4096, 64, 128, True)
    assert 0 < small < big
    # causal keeps only the lower triangle of tile maxima
    assert dsa.workspace_size(2, 16, 4096, 64, 128, True) < dsa.workspace_size(2, 16, 4096, 64, 128, False)
    assert dsa.workspace_size(1, 1, 0, 64, 128, True) == 0


def test_error_strings(lib):
    for code in (0, -1, -2, -3, -4, -5, -6, -7, -8, -99):
        s = dsa.error_string(code)
        assert isinstance(s, str) and s


def test_wait_selftest_validation(lib):
    assert lib.entmax_attn_wait_selftest(None, FAKE, 1000, None) == dsa.E_NULL
    assert lib.entmax_attn_wait_selftest(FAKE, None, 1000, None) == dsa.E_NULL
    assert lib.entmax_attn_wait_selftest(FAKE, FAKE, 0, None) == dsa.E_SHAPE
    assert lib.entmax_attn_wait_selftest(FAKE, FAKE, 2_000_000_000, None) == dsa.E_SHAPE
    assert lib.entmax_attn_wait_selftest(MISALIGNED, FAKE, 1000, None) == dsa.E_ALIGN


def test_grid_size_limit(lib):
    # one CTA per (batch, head, 128-row tile): B * H * ceil(N / 128) must fit 31 bits
    assert fwd(lib, B=1 << 14, H=1 << 14, N=1024, ws_bytes=1 << 40) == dsa.E_SHAPE
    assert fwd(lib, B=1 << 14, H=1 << 13, N=1024, ws_bytes=0) == dsa.E_WORKSPACE


def noalloc(lib, *, q=FAKE, B=1, H=1, N=256, D=64, dtype=0, alpha=1.5, causal=1, block=128,
            max_iter=2, out=FAKE):
    return lib.entmax_attn_fwd_noalloc(q, FAKE, FAKE, B, H, N, D, dtype, alpha, causal, block,
                                       max_iter, out, FAKE, FAKE, None)


def test_noalloc_argument_validation(lib):
    assert noalloc(lib, q=None) == dsa.E_NULL
    assert noalloc(lib, out=None) == dsa.E_NULL
    assert noalloc(lib, N=0) == dsa.E_SHAPE
    assert noalloc(lib, D=96) == dsa.E_UNSUPPORTED
    # fp32 inputs take the workspace forward: the fixed scratch serves bf16 only
    assert noalloc(lib, dtype=1) == dsa.E_UNSUPPORTED
    assert noalloc(lib, alpha=3.5) == dsa.E_ALPHA
    assert noalloc(lib, max_iter=17) == dsa.E_MAXITER
    assert noalloc(lib, q=MISALIGNED) == dsa.E_ALIGN


def test_noalloc_status_argument_validation(lib):
    assert lib.entmax_attn_noalloc_status(None, None) == dsa.E_NULL


def test_noalloc_scratch_limit(lib):
    # causal scratch: 256 + B*H*T(T+1)/2*512 bytes against 8 MiB, T = ceil(N / 128)
    t = 181
    assert 256 + t * (t + 1) // 2 * 512 > dsa.NOALLOC_SCRATCH_BYTES
    assert 256 + (t - 1) * t // 2 * 512 <= dsa.NOALLOC_SCRATCH_BYTES
    assert noalloc(lib, N=t * 128) == dsa.E_SCRATCH
    assert noalloc(lib, N=262144) == dsa.E_SCRATCH
    assert noalloc(lib, B=2, H=16, N=8192) == dsa.E_SCRATCH
    # non-causal keeps all T^2 tile maxima: T = 128 already exceeds 8 MiB
    assert noalloc(lib, N=128 * 128, causal=0) == dsa.E_SCRATCH
