"""The Python binding's checks of caller-supplied buffers, on CPU.

The library only receives pointers, so the binding must reject an output,
tau, mask or workspace tensor whose shape, dtype, device or layout differs
from what the kernels access.  Here CPU tensors stand in for device tensors:
the CUDA-device check of q, k, v is lifted, and the stream lookup (the step
after validation) is replaced by a sentinel, so a call that passes
validation stops there without reaching the library's compute entry points.
"""

import pytest
import torch

import differentiable_sparse_attention_b200 as dsa


class Validated(Exception):
    """Raised where the binding would look up the CUDA stream."""


@pytest.fixture
def cpu_binding(monkeypatch):
    def check_qkv(*ts):
        ref = ts[0]
        for t in ts:
            assert t.shape == ref.shape and t.dtype == ref.dtype and t.is_contiguous()

    def stream_ptr(stream, device):
        raise Validated

    monkeypatch.setattr(dsa, "_check_qkv", check_qkv)
    monkeypatch.setattr(dsa, "_stream_ptr", stream_ptr)
    return dsa


B, H, N, D = 1, 2, 256, 64


def qkv(dtype=torch.bfloat16):
    return [torch.zeros((B, H, N, D), dtype=dtype) for _ in range(4)]


def fwd_bufs(block=128):
    mrows = (N + block - 1) // block
    return dict(out=torch.empty((B, H, N, D), dtype=torch.bfloat16),
                tau=torch.empty((B, H, N), dtype=torch.float32),
                mask=torch.empty((B, H, mrows, dsa.mask_words(N, block)), dtype=torch.int32),
                workspace=dsa.alloc_workspace(B, H, N, D, block, True, "cpu"))


def test_forward_accepts_matching_buffers(cpu_binding):
    q, k, v, _ = qkv()
    with pytest.raises(Validated):
        dsa.entmax_attn_fwd(q, k, v, 1.5, True, 128, **fwd_bufs())
    with pytest.raises(Validated):          # buffers allocated by the binding
        dsa.entmax_attn_fwd(q, k, v, 1.5, True, 64)


@pytest.mark.parametrize("name, bad", [
    ("out", torch.empty((B, H, N - 1, D), dtype=torch.bfloat16)),
    ("out", torch.empty((B, H, N, D), dtype=torch.float32)),
    ("out", torch.empty((B, H, D, N), dtype=torch.bfloat16).transpose(-1, -2)),
    ("tau", torch.empty((B, H, N), dtype=torch.float64)),
    ("tau", torch.empty((B, H, N // 2), dtype=torch.float32)),
    ("mask", torch.empty((B, H, 1, 1), dtype=torch.int32)),
    ("mask", torch.empty((B, H, 2, 1), dtype=torch.int64)),
    ("workspace", torch.empty((2, 64), dtype=torch.uint8)),
    ("workspace", torch.empty(64, dtype=torch.float32)),
])
def test_forward_rejects_mismatched_buffers(cpu_binding, name, bad):
    q, k, v, _ = qkv()
    bufs = fwd_bufs()
    bufs[name] = bad
    with pytest.raises(ValueError, match=name):
        dsa.entmax_attn_fwd(q, k, v, 1.5, True, 128, **bufs)


def test_backward_checks_its_buffers(cpu_binding):
    q, k, v, do = qkv()
    f = fwd_bufs()
    ok = dict(dq=torch.empty_like(q), dk=torch.empty_like(k), dv=torch.empty_like(v),
              workspace=f["workspace"])
    with pytest.raises(Validated):
        dsa.entmax_attn_bwd(q, k, v, do, f["tau"], f["mask"], 1.5, True, 128, **ok)
    with pytest.raises(ValueError, match="dq"):
        dsa.entmax_attn_bwd(q, k, v, do, f["tau"], f["mask"], 1.5, True, 128,
                            **{**ok, "dq": torch.empty_like(q, dtype=torch.float32)})
    with pytest.raises(ValueError, match="dv"):
        dsa.entmax_attn_bwd(q, k, v, do, f["tau"], f["mask"], 1.5, True, 128,
                            **{**ok, "dv": torch.empty((B, H, N, D + 1), dtype=torch.bfloat16)})
    with pytest.raises(ValueError, match="tau"):
        dsa.entmax_attn_bwd(q, k, v, do, f["tau"][:, :1], f["mask"], 1.5, True, 128, **ok)
    with pytest.raises(ValueError, match="mask"):   # a block-64 mask given to a block-128 call
        dsa.entmax_attn_bwd(q, k, v, do, f["tau"], fwd_bufs(64)["mask"], 1.5, True, 128, **ok)
    # bf16 gradients need the forward's workspace
    with pytest.raises(ValueError, match="workspace"):
        dsa.entmax_attn_bwd(q, k, v, do, f["tau"], f["mask"], 1.5, True, 128,
                            dq=ok["dq"], dk=ok["dk"], dv=ok["dv"])


def test_router_rejects_bad_chunk_and_dtype():
    q = torch.zeros((1, 2, 64, 64), dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="chunk"):
        dsa.dash_route(q, q, 0, 4.0)
    with pytest.raises(TypeError, match="bfloat16"):
        dsa.dash_route(q.float(), q.float(), 16, 4.0)
    with pytest.raises(ValueError, match="CUDA"):     # CPU tensors never reach the library
        dsa.dash_route(q, q, 16, 4.0)
