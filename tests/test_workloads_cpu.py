"""The input recipe of the synthetic workloads, on CPU.

Every parity test and bench figure is fed from workloads.make_inputs; these
tests pin what that recipe states: seeded N(0, 1) draws in the order q, k, v,
dO; the temperature applied to q before the cast; and, for the planted
workload, 32 key blocks per head whose keys (like every query) have cosine
about 0.8 with one seeded direction of that head, while the other keys do not.
"""

import pytest
import torch

from differentiable_sparse_attention_b200 import workloads as W


def test_seeded_and_deterministic():
    w = W.TINY_FP32.with_(N=64)
    a, b = W.make_inputs(w), W.make_inputs(w)
    for n in ("q", "k", "v", "dout"):
        assert torch.equal(a[n], b[n])
    c = W.make_inputs(w.with_(seed=1))
    assert not torch.equal(a["q"], c["q"])


def test_draw_order_q_k_v_dout():
    w = W.TINY_FP32.with_(N=48, seed=7)
    x = W.make_inputs(w)
    g = torch.Generator().manual_seed(7)
    shape = (w.B, w.H, w.N, w.D)
    for n in ("q", "k", "v", "dout"):
        assert torch.equal(x[n], torch.randn(shape, generator=g, dtype=torch.float32)), n


def test_temperature_scales_q_before_the_cast():
    w = W.TINY_FP32.with_(N=48)
    x1 = W.make_inputs(w)
    x4 = W.make_inputs(w.with_(temperature=4.0))
    assert torch.equal(x4["q"], 4.0 * x1["q"])
    for n in ("k", "v", "dout"):
        assert torch.equal(x4[n], x1[n])
    # bf16: the scaled fp32 q is cast once
    wb = W.ALPHA15_4K.with_(B=1, H=1, N=64, temperature=2.0)
    xb = W.make_inputs(wb)
    ref = W.make_inputs(wb.with_(temperature=1.0, dtype="fp32"))["q"] * 2.0
    assert xb["q"].dtype == torch.bfloat16 and xb["q"].is_contiguous()
    assert torch.equal(xb["q"], ref.to(torch.bfloat16))


def test_without_dout_the_other_tensors_are_unchanged():
    w = W.TINY_FP32.with_(N=48)
    full, part = W.make_inputs(w), W.make_inputs(w, need_grad_inputs=False)
    assert "dout" not in part
    for n in ("q", "k", "v"):
        assert torch.equal(full[n], part[n])


def test_planted_blocks_align_with_one_direction_per_head():
    w = W.PLANTED_32K.with_(H=2, N=8192, dtype="fp32")     # 64 key blocks of 128
    x = W.make_inputs(w, need_grad_inputs=False)
    tc = w.N // w.block
    for h in range(w.H):
        q, k = x["q"][0, h], x["k"][0, h]
        # every query is 0.8 sqrt(D) u + 0.6 noise: their mean points along u
        u = q.mean(dim=0)
        u = u / u.norm()
        cos_q = (q @ u) / q.norm(dim=-1)
        assert abs(cos_q.mean().item() - 0.8) < 0.03
        cos_k = (k @ u) / k.norm(dim=-1)
        per_block = cos_k.view(tc, w.block).mean(dim=1)
        planted = per_block > 0.5
        assert int(planted.sum()) == w.planted_blocks
        assert abs(per_block[planted].mean().item() - 0.8) < 0.03
        assert per_block[~planted].abs().max().item() < 0.1
    # the planted blocks differ between heads (drawn per head)
    blocks = []
    for h in range(w.H):
        q, k = x["q"][0, h], x["k"][0, h]
        u = q.mean(dim=0) / q.mean(dim=0).norm()
        blocks.append(set(torch.nonzero(((k @ u) / k.norm(dim=-1)).view(tc, w.block)
                                        .mean(dim=1) > 0.5).flatten().tolist()))
    assert blocks[0] != blocks[1]


@pytest.mark.parametrize("w", [W.ALPHA15_4K, W.SPARSEMAX_16K, W.PLANTED_32K,
                               W.long_sweep_point(65536, 1.5)], ids=lambda w: w.name)
def test_benchmark_shapes(w):
    # the shapes the parity tests and bench.py use at full size
    assert (w.B, w.H, w.D) in {(2, 16, 64), (1, 16, 128), (1, 8, 128)}
    assert w.causal and w.block == 128 and w.dtype == "bf16"
