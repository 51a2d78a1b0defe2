"""Full-size parity on the benchmark workloads, in the launch configuration
bench.py times (block 128, default max_iter), against the float64 oracle.

For every checked head the oracle's windowed routine (attention_windowed: the
definition, restricted to the scores that can be in a support) gives every
output, so the comparison is element by element over the whole head:

  * O and tau on every query row;
  * the block mask of every row block, bit-exact outside the 1e-3 tie band;
  * dQ on every row, dK and dV on every key -- including the early keys whose
    column kernel accumulates over every later active query tile (1024 of
    them at N = 131072);
  * every head: the device status word flags any row whose probabilities do
    not sum to 1 within 1e-3.

Heads checked: 4K the first and the last of its 32, 16K the first and the
last of its 16, 32K-128K the first.
"""

import numpy as np
import pytest

import oracle as O
from differentiable_sparse_attention_b200 import entmax_attn_bwd, entmax_attn_fwd, status
from differentiable_sparse_attention_b200 import workloads as W
from parity import BF16_TOL, check_full_head, grad_stats, tau_rel_err, to64, unpack_mask

pytestmark = pytest.mark.gpu

POINTS = ([W.ALPHA15_4K.with_(temperature=t) for t in W.ALPHA15_4K_TEMPERATURES]
          + [W.SPARSEMAX_16K, W.PLANTED_32K]
          + [W.long_sweep_point(n, a) for n, a in W.LONG_SWEEP_POINTS]
          # the 4K sweep's sparsest point with a mask of 64 x 64 blocks, where a 128
          # x 128 tile often has only one active 64-wide half
          + [W.ALPHA15_4K.with_(temperature=4.0, block=64, name="alpha1.5_n4096_d64_block64")])


@pytest.mark.parametrize("w", POINTS, ids=[f"{p.name}_t{p.temperature}" for p in POINTS])
def test_full_size_full_head_parity(cuda_device, w):
    x = W.make_inputs(w, device=cuda_device)
    f = entmax_attn_fwd(x["q"], x["k"], x["v"], w.alpha, w.causal, w.block)
    grads = entmax_attn_bwd(x["q"], x["k"], x["v"], x["dout"], f.tau, f.mask, w.alpha,
                            w.causal, w.block, workspace=f.workspace)
    assert status(f.workspace) == 0
    heads = [(0, 0)] if w.N > 16384 else [(0, 0), (w.B - 1, w.H - 1)]
    for b, h in heads:
        q, k, v, do = (to64(x[n], b, h) for n in ("q", "k", "v", "dout"))
        ref = O.attention_windowed(q, k, v, do, w.alpha, w.causal, w.block)
        check_full_head(f, grads, b, h, ref, w.block, label=f"{w.name}_t{w.temperature}")


def test_maximum_n_sampled(cuda_device):
    """N = 262144 (the library's maximum), one head, alpha = 2 at t = 4: O, tau
    and dQ on sampled rows, dK and dV on the last 128 keys (only the last 128
    rows see them), the mask of the first, a middle and the last row block,
    and the status word of every row."""
    w = W.long_sweep_point(262144, 2.0).with_(H=1, name="max_n_262144_alpha2_t4")
    x = W.make_inputs(w, device=cuda_device)
    f = entmax_attn_fwd(x["q"], x["k"], x["v"], w.alpha, w.causal, w.block)
    dq, dk, dv = entmax_attn_bwd(x["q"], x["k"], x["v"], x["dout"], f.tau, f.mask, w.alpha,
                                 w.causal, w.block, workspace=f.workspace)
    assert status(f.workspace) == 0
    q, k, v, do = (to64(x[n], 0, 0) for n in ("q", "k", "v", "dout"))
    rng = np.random.default_rng(262144)
    rows = np.unique(np.concatenate([[0, 1, 127, 128, w.N // 2, w.N - 1],
                                     rng.choice(w.N, 18, replace=False)]))
    ref = O.attention_forward(q, k, v, w.alpha, w.causal, w.block, rows=rows)
    assert np.abs(f.out[0, 0].float().cpu().numpy()[rows] - ref["out"]).max() <= BF16_TOL["out"]
    assert tau_rel_err(f.tau[0, 0].cpu().numpy().astype(np.float64)[rows], ref["tau"]) <= 1e-3
    rq, _, _ = O.attention_backward(q, k, v, do, w.alpha, w.causal, rows=rows, tau=ref["tau"])
    tail = np.arange(w.N - 128, w.N)
    _, rk, rv = O.attention_backward(q, k, v, do, w.alpha, w.causal, rows=tail)
    for name, got, want in (("dq", dq[0, 0].float().cpu().numpy()[rows], rq),
                            ("dk", dk[0, 0].float().cpu().numpy()[tail], rk[tail]),
                            ("dv", dv[0, 0].float().cpu().numpy()[tail], rv[tail])):
        st = grad_stats(got, want)
        assert st["excess"] <= BF16_TOL["grad"], (name, st)
    tb = w.N // w.block
    got_mask = unpack_mask(f.mask[0, 0].cpu().numpy(), tb)
    for rb in (0, tb // 2, tb - 1):
        r = np.arange(rb * w.block, (rb + 1) * w.block)
        s = (w.alpha - 1.0) * O.scores(q, k, w.causal, r)
        t = O.entmax_threshold(s, w.alpha)
        margin = O.block_margins(s, t, rb * w.block, w.block, w.N)[0]
        diff = got_mask[rb] != (margin > 0)
        assert not (diff & (np.abs(margin) > BF16_TOL["mask_tie"])).any(), rb
