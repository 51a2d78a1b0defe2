"""Full-size parity on the benchmark workloads, in the launch configuration
bench.py times (block 128, default max_iter), against the float64 oracle on
sampled outputs:

  * O, tau and dQ on sampled query rows (first, last, tile boundaries, random);
  * dK and dV on the last key rows, which under causal masking only the last
    query rows see, so the oracle computes them exactly from those rows;
  * the block mask of the first and the last row block (every row of the
    block), bit-exact outside the 1e-3 tie band;
  * every row: the device status word flags any row whose probabilities do not
    sum to 1 within 1e-3.
"""

import numpy as np
import pytest
import torch

import oracle as O
from differentiable_sparse_attention_b200 import entmax_attn_bwd, entmax_attn_fwd, status
from differentiable_sparse_attention_b200 import workloads as W
from parity import BF16_TOL, bf16_half_ulp, to64, unpack_mask

pytestmark = pytest.mark.gpu

POINTS = ([W.ALPHA15_4K.with_(temperature=t) for t in W.ALPHA15_4K_TEMPERATURES]
          + [W.SPARSEMAX_16K, W.PLANTED_32K]
          + [W.long_sweep_point(n, a) for n, a in W.LONG_SWEEP_POINTS])


def sample_rows(n, k, rng):
    fixed = [0, 1, 127, 128, 129, n // 2, n - 129, n - 128, n - 1]
    rnd = rng.choice(n, size=k, replace=False)
    return np.unique(np.clip(np.concatenate([fixed, rnd]), 0, n - 1))


@pytest.mark.parametrize("w", POINTS, ids=[f"{p.name}_t{p.temperature}" for p in POINTS])
def test_full_size_sampled_parity(cuda_device, w):
    big = w.N >= 65536
    x = W.make_inputs(w, device=cuda_device)
    f = entmax_attn_fwd(x["q"], x["k"], x["v"], w.alpha, w.causal, w.block)
    dq, dk, dv = entmax_attn_bwd(x["q"], x["k"], x["v"], x["dout"], f.tau, f.mask, w.alpha,
                                 w.causal, w.block, workspace=f.workspace)
    assert status(f.workspace) == 0
    rng = np.random.default_rng(w.N + int(10 * w.temperature))
    heads = [(0, 0)] if big else [(0, 0), (w.B - 1, w.H - 1)]
    for b, h in heads:
        q, k, v, do = (to64(x[n], b, h) for n in ("q", "k", "v", "dout"))
        rows = sample_rows(w.N, 16 if big else 40, rng)
        ref = O.attention_forward(q, k, v, w.alpha, w.causal, w.block, rows=rows)
        out = f.out[b, h].float().cpu().numpy()[rows]
        tau = f.tau[b, h].cpu().numpy().astype(np.float64)[rows]
        assert np.abs(out - ref["out"]).max() <= BF16_TOL["out"]
        assert (np.abs(tau - ref["tau"]) / np.maximum(1, np.abs(ref["tau"]))).max() <= 1e-3
        # dQ on the sampled rows; dK / dV on the keys only the tail rows see
        tail = np.arange(w.N - (64 if big else 256), w.N)
        rq, _, _ = O.attention_backward(q, k, v, do, w.alpha, w.causal, rows=rows,
                                        tau=ref["tau"])
        _, rk, rv = O.attention_backward(q, k, v, do, w.alpha, w.causal, rows=tail)
        c0 = tail[0]
        for name, got, want in (("dq", dq[b, h].float().cpu().numpy()[rows], rq),
                                ("dk", dk[b, h].float().cpu().numpy()[c0:], rk[c0:]),
                                ("dv", dv[b, h].float().cpu().numpy()[c0:], rv[c0:])):
            excess = (np.abs(got - want) - bf16_half_ulp(want)).max()
            assert excess <= BF16_TOL["grad"], (name, excess, np.abs(want).max())
        # block mask of the first and the last row block, all rows of each
        tb = (w.N + w.block - 1) // w.block
        got_mask = unpack_mask(f.mask[b, h].cpu().numpy(), tb)
        for rb in (0, tb - 1):
            r = np.arange(rb * w.block, min(w.N, (rb + 1) * w.block))
            s = (w.alpha - 1.0) * O.scores(q, k, w.causal, r)
            t = O.entmax_threshold(s, w.alpha)
            margin = O.block_margins(s, t, rb * w.block, w.block, w.N)[0]
            diff = got_mask[rb] != (margin > 0)
            assert not (diff & (np.abs(margin) > BF16_TOL["mask_tie"])).any()
