"""Generic alpha: any alpha in [1.05, 3] besides the closed forms of 1.5 and 2.
The kernels form p = t^k and g = p^(2 - alpha) = t^(k - 1), k = 1 / (alpha - 1),
with the special-function unit, refine tau with Halley steps (alpha <= 1.5) or
Newton steps, safeguarded by bisection (AdaSplash-2 zh §2.2, it §2B, ja §2.2,
es §2B).  Gradients exist for alpha <= 2 only (beyond, g is unbounded at the
edge of the support), so the alpha > 2 cases check the forward.  Forward and backward are
compared with the float64 oracle, element by element, through the C ABI."""

import numpy as np
import pytest
import torch

import oracle as O
from differentiable_sparse_attention_b200 import entmax_attn_bwd, entmax_attn_fwd, status
from differentiable_sparse_attention_b200.workloads import Workload, make_inputs
from parity import BF16_TOL, bf16_half_ulp, check_forward_head, check_grads_head, tau_rel_err, to64

pytestmark = pytest.mark.gpu

CASES = [
    # name, B, H, N, D, alpha, causal, block, temperature
    ("a125_n300_d64_ragged", 1, 2, 300, 64, 1.25, True, 128, 1.0),     # Halley (k = 4)
    ("a13_n520_d128_t3_b64", 1, 1, 520, 128, 1.3, True, 64, 3.0),      # Halley
    ("a175_n384_d128_noncausal", 1, 1, 384, 128, 1.75, False, 128, 2.0),  # Newton
    ("a25_n200_d64_t4", 1, 1, 200, 64, 2.5, True, 128, 4.0),           # Newton (k = 2/3)
    ("a3_n256_d64_b64", 1, 2, 256, 64, 3.0, True, 64, 2.0),            # Newton (k = 1/2)
]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_generic_alpha_forward_backward(cuda_device, case):
    name, B, H, N, D, alpha, causal, block, temp = case
    w = Workload(name, B=B, H=H, N=N, D=D, alpha=alpha, causal=causal, block=block,
                 temperature=temp, seed=31)
    x = make_inputs(w, device=cuda_device)
    f = entmax_attn_fwd(x["q"], x["k"], x["v"], alpha, causal, block, max_iter=12)
    assert status(f.workspace) == 0
    grads = None
    if alpha <= 2.0:
        grads = entmax_attn_bwd(x["q"], x["k"], x["v"], x["dout"], f.tau, f.mask, alpha,
                                causal, block, workspace=f.workspace)
        assert status(f.workspace) == 0
    for b in range(B):
        for h in range(H):
            q, k, v, do = (to64(x[n], b, h) for n in ("q", "k", "v", "dout"))
            check_forward_head(f, b, h, q, k, v, alpha, causal, block)
            if grads is not None:
                check_grads_head(grads, b, h, q, k, v, do, alpha, causal)


def test_generic_alpha_4k_sampled(cuda_device):
    # B=1 H=4 N=4096 D=64 alpha=1.75 t=2: sampled rows of O, tau and dQ, and the
    # keys that only the tail rows see for dK / dV
    w = Workload("a175_n4096", B=1, H=4, N=4096, D=64, alpha=1.75, temperature=2.0, seed=32)
    x = make_inputs(w, device=cuda_device)
    f = entmax_attn_fwd(x["q"], x["k"], x["v"], w.alpha, True, 128, max_iter=12)
    dq, dk, dv = entmax_attn_bwd(x["q"], x["k"], x["v"], x["dout"], f.tau, f.mask, w.alpha,
                                 True, 128, workspace=f.workspace)
    assert status(f.workspace) == 0
    rng = np.random.default_rng(5)
    rows = np.unique(np.concatenate([[0, 127, 128, 2047, 4095], rng.choice(4096, 24, False)]))
    h = 3
    q, k, v, do = (to64(x[n], 0, h) for n in ("q", "k", "v", "dout"))
    ref = O.attention_forward(q, k, v, w.alpha, True, 128, rows=rows)
    assert np.abs(f.out[0, h].float().cpu().numpy()[rows] - ref["out"]).max() <= BF16_TOL["out"]
    tau = f.tau[0, h].cpu().numpy().astype(np.float64)[rows]
    assert tau_rel_err(tau, ref["tau"]) <= 1e-3
    rq, _, _ = O.attention_backward(q, k, v, do, w.alpha, True, rows=rows, tau=ref["tau"])
    tail = np.arange(4096 - 128, 4096)
    _, rk, rv = O.attention_backward(q, k, v, do, w.alpha, True, rows=tail)
    for name, got, want in (("dq", dq[0, h].float().cpu().numpy()[rows], rq),
                            ("dk", dk[0, h].float().cpu().numpy()[tail[0]:], rk[tail[0]:]),
                            ("dv", dv[0, h].float().cpu().numpy()[tail[0]:], rv[tail[0]:])):
        excess = (np.abs(got - want) - bf16_half_ulp(want)).max()
        assert excess <= BF16_TOL["grad"], (name, excess)
