"""fp32 path parity (CUDA-core kernels): the tiny fp32 workload and variants,
at the fp32 tolerances -- max-abs 1e-5 on O, 1e-4 on dQ/dK/dV, 1e-3 relative
on tau, block mask bit-exact outside the 1e-3 tie band."""

import numpy as np
import pytest

import oracle as O
from differentiable_sparse_attention_b200 import entmax_attn_bwd, entmax_attn_fwd, status
from differentiable_sparse_attention_b200.workloads import TINY_FP32, Workload, make_inputs
from parity import tau_rel_err, to64, unpack_mask

pytestmark = pytest.mark.gpu

FP32_TOL = {"out": 1e-5, "grad": 1e-4, "tau_rel": 1e-3, "mask_tie": 1e-3}

CASES = [
    TINY_FP32,
    TINY_FP32.with_(name="tiny_fp32_alpha2", alpha=2.0),
    TINY_FP32.with_(name="tiny_fp32_ragged_t3", N=300, temperature=3.0, block=128, seed=2),
    TINY_FP32.with_(name="tiny_fp32_noncausal", causal=False, N=200, seed=3),
    TINY_FP32.with_(name="tiny_fp32_n1", N=1, H=1),
    TINY_FP32.with_(name="fp32_n1024_t2", N=1024, H=2, temperature=2.0, seed=4),
]


@pytest.mark.parametrize("w", CASES, ids=[c.name for c in CASES])
def test_fp32_forward_backward(cuda_device, w):
    x = make_inputs(w, device=cuda_device)
    f = entmax_attn_fwd(x["q"], x["k"], x["v"], w.alpha, w.causal, w.block)
    dq, dk, dv = entmax_attn_bwd(x["q"], x["k"], x["v"], x["dout"], f.tau, f.mask, w.alpha,
                                 w.causal, w.block, workspace=f.workspace)
    assert status(f.workspace) == 0
    for b in range(w.B):
        for h in range(w.H):
            q, k, v, do = (to64(x[n], b, h) for n in ("q", "k", "v", "dout"))
            ref = O.attention_forward(q, k, v, w.alpha, w.causal, w.block)
            assert np.abs(f.out[b, h].cpu().numpy() - ref["out"]).max() <= FP32_TOL["out"]
            tau = f.tau[b, h].cpu().numpy().astype(np.float64)
            assert tau_rel_err(tau, ref["tau"]) <= 1e-3
            nb = (w.N + w.block - 1) // w.block
            diff = unpack_mask(f.mask[b, h].cpu().numpy(), nb) != (ref["margin"] > 0)
            assert not (diff & (np.abs(ref["margin"]) > FP32_TOL["mask_tie"])).any()
            rq, rk, rv = O.attention_backward(q, k, v, do, w.alpha, w.causal, tau=ref["tau"])
            for name, got, want in (("dq", dq, rq), ("dk", dk, rk), ("dv", dv, rv)):
                err = np.abs(got[b, h].cpu().numpy() - want).max()
                assert err <= FP32_TOL["grad"], (name, err)
