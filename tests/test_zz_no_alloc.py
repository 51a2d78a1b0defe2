"""entmax_attn_fwd_noalloc, the forward for callers that cannot allocate
device memory when they call it, checked through the C ABI against the regular
entmax_attn_fwd and against the float64 oracle, with its status word read
through entmax_attn_noalloc_status.

Such callers (code running where cudaMalloc is unavailable or must not be
used) get a variant whose scratch lives in a fixed 8 MiB array inside the
library instead of a caller-provided workspace.  This file is named so that
pytest collects it last: a run that stops at the first failure has then
already run every other test.
"""

import ctypes

import numpy as np
import pytest
import torch

import differentiable_sparse_attention_b200 as dsa
import oracle as O
from differentiable_sparse_attention_b200.workloads import Workload, make_inputs
from parity import BF16_TOL, tau_rel_err, to64, unpack_mask

pytestmark = pytest.mark.gpu


def _call_noalloc(w, x, out, tau, mask, max_iter=4):
    lib = dsa._lib()
    stream = torch.cuda.current_stream(x["q"].device).cuda_stream
    return lib.entmax_attn_fwd_noalloc(
        ctypes.c_void_p(x["q"].data_ptr()), ctypes.c_void_p(x["k"].data_ptr()),
        ctypes.c_void_p(x["v"].data_ptr()), w.B, w.H, w.N, w.D, 0, float(w.alpha),
        int(w.causal), w.block, max_iter, ctypes.c_void_p(out.data_ptr()),
        ctypes.c_void_p(tau.data_ptr()), ctypes.c_void_p(mask.data_ptr()),
        ctypes.c_void_p(stream))


def test_noalloc_matches_regular_forward_two_calls_in_a_row(cuda_device):
    # Two calls in a row; the second finds the first call's leftovers in the
    # shared scratch array (and needs more of it).
    cases = [
        Workload("noalloc_a", B=1, H=2, N=512, D=64, alpha=1.5, temperature=2.0, seed=21),
        Workload("noalloc_b", B=2, H=4, N=1000, D=128, alpha=2.0, block=64, temperature=3.0,
                 seed=22),
    ]
    for w in cases:
        x = make_inputs(w, device=cuda_device, need_grad_inputs=False)
        ref = dsa.entmax_attn_fwd(x["q"], x["k"], x["v"], w.alpha, w.causal, w.block, max_iter=4)
        out = torch.full_like(x["q"], float("nan"))
        tau = torch.full((w.B, w.H, w.N), float("nan"), device=cuda_device)
        mask = torch.full_like(ref.mask, -1)
        rc = _call_noalloc(w, x, out, tau, mask)
        assert rc == dsa.OK, dsa.error_string(rc)
        torch.cuda.synchronize(cuda_device)
        assert (out.float() - ref.out.float()).abs().max().item() <= 2e-2
        rel = ((tau - ref.tau).abs() / ref.tau.abs().clamp_min(1.0)).max().item()
        assert rel <= 1e-3
        assert torch.equal(mask, ref.mask)
        assert dsa.noalloc_status(cuda_device) == 0


def test_noalloc_matches_the_oracle(cuda_device):
    # the no-alloc forward on its own, element by element against the float64
    # oracle: O within 2e-2, tau within 1e-3 relative, the mask outside the tie band
    w = Workload("noalloc_oracle", B=1, H=2, N=700, D=128, alpha=1.5, block=64,
                 temperature=2.0, seed=24)
    x = make_inputs(w, device=cuda_device, need_grad_inputs=False)
    out = torch.empty_like(x["q"])
    tau = torch.empty((w.B, w.H, w.N), device=cuda_device)
    nb = (w.N + w.block - 1) // w.block
    mask = torch.empty((w.B, w.H, nb, dsa.mask_words(w.N, w.block)), dtype=torch.int32,
                       device=cuda_device)
    assert _call_noalloc(w, x, out, tau, mask) == dsa.OK
    assert dsa.noalloc_status(cuda_device) == 0
    for h in range(w.H):
        q, k, v = (to64(x[n], 0, h) for n in ("q", "k", "v"))
        ref = O.attention_forward(q, k, v, w.alpha, w.causal, w.block)
        assert np.abs(out[0, h].float().cpu().numpy() - ref["out"]).max() <= BF16_TOL["out"]
        assert tau_rel_err(tau[0, h].cpu().numpy().astype(np.float64), ref["tau"]) <= 1e-3
        diff = unpack_mask(mask[0, h].cpu().numpy(), nb) != (ref["margin"] > 0)
        assert not (diff & (np.abs(ref["margin"]) > BF16_TOL["mask_tie"])).any()


def test_noalloc_status_reports_a_row_that_did_not_converge(cuda_device):
    # max_iter = 0 stops at the histogram bound tau_h < tau*, so rows sum above 1
    w = Workload("noalloc_status", B=1, H=1, N=512, D=64, alpha=1.5, temperature=2.0, seed=25)
    x = make_inputs(w, device=cuda_device, need_grad_inputs=False)
    out = torch.empty_like(x["q"])
    tau = torch.empty((w.B, w.H, w.N), device=cuda_device)
    mask = torch.empty((w.B, w.H, w.N // 128, dsa.mask_words(w.N, 128)), dtype=torch.int32,
                       device=cuda_device)
    assert _call_noalloc(w, x, out, tau, mask, max_iter=0) == dsa.OK
    assert dsa.noalloc_status(cuda_device) & dsa.ST_NOT_CONVERGED
    # the next call clears the word again
    assert _call_noalloc(w, x, out, tau, mask, max_iter=4) == dsa.OK
    assert dsa.noalloc_status(cuda_device) == 0


def test_noalloc_rejects_problems_beyond_its_scratch(cuda_device):
    # B*H = 16 heads at N = 16384 need ~34 MB of tile maxima > 8 MiB.
    w = Workload("too_big", B=1, H=16, N=16384, D=64, alpha=1.5, seed=23)
    x = make_inputs(w, device=cuda_device, need_grad_inputs=False)
    out = torch.zeros_like(x["q"])
    tau = torch.zeros((w.B, w.H, w.N), device=cuda_device)
    mask = torch.zeros((w.B, w.H, w.N // 128, dsa.mask_words(w.N, 128)), dtype=torch.int32,
                       device=cuda_device)
    rc = _call_noalloc(w, x, out, tau, mask)
    assert rc == dsa.E_SCRATCH
    torch.cuda.synchronize(cuda_device)
    assert torch.count_nonzero(out).item() == 0 and torch.count_nonzero(tau).item() == 0
