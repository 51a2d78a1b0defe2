"""Failure handling on the GPU without a fault: every mbarrier wait in the
kernels is bounded, and a wait that runs out raises ENTMAX_ST_TIMEOUT, sets
the CTA's abort flag and lets the kernel return.  The self-test entry point
waits on a barrier that nothing arrives at, with a 5 ms limit; the test then
checks the status word and that the context still runs a forward."""

import ctypes

import pytest
import torch

import differentiable_sparse_attention_b200 as dsa
from differentiable_sparse_attention_b200.workloads import Workload, make_inputs

pytestmark = pytest.mark.gpu


def test_bounded_wait_runs_out_and_reports(cuda_device):
    ws = torch.zeros(256, dtype=torch.uint8, device=cuda_device)
    result = torch.full((3,), 7, dtype=torch.int32, device=cuda_device)
    stream = torch.cuda.current_stream(cuda_device).cuda_stream
    rc = dsa._lib().entmax_attn_wait_selftest(ctypes.c_void_p(ws.data_ptr()),
                                              ctypes.c_void_p(result.data_ptr()),
                                              5_000_000, ctypes.c_void_p(stream))
    assert rc == dsa.OK
    st = dsa.status(ws)
    assert st & dsa.ST_TIMEOUT
    assert result.cpu().tolist() == [1, 0, 1]   # returned; the wait failed; abort raised
    # the context is intact: a forward right after runs and reports nothing
    w = Workload("after_timeout", B=1, H=1, N=256, D=64, alpha=1.5, seed=3)
    x = make_inputs(w, device=cuda_device, need_grad_inputs=False)
    f = dsa.entmax_attn_fwd(x["q"], x["k"], x["v"], 1.5, True, 128)
    assert dsa.status(f.workspace) == 0
    assert torch.isfinite(f.out.float()).all()
