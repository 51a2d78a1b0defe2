"""DashAttention stage-0/1 router: the CUDA path (through the C ABI) against the
float64 oracle in oracle/dash_router.py, on seeded synthetic queries and keys.

The kernel reads q and k in bf16 (q as an exact fp16 copy), rounds the chunk
means to fp16 and forms the logits in fp32, so wbar is compared to 2e-3 and the
masks bit by bit except where some query head's score margin s - tau* of that
chunk lies within the 1e-3 tie band."""

import numpy as np
import pytest
import torch

import oracle as O
from oracle import dash_router as R
from differentiable_sparse_attention_b200 import dash_route, status
from parity import unpack_mask

pytestmark = pytest.mark.gpu

W_TOL = 2e-3
TIE = 1e-3


def inputs(B, Hq, Hkv, N, D, seed, device):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn((B, Hq, N, D), generator=g).to(torch.bfloat16)
    k = torch.randn((B, Hkv, N, D), generator=g).to(torch.bfloat16)
    return q, k, q.to(device), k.to(device)


def margins(q64, kbar, alpha, gamma, chunk, rows):
    """s - tau* per (row, chunk) for one query head (nan where not visible)."""
    z = gamma * (q64[rows] @ kbar.T) / np.sqrt(q64.shape[1])
    out = np.full(z.shape, np.nan)
    for i, r in enumerate(rows):
        nvis = min(r // chunk, kbar.shape[0])
        if nvis:
            s = (alpha - 1.0) * z[i, :nvis]
            out[i, :nvis] = s - O.entmax_threshold(s[None, :], alpha)[0]
    return out


def check(res, qc, kc, alpha, gamma, chunk, rows):
    B, Hq, N, D = qc.shape
    Hkv = kc.shape[1]
    G = Hq // Hkv
    C = N // chunk
    wb = res.wbar.cpu().numpy()
    rm = res.row_mask.cpu().numpy()
    bm = res.block_mask.cpu().numpy()
    for b in range(B):
        q64 = qc[b].double().numpy()
        k64 = kc[b].double().numpy()
        ref = R.route(q64, k64, alpha, gamma, chunk, rows=rows)
        for j in range(Hkv):
            assert np.abs(wb[b, j][rows] - ref[j]).max() <= W_TOL
            got_bits = unpack_mask(rm[b, j][rows], C)
            want_bits = ref[j] > 0
            kbar = R.chunk_summaries(k64[j], chunk)
            tie = np.zeros_like(want_bits)
            for g in range(G):
                m = margins(q64[j * G + g], kbar, alpha, gamma, chunk, rows)
                tie |= np.nan_to_num(np.abs(m), nan=1.0) <= TIE
            assert not ((got_bits != want_bits) & ~tie).any()
            # the block mask is the OR of the row mask over each 128-row block
            all_bits = unpack_mask(rm[b, j], C)
            for t in range((N + 127) // 128):
                assert np.array_equal(unpack_mask(bm[b, j, t:t + 1], C)[0],
                                      all_bits[t * 128:(t + 1) * 128].any(axis=0))


CASES = [
    # name, B, Hq, Hkv, N, D, chunk, alpha, gamma
    ("g2_n300_d64_c16_a15", 1, 4, 2, 300, 64, 16, 1.5, 8.0),
    ("g1_b2_n512_d128_c32_a2", 2, 2, 2, 512, 128, 32, 2.0, 6.0),
    ("g4_n1000_d64_c8_a175", 1, 8, 2, 1000, 64, 8, 1.75, 8.0),
    ("g2_n640_d128_c5_a125_ragged", 1, 2, 1, 640, 128, 5, 1.25, 10.0),
]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_router_matches_oracle(cuda_device, case):
    name, B, Hq, Hkv, N, D, chunk, alpha, gamma = case
    qc, kc, q, k = inputs(B, Hq, Hkv, N, D, 41, cuda_device)
    res = dash_route(q, k, chunk, gamma, alpha)
    assert status(res.workspace) == 0
    check(res, qc, kc, alpha, gamma, chunk, np.arange(N))


def test_router_16k_sampled(cuda_device):
    # B=1, 8 query heads over 2 KV heads, N=16384, D=128, chunks of 64 (256 chunks)
    qc, kc, q, k = inputs(1, 8, 2, 16384, 128, 42, cuda_device)
    res = dash_route(q, k, 64, 16.0, 1.5)
    assert status(res.workspace) == 0
    rng = np.random.default_rng(3)
    rows = np.unique(np.concatenate([[0, 63, 64, 127, 128, 8191, 16383],
                                     rng.choice(16384, 40, replace=False)]))
    B, Hq, N, D = qc.shape
    wb = res.wbar.cpu().numpy()
    ref = R.route(qc[0].double().numpy(), kc[0].double().numpy(), 1.5, 16.0, 64, rows=rows)
    assert np.abs(wb[0][:, rows] - ref).max() <= W_TOL
    # every visible row sums to 1
    sums = wb[0].sum(axis=-1)
    assert np.abs(sums[:, 64:] - 1.0).max() <= 1e-3 and not sums[:, :64].any()


def test_router_no_complete_chunk(cuda_device):
    _, _, q, k = inputs(1, 2, 1, 40, 64, 43, cuda_device)
    res = dash_route(q, k, 64, 4.0, 1.5)
    assert res.wbar.shape == (1, 1, 40, 0) and res.row_mask.shape == (1, 1, 40, 0)
