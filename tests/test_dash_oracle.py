"""Pins for the DashAttention stage-0/1 router oracle (oracle/dash_router.py),
each against something other than the oracle itself: closed forms, brute force
and invariants of the definitions in the Italian summary of DashAttention
(gist.science/it/paper/2605.18753, "Stadio 0", "Stadio 1", "Gestione GQA")."""

import numpy as np
import pytest

from oracle import dash_router as R
from oracle import entmax_oracle as O


def test_stage0_zero_query_is_the_chunk_mean():
    rng = np.random.default_rng(0)
    k = rng.standard_normal((70, 8))
    s = R.chunk_summaries(k, 16)
    assert s.shape == (4, 8)                      # the trailing 6 keys: no summary
    for c in range(4):
        assert np.allclose(s[c], k[16 * c:16 * (c + 1)].mean(axis=0), atol=1e-14)


def test_stage0_learned_query_brute_force():
    # qbar != 0: softmax weights written out by hand for a 3-key chunk
    k = np.array([[1.0, 0.0], [0.0, 2.0], [1.0, 1.0]])
    qbar = np.array([0.5, -1.0])
    logits = np.array([0.5, -2.0, -0.5]) / np.sqrt(2.0)
    a = np.exp(logits) / np.exp(logits).sum()
    assert np.allclose(R.chunk_summaries(k, 3, qbar)[0], a @ k, atol=1e-14)


def test_stage1_two_chunks_sparsemax_closed_form():
    # alpha = 2 over two visible chunks: p1 = clip((x1 - x2 + 1) / 2, 0, 1)
    rng = np.random.default_rng(1)
    q = rng.standard_normal((40, 4))
    kbar = rng.standard_normal((2, 4))
    gamma = 0.7
    w = R.route_head(q, kbar, 2.0, gamma, chunk=16)
    x = gamma * (q @ kbar.T) / 2.0
    for r in range(40):
        if r < 16:
            assert not w[r].any()                 # no complete chunk before the row
        elif r < 32:
            assert w[r, 0] == pytest.approx(1.0) and w[r, 1] == 0.0   # only chunk 0
        else:
            p1 = np.clip((x[r, 0] - x[r, 1] + 1.0) / 2.0, 0.0, 1.0)
            assert w[r, 0] == pytest.approx(p1, abs=1e-10)
            assert w[r, 1] == pytest.approx(1.0 - p1, abs=1e-10)


@pytest.mark.parametrize("alpha", [1.5, 2.0, 1.25])
def test_stage1_matches_entmax_of_the_visible_logits(alpha):
    rng = np.random.default_rng(2)
    q = rng.standard_normal((200, 8))
    kbar = rng.standard_normal((12, 8))
    w = R.route_head(q, kbar, alpha, 2.0, chunk=16)
    for r in (16, 47, 100, 199):
        nvis = min(r // 16, 12)
        x = 2.0 * (q[r] @ kbar[:nvis].T) / np.sqrt(8)
        # exact for alpha = 1.5: the sorted closed form; otherwise entmax itself
        p, _ = O.entmax(x[None, :], alpha)
        assert np.allclose(w[r, :nvis], p[0], atol=1e-10)
        assert not w[r, nvis:].any()
        assert w[r].sum() == pytest.approx(1.0, abs=1e-10)


def test_stage1_causality_of_the_routing():
    # changing keys in the row's own chunk or later ones leaves the row unchanged
    rng = np.random.default_rng(3)
    q = rng.standard_normal((3, 128, 8))
    k = rng.standard_normal((1, 128, 8))
    w0 = R.route(q, k, 1.5, 1.0, chunk=16, rows=np.array([70]))
    k2 = k.copy()
    k2[0, 64:] = rng.standard_normal((64, 8))     # chunks 4.. (row 70 is in chunk 4)
    w1 = R.route(q, k2, 1.5, 1.0, chunk=16, rows=np.array([70]))
    assert np.array_equal(w0, w1)


def test_gqa_average_support_is_the_union_and_sums_to_one():
    rng = np.random.default_rng(4)
    q = 3.0 * rng.standard_normal((4, 96, 8))     # 4 query heads
    k = rng.standard_normal((2, 96, 8))           # 2 KV heads: groups of 2
    wbar = R.route(q, k, 1.5, 1.0, chunk=8)
    for j in range(2):
        kbar = R.chunk_summaries(k[j], 8)
        wa = R.route_head(q[2 * j], kbar, 1.5, 1.0, 8)
        wb = R.route_head(q[2 * j + 1], kbar, 1.5, 1.0, 8)
        assert np.allclose(wbar[j], 0.5 * (wa + wb), atol=1e-14)
        assert np.array_equal(wbar[j] > 0, (wa > 0) | (wb > 0))
        sums = wbar[j].sum(axis=1)
        assert np.allclose(sums[8:], 1.0, atol=1e-10) and not sums[:8].any()


def test_route_masks_bit_order_and_block_or():
    w = np.zeros((130, 40))
    w[0, 0] = 0.5
    w[5, 33] = 1.0
    w[129, 39] = 0.1
    row, blk = R.route_masks(w, 130, block=128)
    assert row.shape == (130, 2) and blk.shape == (2, 2)
    assert row[0, 0] == 1 and row[5, 1] == 2 and row[129, 1] == 1 << 7
    assert blk[0, 0] == 1 and blk[0, 1] == 2 and blk[1, 1] == 1 << 7 and blk[1, 0] == 0
