"""Plain float64 reference for DashAttention's stage-1 entmax router (test
infrastructure).

The AdaSplash-2 pages include the Italian summary of DashAttention
(gist.science/it/paper/2605.18753), a hierarchical attention that routes each
query to whole chunks of the context with alpha-entmax instead of top-k.  Only
its first two stages are written out here, as the definitions read:

* Stage 0, "Riassunto Locale dei Chunk": the context is cut into contiguous
  chunks of B tokens, and a learned query qbar attends to the keys of each chunk
  with local scaled dot-product attention; the chunk summary is that attention's
  output over the keys.  qbar is initialised to zero, where the attention is
  uniform and the summary is the mean of the chunk's keys.  Only complete
  chunks have a summary (a chunk's summary is fixed once it is complete).
* Stage 1, "Routing dei Chunk con Entmax": per query, logits against the chunk
  summaries, w = alpha-entmax(gamma * zbar).  Readings taken here (the summary
  gives no formula for zbar or the visible set): zbar = q . kbar / sqrt(D) as in
  the attention itself, and query r routes over the complete chunks before its
  own, c < floor(r / B) (its own chunk, which has no summary yet, belongs to
  the separate diagonal branch of stage 2).  A row with no visible chunk routes
  nowhere (all zeros).
* GQA, "Gestione GQA": the routing probabilities of the query heads that share
  a KV head are averaged, giving one shared sparse support per KV head.
* The result is emitted as a bit-packed chunk mask, 32 chunks per uint32, least
  significant bit = lowest chunk, per query row and OR-ed over 128-row query
  blocks (what a stage-2 kernel that walks a bit-packed mask reads).

Stage 2 (prior-induced sparse softmax) and training are not part of this file.
Pins live in tests/test_dash_oracle.py.
"""

from __future__ import annotations

import numpy as np

from .entmax_oracle import entmax, pack_block_mask


def _f64(x):
    return np.asarray(x, dtype=np.float64)


def chunk_summaries(k, chunk: int, qbar=None):
    """Stage 0 for one KV head: k [N, D] -> [N // chunk, D].

    Summary c = softmax(qbar . k_i / sqrt(D) over the chunk's keys i) . k_i,
    the chunk's keys weighted by local attention with query qbar (zero by
    default).  Partial trailing chunks have no summary."""
    k = _f64(k)
    n_chunks = k.shape[0] // chunk
    d = k.shape[1]
    qbar = np.zeros(d) if qbar is None else _f64(qbar)
    out = np.empty((n_chunks, d))
    for c in range(n_chunks):
        kc = k[c * chunk:(c + 1) * chunk]
        logits = kc @ qbar / np.sqrt(d)
        a = np.exp(logits - logits.max())
        a /= a.sum()
        out[c] = a @ kc
    return out


def route_head(q, kbar, alpha: float, gamma: float, chunk: int, rows=None):
    """Stage 1 for one query head: w [len(rows), n_chunks] = alpha-entmax(gamma
    zbar) over the visible chunks c < floor(r / chunk); zero rows where none is
    visible."""
    q = _f64(q)
    kbar = _f64(kbar)
    r = np.arange(q.shape[0]) if rows is None else np.asarray(rows, dtype=np.int64)
    n_chunks = kbar.shape[0]
    zbar = (q[r] @ kbar.T) / np.sqrt(q.shape[1])
    visible = np.arange(n_chunks)[None, :] < (r // chunk)[:, None]
    w = np.zeros((len(r), n_chunks))
    for i in range(len(r)):
        if visible[i].any():
            x = np.where(visible[i], gamma * zbar[i], -np.inf)
            p, _ = entmax(x[None, :], alpha)
            w[i] = np.nan_to_num(p[0], nan=0.0)
    return w


def route(q, k, alpha: float, gamma: float, chunk: int, rows=None, qbar=None):
    """Stage 0 + 1 with GQA averaging for one batch entry.

    q [Hq, N, D], k [Hkv, N, D], Hq a multiple of Hkv (query head h uses KV head
    h // (Hq / Hkv)).  Returns wbar [Hkv, len(rows), n_chunks]: the mean of the
    routing probabilities over each KV head's query heads."""
    q = _f64(q)
    k = _f64(k)
    hq, hkv = q.shape[0], k.shape[0]
    g = hq // hkv
    out = []
    for j in range(hkv):
        kbar = chunk_summaries(k[j], chunk, qbar)
        ws = [route_head(q[j * g + i], kbar, alpha, gamma, chunk, rows) for i in range(g)]
        out.append(np.mean(ws, axis=0))
    return np.stack(out)


def route_masks(wbar, n_rows: int, block: int = 128):
    """Bit-packed chunk masks of one KV head's wbar [n_rows, n_chunks]: per row
    ([n_rows, W]) and OR-ed over `block`-row query blocks ([ceil(n_rows/block), W]),
    W = ceil(n_chunks / 32)."""
    active = np.asarray(wbar) > 0.0
    row_mask = pack_block_mask(active)
    n_blocks = (n_rows + block - 1) // block
    blk = np.zeros((n_blocks, active.shape[1]), dtype=bool)
    for b in range(n_blocks):
        blk[b] = active[b * block:(b + 1) * block].any(axis=0)
    return row_mask, pack_block_mask(blk)
