"""Plain float64 reference for alpha-entmax attention (test infrastructure).

Everything here is a direct transcription of the definition, with no blocking,
fusion or reordering beyond chunking rows to bound memory:

* alpha-entmax (the sparse softmax replacement the AdaSplash-2 summaries build
  on -- zh §1, it §1, ja §1, es "Resumen Técnico" §1 -- whose formula the pages
  name but do not print; this is the standard form of Peters, Niculae & Martins
  2019):  p_i = [ s_i - tau ]_+ ** (1/(alpha-1)),  s = (alpha-1) * z,
  with the per-row threshold tau chosen so that sum_i p_i = 1.  tau is kept in
  s-units throughout (the library's convention as well).
* tau is found by plain bisection on f(tau) = sum_i [s_i - tau]_+^k - 1 over the
  bracket [max s - 1, max s - n**(1-alpha)] down to a width of 1e-12.
* Attention: z = q k^T / sqrt(d) (causal: key c visible to query r iff c <= r),
  O = P V.  The bit-packed block mask marks a (row block, key block) pair as
  active iff some probability inside it is non-zero -- zh §2.3, ja §2.3,
  es §2C.  32 blocks per uint32 word, least significant bit = lowest block.
* Backward through the entmax Jacobian  dZ = g * (dP - <g, dP>/<g, 1>) with
  g = p**(2-alpha) on the support and 0 elsewhere; dQ = dZ K / sqrt(d),
  dK = dZ^T Q / sqrt(d), dV = P^T dO.  The summaries only say the backward is
  sparse and skips zero blocks (zh §2.3, it §2C, ja §2.3).
* Histogram threshold tau_h (zh §2.1, it §2A, ja §2.1, es §2A): scores are
  binned into n_bins bins of width h = 1/n_bins on a unit window below the row
  maximum, each bin represented by its lower edge, and the reduced problem
  sum_b c_b [r_b - tau]_+^k = 1 is solved (here by bisection).  Proposition 1
  of the paper, as the summaries state it: tau* - h < tau_h <= tau*.

Parity pins for every function live in tests/test_oracle.py.
"""

from __future__ import annotations

import numpy as np

_MAX_BISECT = 200


def _f64(x):
    return np.asarray(x, dtype=np.float64)


def scores(q, k, causal: bool, rows=None):
    """Scaled logits z = q k^T / sqrt(d) for one head.

    q: [N, D] queries, k: [N_k, D] keys. ``rows`` selects query rows (all if
    None).  Entries a causal query may not see are -inf.
    """
    q = _f64(q)
    k = _f64(k)
    d = q.shape[-1]
    r = np.arange(q.shape[0]) if rows is None else np.asarray(rows, dtype=np.int64)
    z = (q[r] @ k.T) / np.sqrt(d)
    if causal:
        c = np.arange(k.shape[0])
        z = np.where(c[None, :] <= r[:, None], z, -np.inf)
    return z


def _mass(s, tau, k):
    """sum_i [s_i - tau]_+^k per row (-inf entries contribute nothing)."""
    t = np.maximum(s - tau[:, None], 0.0)
    return np.power(t, k).sum(axis=-1)


def entmax_threshold(s, alpha: float, tol: float = 1e-12):
    """tau* per row of s (s-units) by bisection on sum [s - tau]_+^k = 1.

    The bracket [m - 1, m - n**(1 - alpha)] (m = row max, n = number of finite
    entries) always contains the root: at tau = m - 1 the maximum alone
    contributes 1, and at tau = m - n**(1-alpha) even n copies of the maximum
    contribute at most 1.
    """
    s = np.atleast_2d(_f64(s))
    k = 1.0 / (alpha - 1.0)
    n = np.isfinite(s).sum(axis=-1).astype(np.float64)
    m = np.max(s, axis=-1)
    lo = m - 1.0
    hi = m - np.power(n, 1.0 - alpha)
    for _ in range(_MAX_BISECT):
        if np.all(hi - lo <= tol):
            break
        mid = 0.5 * (lo + hi)
        pos = _mass(s, mid, k) - 1.0 > 0.0
        lo = np.where(pos, mid, lo)
        hi = np.where(pos, hi, mid)
    return 0.5 * (lo + hi)


def entmax_probs(s, tau, alpha: float):
    """p = [s - tau]_+ ** (1/(alpha-1)), row-wise."""
    s = np.atleast_2d(_f64(s))
    t = np.maximum(s - _f64(tau)[:, None], 0.0)
    return np.power(t, 1.0 / (alpha - 1.0))


def entmax(z, alpha: float, tol: float = 1e-12):
    """alpha-entmax of logits z (rows).  Returns (p, tau) with tau in s-units."""
    s = (alpha - 1.0) * np.atleast_2d(_f64(z))
    tau = entmax_threshold(s, alpha, tol)
    return entmax_probs(s, tau, alpha), tau


def entmax_jvp(p, v, alpha: float):
    """Jacobian-vector product of entmax w.r.t. its logits z.

    J v = g * (v - <g, v>/<g, 1>), g = p**(2 - alpha) where p > 0, else 0.
    """
    p = np.atleast_2d(_f64(p))
    v = np.atleast_2d(_f64(v))
    supp = p > 0
    g = np.where(supp, np.power(np.where(supp, p, 1.0), 2.0 - alpha), 0.0)
    delta = (g * v).sum(-1, keepdims=True) / g.sum(-1, keepdims=True)
    return g * (v - delta)


def histogram_threshold(s, alpha: float, n_bins: int, anchor: str = "grid",
                        tol: float = 1e-13):
    """tau_h per row from an n_bins histogram of the scores s (s-units).

    Only scores above m - 1 can be in the support (tau* >= m - 1), so a unit
    window below the row maximum m is binned with bin width h = 1/n_bins and
    every bin is represented by its lower edge r_b (so r_b <= s < r_b + h).

    anchor="grid":  bin edges on the absolute grid h*Z; the window holds the
        n_bins + 1 grid bins from floor(n_bins*m) - n_bins up to floor(n_bins*m).
    anchor="max":   the window (m - 1, m] itself is cut into n_bins equal bins
        (u = s - (m - 1) in (0, 1], bin = min(floor(u*n_bins), n_bins - 1)).

    The reduced problem sum_b c_b [r_b - tau]_+^k = 1 over the bin counts c_b is
    solved by bisection on [r_top - 1, r_top] (r_top = highest non-empty edge).
    """
    s = np.atleast_2d(_f64(s))
    k = 1.0 / (alpha - 1.0)
    out = np.empty(s.shape[0])
    for i, row in enumerate(s):
        row = row[np.isfinite(row)]
        m = row.max()
        if anchor == "grid":
            g = np.floor(n_bins * row)
            gmax = np.floor(n_bins * m)
            keep = g >= gmax - n_bins
            idx = (g[keep] - (gmax - n_bins)).astype(np.int64)       # 0..n_bins
            counts = np.bincount(idx, minlength=n_bins + 1).astype(np.float64)
            reps = (gmax - n_bins + np.arange(n_bins + 1)) / n_bins
        elif anchor == "max":
            u = row - (m - 1.0)
            keep = u > 0.0
            idx = np.minimum(np.floor(u[keep] * n_bins), n_bins - 1).astype(np.int64)
            counts = np.bincount(idx, minlength=n_bins).astype(np.float64)
            reps = (m - 1.0) + np.arange(n_bins) / n_bins
        else:
            raise ValueError(f"unknown anchor {anchor!r}")
        r_top = reps[np.nonzero(counts)[0].max()]
        lo, hi = r_top - 1.0, r_top
        for _ in range(_MAX_BISECT):
            if hi - lo <= tol:
                break
            mid = 0.5 * (lo + hi)
            f = (counts * np.power(np.maximum(reps - mid, 0.0), k)).sum() - 1.0
            if f > 0.0:
                lo = mid
            else:
                hi = mid
        out[i] = 0.5 * (lo + hi)
    return out


def pack_block_mask(active):
    """Pack a boolean [Tr, Tc] block map into uint32 [Tr, ceil(Tc/32)] words.

    Bit (j % 32) of word j // 32 is block j; 32 blocks per word (zh §2.3).
    """
    active = np.asarray(active, dtype=bool)
    tr, tc = active.shape
    words = (tc + 31) // 32
    out = np.zeros((tr, words), dtype=np.uint32)
    for j in range(tc):
        out[:, j // 32] |= active[:, j].astype(np.uint32) << np.uint32(j % 32)
    return out


def block_margins(s, tau, row0: int, block: int, n_keys: int):
    """Per (row block, key block) the largest s - tau over its valid entries.

    s: [R, n_keys] scores for rows row0 .. row0+R-1 (row0 a multiple of block);
    returns [ceil(R/block), ceil(n_keys/block)], -inf where a block has no
    valid entry.  A block is active iff its margin is > 0.
    """
    t = _f64(s) - _f64(tau)[:, None]
    nrow = t.shape[0]
    tr = (nrow + block - 1) // block
    tc = (n_keys + block - 1) // block
    pad = np.full((tr * block, tc * block), -np.inf)
    pad[:nrow, :n_keys] = t
    return pad.reshape(tr, block, tc, block).max(axis=(1, 3))


def _chunk_rows(n, block):
    per = max(block, min(1024, (1 << 22) // max(n, 1)))
    return max(block, (per // block) * block)


def attention_forward(q, k, v, alpha: float, causal: bool = True, block: int = 128,
                      rows=None, tol: float = 1e-12):
    """alpha-entmax attention forward for ONE head.

    q, k, v: [N, D].  Returns a dict with
      out  [R, D]     O = P V
      tau  [R]        per-row threshold (s-units)
      rowsum [R]      sum of p (1 up to the bisection tolerance)
      and, when rows is None (all rows):
      margin [Tr, Tc] block margins (max s - tau), mask [Tr, ceil(Tc/32)] uint32.
    ``rows`` restricts the computation to the listed query rows (each is
    independent of the others).
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    n = q.shape[0]
    if rows is not None:
        rows = np.asarray(rows, dtype=np.int64)
        s = (alpha - 1.0) * scores(q, k, causal, rows)
        tau = entmax_threshold(s, alpha, tol)
        p = entmax_probs(s, tau, alpha)
        return {"out": p @ v, "tau": tau, "rowsum": p.sum(-1)}
    tr = (n + block - 1) // block
    tc = (n + block - 1) // block
    out = np.empty_like(q)
    tau_all = np.empty(n)
    rowsum = np.empty(n)
    margin = np.empty((tr, tc))
    step = _chunk_rows(n, block)
    for r0 in range(0, n, step):
        r = np.arange(r0, min(n, r0 + step))
        s = (alpha - 1.0) * scores(q, k, causal, r)
        tau = entmax_threshold(s, alpha, tol)
        p = entmax_probs(s, tau, alpha)
        out[r] = p @ v
        tau_all[r] = tau
        rowsum[r] = p.sum(-1)
        b0 = r0 // block
        mg = block_margins(s, tau, r0, block, n)
        margin[b0:b0 + mg.shape[0]] = mg
    return {"out": out, "tau": tau_all, "rowsum": rowsum, "margin": margin,
            "mask": pack_block_mask(margin > 0.0)}


def attention_backward(q, k, v, dout, alpha: float, causal: bool = True, rows=None,
                       tau=None, tol: float = 1e-12):
    """alpha-entmax attention backward for ONE head.

    Returns (dq, dk, dv).  With ``rows`` given, dq holds those rows only and
    dk/dv hold the contributions of those query rows alone (exact for every key
    column c whose visible rows are all listed, e.g. the last rows under
    causal masking).  ``tau`` (for the same rows) may be passed to skip the
    threshold solve.
    """
    q, k, v, dout = _f64(q), _f64(k), _f64(v), _f64(dout)
    n, d = q.shape
    scale = 1.0 / np.sqrt(d)
    all_rows = np.arange(n) if rows is None else np.asarray(rows, dtype=np.int64)
    dq = np.zeros((all_rows.size, d))
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    step = _chunk_rows(n, 128)
    for c0 in range(0, all_rows.size, step):
        sel = slice(c0, min(all_rows.size, c0 + step))
        r = all_rows[sel]
        s = (alpha - 1.0) * scores(q, k, causal, r)
        t_r = entmax_threshold(s, alpha, tol) if tau is None else _f64(tau)[sel]
        p = entmax_probs(s, t_r, alpha)
        dp = dout[r] @ v.T
        dz = entmax_jvp(p, dp, alpha)
        dq[sel] = (dz @ k) * scale
        dk += (dz.T @ q[r]) * scale
        dv += p.T @ dout[r]
    return dq, dk, dv



def _window_chunk(q, k, v, dout, alpha, causal, block, r, tol, window):
    """attention_windowed's work for the query rows r (one row block or
    more, starting on a block boundary): tau, p and dZ on the window entries,
    their rows of O and dQ, and their contributions to dK and dV."""
    from scipy import sparse

    n, d = q.shape
    scale = 1.0 / np.sqrt(d)
    kend = int(r[-1]) + 1 if causal else n          # keys any row of the chunk sees
    s = (alpha - 1.0) * scores(q, k[:kend], causal, r)
    # per row the maximum of each key block (the last one may be partial)
    nfull = kend // block
    parts = [s[:, :nfull * block].reshape(r.size, nfull, block).max(axis=-1)]
    if kend > nfull * block:
        parts.append(s[:, nfull * block:].max(axis=-1, keepdims=True))
    bmax = np.concatenate(parts, axis=1) if len(parts) > 1 else parts[0]
    m = bmax.max(axis=-1)
    ri, ci = np.nonzero(s > (m - window)[:, None])
    counts = np.bincount(ri, minlength=r.size)
    starts = np.concatenate(([0], np.cumsum(counts)[:-1]))
    pos = np.arange(ri.size) - starts[ri]
    s_win = np.full((r.size, int(counts.max())), -np.inf)
    s_win[ri, pos] = s[ri, ci]
    del s
    tau = entmax_threshold(s_win, alpha, tol)
    p_win = entmax_probs(s_win, tau, alpha)
    # dP = dO V^T on the window entries
    dp_win = np.zeros_like(s_win)
    if ri.size * d < r.size * kend:
        for e0 in range(0, ri.size, 1 << 16):
            sl = slice(e0, min(ri.size, e0 + (1 << 16)))
            dp_win[ri[sl], pos[sl]] = np.einsum("ed,ed->e", dout[r[ri[sl]]], v[ci[sl]])
    else:
        dp_win[ri, pos] = (dout[r] @ v[:kend].T)[ri, ci]
    dz_win = entmax_jvp(p_win, dp_win, alpha)
    pm = sparse.csr_matrix((p_win[ri, pos], (ri, ci)), shape=(r.size, kend))
    zm = sparse.csr_matrix((dz_win[ri, pos], (ri, ci)), shape=(r.size, kend))
    res = {"out": pm @ v[:kend], "rowsum": p_win.sum(axis=-1), "tau": tau,
           "dq": (zm @ k[:kend]) * scale, "dk": (zm.T @ q[r]) * scale, "dv": pm.T @ dout[r],
           "kend": kend, "bm": bmax - tau[:, None]}
    return res


def attention_windowed(q, k, v, dout, alpha: float, causal: bool = True, block: int = 128,
                       rows_per_chunk: int = 0, workers: int = 0, tol: float = 1e-12,
                       _window: float = 1.0):
    """Forward AND backward of ONE head, exactly as attention_forward and
    attention_backward define them, with the threshold solved over the scores
    of the unit window below each row's maximum only.

    Why this is the same computation: tau* >= m - 1 (the lower end of the
    bracket of entmax_threshold; the summaries use the same fact when they map
    the scores into a unit window below the maximum before binning them,
    zh §2.1, it §2A, ja §2.1, es §2A), and every bisection midpoint lies above
    m - 1.  A score s <= m - 1 therefore adds [s - tau]_+^k = 0 at every point
    the bisection evaluates and has p = 0 and g = 0 at tau*: dropping it changes
    neither tau*, nor p, nor dZ = g (dP - delta).  The remaining entries form a
    sparse matrix per row chunk, and O = P V, dQ = dZ K / sqrt(d),
    dK = dZ^T Q / sqrt(d) and dV = P^T dO are sparse-times-dense library
    products over exactly the entries that can be non-zero.  That makes the
    full head affordable at 4K-128K keys, where the dense routines run the
    bisection over all N^2 scores.

    ``_window`` (1, the width the bound gives) exists only so that a test can
    narrow it and check that the pins notice.

    Row chunks are independent; ``workers`` threads (default: the host's
    cores, at most 16) take them in turn and each keeps its own dK / dV sums,
    added at the end.

    Returns a dict with out, tau, rowsum, dq, dk, dv (all rows / keys), the
    block margins [Tr, Tc] (max s - tau over each block, -inf where a block
    has no valid entry) and the packed mask.
    """
    import os
    from concurrent.futures import ThreadPoolExecutor

    q, k, v, dout = _f64(q), _f64(k), _f64(v), _f64(dout)
    n, d = q.shape
    tr = (n + block - 1) // block
    if rows_per_chunk <= 0:
        rows_per_chunk = max(block, min(1024, (1 << 23) // max(n, 1)) // block * block)
    if workers <= 0:
        workers = max(1, min(16, os.cpu_count() or 1))
    chunks = [np.arange(r0, min(n, r0 + rows_per_chunk)) for r0 in range(0, n, rows_per_chunk)]
    out = np.empty((n, d))
    dq = np.empty((n, d))
    tau_all = np.empty(n)
    rowsum = np.empty(n)
    margin = np.full((tr, tr), -np.inf)

    def run(wid):
        dk_w = np.zeros((n, d))
        dv_w = np.zeros((n, d))
        for ci_ in range(wid, len(chunks), workers):
            r = chunks[ci_]
            c = _window_chunk(q, k, v, dout, alpha, causal, block, r, tol, _window)
            out[r] = c["out"]
            dq[r] = c["dq"]
            tau_all[r] = c["tau"]
            rowsum[r] = c["rowsum"]
            dk_w[:c["kend"]] += c["dk"]
            dv_w[:c["kend"]] += c["dv"]
            bm = c["bm"]
            for rb in range(int(r[0]) // block, int(r[-1]) // block + 1):
                sel = (r >= rb * block) & (r < (rb + 1) * block)
                margin[rb, :bm.shape[1]] = bm[sel].max(axis=0)
        return dk_w, dv_w

    with ThreadPoolExecutor(max_workers=workers) as ex:
        parts = list(ex.map(run, range(workers)))
    dk = np.sum([p_[0] for p_ in parts], axis=0)
    dv = np.sum([p_[1] for p_ in parts], axis=0)
    return {"out": out, "tau": tau_all, "rowsum": rowsum, "dq": dq, "dk": dk, "dv": dv,
            "margin": margin, "mask": pack_block_mask(margin > 0.0)}
