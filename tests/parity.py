"""Shared comparison helpers for the GPU parity tests (CUDA path vs oracle).

Tolerances, bf16 inputs:
  O, dQ, dK, dV   max-abs <= 2e-2
  tau             |tau - tau*| <= 1e-3 * max(1, |tau*|)
  mask            bit-exact, except blocks whose best margin max(s - tau*)
                  lies within 1e-3 of zero (a tie between tau and the block).
"""

from __future__ import annotations

import numpy as np
import torch

import oracle as O

BF16_TOL = {"out": 2e-2, "grad": 2e-2, "tau_rel": 1e-3, "mask_tie": 1e-3}


def unpack_mask(words: np.ndarray, n_blocks: int) -> np.ndarray:
    """[Tb, W] int32/uint32 words -> [Tb, n_blocks] bool (bit j%32 of word j//32)."""
    w = words.astype(np.int64) & 0xFFFFFFFF
    bits = np.zeros((w.shape[0], n_blocks), dtype=bool)
    for j in range(n_blocks):
        bits[:, j] = (w[:, j // 32] >> (j % 32)) & 1
    return bits


def check_forward_head(res, b, h, q64, k64, v64, alpha, causal, block, tol=BF16_TOL,
                       rows=None):
    """Compare one (b, h) of a FwdResult with the oracle.  Returns a dict of
    the observed errors (and asserts the tolerances)."""
    n = q64.shape[0]
    out = res.out[b, h].float().cpu().numpy()
    tau = res.tau[b, h].cpu().numpy().astype(np.float64)
    if rows is None:
        ref = O.attention_forward(q64, k64, v64, alpha, causal, block)
        err_o = np.abs(out - ref["out"]).max()
        tau_err = (np.abs(tau - ref["tau"]) / np.maximum(1.0, np.abs(ref["tau"]))).max()
        nb = (n + block - 1) // block
        got = unpack_mask(res.mask[b, h].cpu().numpy(), nb)
        want = ref["margin"] > 0
        diff = got != want
        tie = np.abs(ref["margin"]) <= tol["mask_tie"]
        bad = diff & ~tie
        assert not bad.any(), f"mask differs outside the tie band at {np.argwhere(bad)[:5]}"
        mask_diff = int(diff.sum())
    else:
        ref = O.attention_forward(q64, k64, v64, alpha, causal, block, rows=rows)
        err_o = np.abs(out[rows] - ref["out"]).max()
        tau_err = (np.abs(tau[rows] - ref["tau"]) / np.maximum(1.0, np.abs(ref["tau"]))).max()
        mask_diff = None
    assert err_o <= tol["out"], f"O max-abs error {err_o}"
    assert tau_err <= tol["tau_rel"], f"tau relative error {tau_err}"
    return {"err_out": float(err_o), "err_tau": float(tau_err), "mask_diff_in_ties": mask_diff}


def to64(t: torch.Tensor, b: int, h: int) -> np.ndarray:
    return t[b, h].to(torch.float64).cpu().numpy()


def bf16_half_ulp(x: np.ndarray) -> np.ndarray:
    """Half a bf16 unit in the last place at |x| (8 significant bits):
    the rounding error of storing x in bf16."""
    ax = np.maximum(np.abs(x), 2.0 ** -126)
    return np.exp2(np.floor(np.log2(ax)) - 8.0)


def check_grads_head(grads, b, h, q64, k64, v64, do64, alpha, causal, tol=BF16_TOL, rows=None):
    """Compare (dq, dk, dv) of one head with the oracle.  The bar is
    max |gpu - ref| <= tol + (bf16 storage rounding of ref), i.e. 2e-2 beyond
    the unavoidable rounding of the bf16 output itself.  With ``rows`` the
    oracle uses only those query rows: dq is compared on them and dk/dv on the
    key columns c >= rows.min() (causal: exactly the keys those rows see)."""
    dq, dk, dv = (g[b, h].float().cpu().numpy() for g in grads)
    rq, rk, rv = O.attention_backward(q64, k64, v64, do64, alpha, causal, rows=rows)
    out = {}
    if rows is None:
        pairs = (("dq", dq, rq), ("dk", dk, rk), ("dv", dv, rv))
    else:
        c0 = int(np.min(rows))
        pairs = (("dq", dq[rows], rq), ("dk", dk[c0:], rk[c0:]), ("dv", dv[c0:], rv[c0:]))
    for name, got, ref in pairs:
        excess = np.abs(got - ref) - bf16_half_ulp(ref)
        out[name] = {"max_abs": float(np.abs(got - ref).max()), "excess": float(excess.max()),
                     "max_ref": float(np.abs(ref).max())}
        assert excess.max() <= tol["grad"], f"{name}: {out[name]}"
    return out
