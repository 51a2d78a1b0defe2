"""Shared comparison helpers for the GPU parity tests (CUDA path vs oracle).

Tolerances, bf16 inputs:
  O               max-abs <= 2e-2
  dQ, dK, dV      max-abs <= 2e-2 beyond the bf16 half-ulp of the reference
                  value (the rounding of storing it in bf16); the entries above
                  the literal 2e-2 are counted and reported, with their
                  relative error
  tau             |tau - tau*| <= 1e-3 * max(|tau*|, 1e-2): relative, with a
                  floor of 1e-5 s-units where tau* crosses zero (there the
                  error is the fp32 rounding of the scores, not of tau)
  mask            bit-exact, except blocks whose best margin max(s - tau*)
                  lies within 1e-3 of zero (a tie between tau and the block).

Setting the environment variable PARITY_REPORT to a file path makes the
full-head checks append one JSON line per head with the observed errors.
"""

from __future__ import annotations

import json
import os

import numpy as np
import torch

import oracle as O

BF16_TOL = {"out": 2e-2, "grad": 2e-2, "tau_rel": 1e-3, "tau_floor": 1e-2, "mask_tie": 1e-3}


def tau_rel_err(tau, ref, tol=BF16_TOL):
    """max |tau - tau*| / max(|tau*|, floor)."""
    return float((np.abs(tau - ref) / np.maximum(np.abs(ref), tol["tau_floor"])).max())


def grad_stats(got, want, tol=BF16_TOL):
    """Errors of one gradient: max-abs, the excess over the bf16 half-ulp of
    the reference, and the entries beyond the literal tolerance (how many, the
    largest reference magnitude and the largest relative error among them)."""
    err = np.abs(got - want)
    excess = err - bf16_half_ulp(want)
    over = err > tol["grad"]
    rel = err[over] / np.maximum(np.abs(want[over]), 1e-30)
    return {"max_abs": float(err.max()), "excess": float(excess.max()),
            "max_ref": float(np.abs(want).max()), "n": int(err.size),
            "n_over_literal": int(over.sum()),
            "max_rel_over_literal": float(rel.max()) if rel.size else 0.0,
            "min_ref_over_literal": float(np.abs(want[over]).min()) if rel.size else None}


def report(record: dict):
    path = os.environ.get("PARITY_REPORT")
    if path:
        with open(path, "a") as f:
            f.write(json.dumps(record) + "\n")


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
        tau_err = tau_rel_err(tau, ref["tau"], tol)
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
        tau_err = tau_rel_err(tau[rows], ref["tau"], tol)
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
        out[name] = grad_stats(got, ref, tol)
        assert out[name]["excess"] <= tol["grad"], f"{name}: {out[name]}"
    return out


def check_full_head(f, grads, b, h, ref, block, tol=BF16_TOL, label=""):
    """Every output of one (b, h) against attention_windowed's result ``ref``:
    O and tau on every row, the mask of every row block (outside the tie
    band), dQ on every row and dK, dV on every key.  Asserts the tolerances and
    returns (and reports) the observed errors."""
    out = f.out[b, h].float().cpu().numpy()
    tau = f.tau[b, h].cpu().numpy().astype(np.float64)
    n = out.shape[0]
    rec = {"case": label, "b": b, "h": h, "N": n}
    rec["err_out"] = float(np.abs(out - ref["out"]).max())
    rec["err_tau_rel"] = tau_rel_err(tau, ref["tau"], tol)
    nb = (n + block - 1) // block
    got = unpack_mask(f.mask[b, h].cpu().numpy(), nb)
    want = ref["margin"] > 0
    diff = got != want
    tie = np.abs(ref["margin"]) <= tol["mask_tie"]
    rec["mask_blocks"] = int(np.isfinite(ref["margin"]).sum())
    rec["mask_diff_in_ties"] = int((diff & tie).sum())
    rec["mask_diff_outside_ties"] = int((diff & ~tie).sum())
    if grads is not None:
        for name, g, r in zip(("dq", "dk", "dv"), grads, (ref["dq"], ref["dk"], ref["dv"])):
            rec[name] = grad_stats(g[b, h].float().cpu().numpy(), r, tol)
    report(rec)
    assert rec["mask_diff_outside_ties"] == 0, (
        f"mask differs outside the tie band at {np.argwhere(diff & ~tie)[:5]}")
    assert rec["err_out"] <= tol["out"], rec
    assert rec["err_tau_rel"] <= tol["tau_rel"], rec
    if grads is not None:
        for name in ("dq", "dk", "dv"):
            assert rec[name]["excess"] <= tol["grad"], (name, rec[name])
    return rec
