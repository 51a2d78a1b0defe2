"""The comparison helpers of the GPU parity tests (tests/parity.py), on CPU.

A helper that compared the wrong bits or applied a loose bound would let a
wrong GPU result pass.  Each helper is checked against an independent fact:
- the mask unpacking inverts the oracle's packing;
- the bf16 half-ulp is the largest rounding error torch's bf16 cast makes;
- the forward and gradient checks accept the oracle's own results, stored as
  the GPU stores them, and reject them once an error is planted.
Here the "GPU result" is built on the CPU.
"""

from types import SimpleNamespace

import numpy as np
import pytest
import torch

import oracle as O
from parity import bf16_half_ulp, check_forward_head, check_grads_head, unpack_mask


def test_unpack_inverts_the_oracle_packing():
    rng = np.random.default_rng(0)
    for tr, tc in ((1, 1), (3, 31), (4, 32), (2, 33), (5, 70)):
        active = rng.random((tr, tc)) < 0.5
        active[:, -1] = True                       # the highest bit of the last word
        words = O.pack_block_mask(active)
        assert np.array_equal(unpack_mask(words, tc), active)
        # the library's int32 view of the same bits
        assert np.array_equal(unpack_mask(words.view(np.int32), tc), active)


def test_bf16_half_ulp_bounds_the_cast():
    rng = np.random.default_rng(1)
    x = np.concatenate([rng.normal(size=20000) * 10.0 ** rng.integers(-6, 4, 20000),
                        [1.0, 1.5, 2.0 - 2.0 ** -9, 3.0, 1e-3]])
    stored = torch.from_numpy(x).to(torch.bfloat16).double().numpy()
    err = np.abs(stored - x)
    bound = bf16_half_ulp(x)
    assert np.all(err <= bound * (1 + 1e-12))
    # and it is tight: some values are rounded by nearly the full half ulp
    assert np.max(err / bound) > 0.99


def _head(n=200, d=16, seed=3, alpha=1.5):
    g = torch.Generator().manual_seed(seed)
    q, k, v, do = (torch.randn((n, d), generator=g, dtype=torch.float64) for _ in range(4))
    return q.numpy(), k.numpy(), v.numpy(), do.numpy()


def _as_gpu_forward(ref, n, block):
    # what the library returns for one (b, h) = (0, 0): bf16 O, fp32 tau, int32 mask
    out = torch.from_numpy(ref["out"]).to(torch.bfloat16)[None, None]
    tau = torch.from_numpy(ref["tau"]).to(torch.float32)[None, None]
    mask = torch.from_numpy(ref["mask"].view(np.int32).copy())[None, None]
    return SimpleNamespace(out=out, tau=tau, mask=mask)


@pytest.mark.parametrize("alpha", [1.5, 2.0])
def test_forward_check_accepts_exact_and_rejects_planted_errors(alpha):
    n, block = 200, 64
    q, k, v, _ = _head(n, alpha=alpha)
    ref = O.attention_forward(q, k, v, alpha, True, block)
    res = _as_gpu_forward(ref, n, block)
    got = check_forward_head(res, 0, 0, q, k, v, alpha, True, block)
    assert got["err_out"] <= 1e-2 and got["err_tau"] <= 1e-6

    bad = _as_gpu_forward(ref, n, block)
    bad.out[0, 0, 17, 3] += 0.05                       # one output entry off by 0.05
    with pytest.raises(AssertionError, match="O max-abs"):
        check_forward_head(bad, 0, 0, q, k, v, alpha, True, block)

    bad = _as_gpu_forward(ref, n, block)
    bad.tau[0, 0, 150] += 0.01 * max(1.0, abs(float(ref["tau"][150])))
    with pytest.raises(AssertionError, match="tau"):
        check_forward_head(bad, 0, 0, q, k, v, alpha, True, block)

    # flip a mask bit whose block margin is far from the tie band
    margin = ref["margin"]
    i, j = np.argwhere(np.abs(margin) > 0.1)[0]
    words = ref["mask"].copy()
    words[i, j // 32] ^= np.uint32(1) << np.uint32(j % 32)
    bad = _as_gpu_forward({**ref, "mask": words}, n, block)
    with pytest.raises(AssertionError, match="mask differs"):
        check_forward_head(bad, 0, 0, q, k, v, alpha, True, block)


def test_gradient_check_accepts_exact_and_rejects_planted_errors():
    q, k, v, do = _head(160, alpha=1.5)
    rq, rk, rv = O.attention_backward(q, k, v, do, 1.5, True)

    def as_gpu(*gs):
        return tuple(torch.from_numpy(g).to(torch.bfloat16)[None, None] for g in gs)

    out = check_grads_head(as_gpu(rq, rk, rv), 0, 0, q, k, v, do, 1.5, True)
    assert all(e["excess"] <= 0 for e in out.values())
    for which in range(3):
        gs = [rq.copy(), rk.copy(), rv.copy()]
        gs[which][5, 2] += 0.05
        with pytest.raises(AssertionError, match=("dq", "dk", "dv")[which]):
            check_grads_head(as_gpu(*gs), 0, 0, q, k, v, do, 1.5, True)


@pytest.mark.parametrize("alpha", [1.5, 2.0])
def test_full_head_check_accepts_exact_and_rejects_planted_errors(alpha):
    from parity import check_full_head

    n, block = 200, 64
    q, k, v, do = _head(n, alpha=alpha)
    ref = O.attention_windowed(q, k, v, do, alpha, True, block, workers=1)

    def as_gpu(r):
        f = _as_gpu_forward(r, n, block)
        grads = tuple(torch.from_numpy(r[g]).to(torch.bfloat16)[None, None]
                      for g in ("dq", "dk", "dv"))
        return f, grads

    f, grads = as_gpu(ref)
    rec = check_full_head(f, grads, 0, 0, ref, block)
    assert rec["err_out"] <= 1e-2 and rec["err_tau_rel"] <= 1e-6
    assert rec["mask_diff_outside_ties"] == 0
    assert all(rec[g]["excess"] <= 0 for g in ("dq", "dk", "dv"))

    for planted, match in ((("out", 17, 3, 0.05), "err_out"), (("tau", 150, None, None), "err_tau"),
                           (("dq", 5, 2, 0.05), "dq"), (("dk", 0, 1, 0.05), "dk"),
                           (("dv", 199, 0, 0.05), "dv")):
        name, r, c, dlt = planted
        bad = {key: (val.copy() if isinstance(val, np.ndarray) else val) for key, val in ref.items()}
        if name == "tau":
            bad["tau"][r] += 0.01 * max(abs(bad["tau"][r]), 1.0)
        else:
            bad[name][r, c] += dlt
        f, grads = as_gpu(bad)
        # the mask stays the reference's own
        f.mask = _as_gpu_forward(ref, n, block).mask
        with pytest.raises(AssertionError, match=match):
            check_full_head(f, grads, 0, 0, ref, block)

    # a flipped mask bit far from the tie band
    i, j = np.argwhere(np.abs(ref["margin"]) > 0.1)[0]
    words = ref["mask"].copy()
    words[i, j // 32] ^= np.uint32(1) << np.uint32(j % 32)
    f, grads = as_gpu({**ref, "mask": words})
    with pytest.raises(AssertionError, match="mask differs"):
        check_full_head(f, grads, 0, 0, ref, block)


def test_grad_stats_counts_entries_beyond_the_literal_bound():
    from parity import grad_stats

    want = np.array([[0.5, 10.0, 30.0], [-40.0, 0.01, 1.0]])
    got = want.copy()
    got[0, 1] += 0.03          # beyond 2e-2, relative 3e-3 (inside 10's half ulp 0.03125)
    got[1, 0] -= 0.1           # beyond, relative 2.5e-3
    got[1, 2] += 0.01          # inside the literal bound
    st = grad_stats(got, want)
    assert st["n_over_literal"] == 2
    assert st["max_rel_over_literal"] == pytest.approx(0.03 / 10.0)
    assert st["min_ref_over_literal"] == pytest.approx(10.0)
    assert st["max_abs"] == pytest.approx(0.1)
    # excess over the bf16 half ulp: 10 -> 0.03 - 2^-5, 40 -> 0.1 - 2^-3, 1 -> 0.01 - 2^-8
    assert st["excess"] == pytest.approx(0.01 - 2.0 ** -8)
