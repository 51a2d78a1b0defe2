"""Pins for the float64 oracle: it is checked against facts that do not come
from itself -- closed forms, limits, bounds, finite differences and
hand-derived worked examples -- so that a dropped term, a wrong sign or a
transposed operand in it fails one of these tests.
"""

import json
import os

import numpy as np
import pytest

import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
RNG = np.random.default_rng(12345)


# ---------------------------------------------------------------- closed forms
def sparsemax_sort(z):
    """Textbook sort-based sparsemax (Martins & Astudillo 2016): support size
    k* = max{k : 1 + k z_(k) > sum_{j<=k} z_(j)}, tau = (sum_{j<=k*} z_(j) - 1)/k*."""
    zs = np.sort(z)[::-1]
    cs = np.cumsum(zs)
    ks = np.arange(1, len(z) + 1)
    kstar = ks[1 + ks * zs > cs].max()
    tau = (cs[kstar - 1] - 1.0) / kstar
    return np.maximum(z - tau, 0.0), tau


def entmax15_sort(z):
    """Exact sort-based 1.5-entmax (Peters, Niculae & Martins 2019).

    With s = z/2 sorted descending and the top K active, sum (s_j - tau)^2 = 1
    is a quadratic in tau whose smaller root is tau_K = mean_K - sqrt((1 - ss_K)/K),
    ss_K = sum_{j<=K} (s_j - mean_K)^2.  The support is the largest K with
    tau_K <= s_(K).
    """
    s = np.sort(z / 2.0)[::-1]
    best = None
    for K in range(1, len(s) + 1):
        top = s[:K]
        mean = top.mean()
        ss = ((top - mean) ** 2).sum()
        disc = (1.0 - ss) / K
        if disc < 0:
            continue
        tau = mean - np.sqrt(disc)
        if tau <= s[K - 1]:
            best = tau
    return np.maximum(z / 2.0 - best, 0.0) ** 2, best


def softmax(z):
    e = np.exp(z - z.max(-1, keepdims=True))
    return e / e.sum(-1, keepdims=True)


@pytest.mark.parametrize("n", [2, 5, 17, 64, 300])
def test_t1_sparsemax_closed_form(n):
    for _ in range(20):
        z = RNG.normal(size=n) * RNG.uniform(0.2, 5.0)
        p, tau = O.entmax(z, 2.0)
        p_ref, tau_ref = sparsemax_sort(z)
        assert abs(tau[0] - tau_ref) <= 1e-12
        np.testing.assert_allclose(p[0], p_ref, rtol=0, atol=1e-12)


@pytest.mark.parametrize("n", [2, 5, 17, 64, 300])
def test_t1_entmax15_closed_form(n):
    for _ in range(20):
        z = RNG.normal(size=n) * RNG.uniform(0.2, 5.0)
        p, tau = O.entmax(z, 1.5)
        p_ref, tau_ref = entmax15_sort(z)
        assert abs(tau[0] - tau_ref) <= 1e-12
        np.testing.assert_allclose(p[0], p_ref, rtol=0, atol=1e-11)


def test_golden_worked_examples():
    with open(os.path.join(GOLDEN, "entmax_worked_examples.json")) as f:
        cases = json.load(f)["cases"]
    assert len(cases) >= 5
    for c in cases:
        p, tau = O.entmax(np.array(c["z"]), c["alpha"])
        assert abs(tau[0] - c["tau"]) <= 1e-11, c["name"]
        np.testing.assert_allclose(p[0], c["p"], rtol=0, atol=1e-11, err_msg=c["name"])


def test_t2_softmax_limit():
    z = RNG.normal(size=(8, 40)) * 2.0
    errs = []
    for eps in (1e-1, 1e-2, 1e-3):
        p, _ = O.entmax(z, 1.0 + eps)
        errs.append(np.abs(p - softmax(z)).max())
    assert errs[0] > errs[1] > errs[2]
    assert errs[2] < 1e-2


@pytest.mark.parametrize("alpha", [1.25, 1.5, 2.0, 3.0])
def test_t3_t4_row_sums_and_bounds(alpha):
    z = RNG.normal(size=(32, 257)) * 3.0
    z[:, 100:] = -np.inf                       # ragged valid length
    z[5, 1:] = -np.inf                         # single valid entry
    p, tau = O.entmax(z, alpha)
    assert np.abs(p.sum(-1) - 1.0).max() <= 1e-10
    s = (alpha - 1.0) * z
    m = s.max(-1)
    n = np.isfinite(s).sum(-1)
    assert np.all(tau >= m - 1.0 - 1e-12)
    assert np.all(tau <= m - n ** (1.0 - alpha) + 1e-12)
    assert abs(tau[5] - (m[5] - 1.0)) <= 1e-12 and abs(p[5, 0] - 1.0) <= 1e-12


@pytest.mark.parametrize("anchor", ["grid", "max"])
@pytest.mark.parametrize("n_bins", [8, 16, 32])
@pytest.mark.parametrize("alpha", [1.5, 2.0, 1.25, 3.0])
def test_t5_histogram_lower_bound(anchor, n_bins, alpha):
    """Proposition 1 as the summaries state it (zh §2.1, ja §2.1):
    tau* - h < tau_h <= tau*, and the support at tau_h contains the true one
    (es §2A).  The max-anchored window puts the maximum itself at the lower
    edge of the top bin (its representative is m - h), so there the lower
    bound holds with equality when the maximum alone is in the support."""
    h = 1.0 / n_bins
    for scale in (0.5, 2.0, 6.0):
        z = RNG.normal(size=(24, 513)) * scale
        s = (alpha - 1.0) * z
        tau = O.entmax_threshold(s, alpha)
        tau_h = O.histogram_threshold(s, alpha, n_bins, anchor)
        assert np.all(tau_h <= tau + 1e-12)
        if anchor == "grid":
            assert np.all(tau_h > tau - h)
        else:
            assert np.all(tau_h >= tau - h - 1e-12)
        assert np.all((s > tau_h[:, None]) | ~(s > tau[:, None]))


def test_t5_histogram_is_not_trivial():
    """The bound is informative: tau_h moves with n_bins toward tau*."""
    z = RNG.normal(size=(64, 1000)) * 3.0
    s = 0.5 * z
    tau = O.entmax_threshold(s, 1.5)
    gaps = [np.abs(tau - O.histogram_threshold(s, 1.5, nb, "grid")).mean()
            for nb in (4, 16, 64)]
    assert gaps[0] > gaps[1] > gaps[2]
    assert gaps[2] < 1.0 / 64


def _rand_row_with_gap(n, alpha, gap=1e-3):
    while True:
        z = RNG.normal(size=n) * 2.0
        s = (alpha - 1.0) * z
        tau = O.entmax_threshold(s, alpha)[0]
        if np.abs(s - tau).min() > gap:
            return z


@pytest.mark.parametrize("alpha", [1.5, 2.0, 1.3])
def test_t6_jacobian_finite_differences(alpha):
    for n in (6, 9, 12):
        z = _rand_row_with_gap(n, alpha)
        v = RNG.normal(size=n)
        eps = 1e-6
        # tol=0: bisect to float resolution so that the threshold's own
        # stopping error (divided by 2*eps) does not swamp the difference
        fd = (O.entmax(z + eps * v, alpha, tol=0.0)[0]
              - O.entmax(z - eps * v, alpha, tol=0.0)[0]) / (2 * eps)
        p = O.entmax(z, alpha)[0]
        np.testing.assert_allclose(O.entmax_jvp(p, v, alpha), fd, rtol=0, atol=1e-7)


@pytest.mark.parametrize("alpha", [1.5, 2.0, 1.3, 3.0])
@pytest.mark.parametrize("causal", [True, False])
def test_t6_attention_gradients_finite_differences(alpha, causal):
    """dQ, dK, dV against central differences of L = <O, dO>."""
    n, d = 8, 4
    for _ in range(3):
        q, k, v, do = (RNG.normal(size=(n, d)) for _ in range(4))
        q *= 2.0

        def loss(q_, k_, v_):
            return (O.attention_forward(q_, k_, v_, alpha, causal, block=4,
                                        tol=0.0)["out"] * do).sum()

        # skip draws with a score within 1e-4 of its threshold (kink of [.]_+)
        s = (alpha - 1.0) * O.scores(q, k, causal)
        tau = O.entmax_threshold(s, alpha)
        t = s - tau[:, None]
        if np.abs(t[np.isfinite(t)]).min() < 1e-4:
            continue
        dq, dk, dv = O.attention_backward(q, k, v, do, alpha, causal)
        eps = 1e-6
        for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
            fd = np.zeros_like(x)
            for idx in np.ndindex(*x.shape):
                xp, xm = x.copy(), x.copy()
                xp[idx] += eps
                xm[idx] -= eps
                args_p = {"q": q, "k": k, "v": v}
                args_m = dict(args_p)
                args_p[name], args_m[name] = xp, xm
                fd[idx] = (loss(**{f"{a}_": b for a, b in args_p.items()})
                           - loss(**{f"{a}_": b for a, b in args_m.items()})) / (2 * eps)
            np.testing.assert_allclose(g, fd, rtol=0, atol=1e-6, err_msg=name)


def test_t7_special_cases():
    # causal row 0 sees only key 0: p = 1, O = v_0, tau = s_0 - 1
    n, d = 16, 8
    q, k, v = (RNG.normal(size=(n, d)) for _ in range(3))
    for alpha in (1.5, 2.0):
        r = O.attention_forward(q, k, v, alpha, True, block=8)
        s00 = (alpha - 1.0) * (q[0] @ k[0]) / np.sqrt(d)
        np.testing.assert_allclose(r["out"][0], v[0], atol=1e-14)
        assert abs(r["tau"][0] - (s00 - 1.0)) <= 1e-12
    # all-equal scores: uniform, tau = s - n^(1-alpha)
    for alpha in (1.5, 2.0, 3.0):
        z = np.full((1, 10), 0.7)
        p, tau = O.entmax(z, alpha)
        np.testing.assert_allclose(p, 0.1, atol=1e-12)
        assert abs(tau[0] - ((alpha - 1) * 0.7 - 10 ** (1 - alpha))) <= 1e-12
    # two elements at alpha=2: p_1 = clip((z_1 - z_2 + 1)/2, 0, 1)
    for a, b in ((0.3, 0.1), (2.0, 0.1), (-0.4, 0.5), (0.0, 3.0)):
        p, _ = O.entmax(np.array([a, b]), 2.0)
        assert abs(p[0, 0] - np.clip((a - b + 1) / 2, 0, 1)) <= 1e-12


def test_t8_invariances():
    n, d = 24, 8
    q, k, v = (RNG.normal(size=(n, d)) for _ in range(3))
    for alpha in (1.5, 2.0):
        z = RNG.normal(size=(5, 30)) * 2
        p, tau = O.entmax(z, alpha)
        p2, tau2 = O.entmax(z + 1.7, alpha)
        np.testing.assert_allclose(p2, p, atol=1e-11)
        np.testing.assert_allclose(tau2, tau + (alpha - 1) * 1.7, atol=1e-11)
        perm = RNG.permutation(30)
        p3, _ = O.entmax(z[:, perm], alpha)
        np.testing.assert_allclose(p3, p[:, perm], atol=1e-11)
        # non-causal attention: permuting keys and values together leaves O
        o = O.attention_forward(q, k, v, alpha, False, block=8)["out"]
        pk = RNG.permutation(n)
        o2 = O.attention_forward(q, k[pk], v[pk], alpha, False, block=8)["out"]
        np.testing.assert_allclose(o2, o, atol=1e-11)
        # linear in V
        o3 = O.attention_forward(q, k, 2 * v + 1.0, alpha, True, block=8)["out"]
        o1 = O.attention_forward(q, k, v, alpha, True, block=8)["out"]
        np.testing.assert_allclose(o3, 2 * o1 + 1.0, atol=1e-11)


def test_t9_mask_invariants():
    n, d, blk = 200, 16, 32
    q, k, v = (RNG.normal(size=(n, d)) for _ in range(3))
    q *= 3.0
    for alpha in (1.5, 2.0):
        r = O.attention_forward(q, k, v, alpha, True, block=blk)
        tr = (n + blk - 1) // blk
        # mask from the probabilities themselves, built independently
        s = (alpha - 1) * O.scores(q, k, True)
        p = O.entmax_probs(s, r["tau"], alpha)
        act = np.zeros((tr, tr), bool)
        for i in range(tr):
            for j in range(tr):
                act[i, j] = (p[i * blk:(i + 1) * blk, j * blk:(j + 1) * blk] > 0).any()
        np.testing.assert_array_equal(O.pack_block_mask(act), r["mask"])
        assert act.sum() >= tr
        # every row block holds the block of each of its rows' maxima
        for row in range(n):
            assert act[row // blk, np.argmax(s[row]) // blk]
        # causal: nothing above the block diagonal
        assert not np.triu(act, 1).any()


def test_pack_block_mask_bit_order():
    act = np.zeros((2, 40), bool)
    act[0, 0] = act[0, 33] = act[1, 31] = act[1, 39] = True
    w = O.pack_block_mask(act)
    assert w.dtype == np.uint32 and w.shape == (2, 2)
    assert w[0, 0] == 1 and w[0, 1] == 2
    assert w[1, 0] == np.uint32(1 << 31) and w[1, 1] == np.uint32(1 << 7)


def test_sampled_rows_match_full():
    n, d = 300, 16
    q, k, v, do = (RNG.normal(size=(n, d)) for _ in range(4))
    full = O.attention_forward(q, k, v, 1.5, True, block=64)
    rows = np.array([0, 7, 64, 299])
    part = O.attention_forward(q, k, v, 1.5, True, block=64, rows=rows)
    np.testing.assert_allclose(part["out"], full["out"][rows], atol=1e-13)
    np.testing.assert_allclose(part["tau"], full["tau"][rows], atol=1e-13)
    dq, dk, dv = O.attention_backward(q, k, v, do, 1.5, True)
    tail = np.arange(250, n)
    dq_t, dk_t, dv_t = O.attention_backward(q, k, v, do, 1.5, True, rows=tail)
    np.testing.assert_allclose(dq_t, dq[tail], atol=1e-12)
    np.testing.assert_allclose(dk_t[250:], dk[250:], atol=1e-12)
    np.testing.assert_allclose(dv_t[250:], dv[250:], atol=1e-12)


def test_block_margins_hand_computed():
    # 4 rows x 4 keys, blocks of 2: margin(i, j) = max over the block of s - tau_row.
    s = np.array([[0.5, -np.inf, -np.inf, -np.inf],
                  [0.2, 0.9, -np.inf, -np.inf],
                  [1.0, 0.3, 0.4, -np.inf],
                  [0.0, 2.0, 0.6, 0.7]])
    tau = np.array([0.1, 0.5, 0.8, 1.5])
    # block (0, 0): max(0.5 - 0.1, 0.2 - 0.5, 0.9 - 0.5) = 0.4
    # block (0, 1): no valid entry -> -inf
    # block (1, 0): max(1.0 - 0.8, 0.3 - 0.8, 0.0 - 1.5, 2.0 - 1.5) = 0.5
    # block (1, 1): max(0.4 - 0.8, 0.6 - 1.5, 0.7 - 1.5) = -0.4
    want = np.array([[0.4, -np.inf], [0.5, -0.4]])
    got = O.block_margins(s, tau, 0, 2, 4)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-15)
    # a ragged tail: 3 keys, the last block holds one key only
    got3 = O.block_margins(s[:3, :3], tau[:3], 0, 2, 3)
    np.testing.assert_allclose(got3, np.array([[0.4, -np.inf], [0.2, -0.4]]), rtol=0,
                               atol=1e-15)


WINDOWED_CASES = [
    # n, d, alpha, causal, block, q scale, rows_per_chunk, workers
    (1, 8, 1.5, True, 64, 1.0, 0, 1),
    (200, 16, 1.5, True, 64, 2.0, 64, 3),
    (300, 16, 2.0, True, 128, 3.0, 128, 2),
    (300, 16, 1.25, False, 64, 1.0, 0, 4),
    (517, 8, 3.0, True, 64, 1.5, 192, 2),
    (256, 16, 1.5, False, 128, 0.3, 128, 1),
]


@pytest.mark.parametrize("case", WINDOWED_CASES, ids=[str(i) for i in range(len(WINDOWED_CASES))])
def test_windowed_matches_dense_definition(case):
    n, d, alpha, causal, block, qs, rpc, workers = case
    rng = np.random.default_rng(n * 7 + d)
    q = rng.normal(size=(n, d)) * qs
    k, v, do = (rng.normal(size=(n, d)) for _ in range(3))
    f = O.attention_forward(q, k, v, alpha, causal, block)
    dq, dk, dv = O.attention_backward(q, k, v, do, alpha, causal)
    w = O.attention_windowed(q, k, v, do, alpha, causal, block, rows_per_chunk=rpc,
                             workers=workers)
    # both thresholds are within the 1e-12 bisection tolerance of tau*; beyond
    # alpha = 2, p = t^(1/(alpha-1)) has an unbounded slope where a score
    # enters the support, so that tolerance shows up amplified in O and dV
    atol = 1e-10 if alpha <= 2.0 else 1e-8
    np.testing.assert_allclose(w["tau"], f["tau"], rtol=0, atol=1e-11)
    np.testing.assert_allclose(w["out"], f["out"], rtol=0, atol=atol)
    np.testing.assert_allclose(w["rowsum"], 1.0, rtol=0, atol=atol)
    # gradients for alpha <= 2 only: beyond, g = p^(2-alpha) itself is
    # unbounded at the edge of the support (the library rejects that case)
    if alpha <= 2.0:
        for got, want in ((w["dq"], dq), (w["dk"], dk), (w["dv"], dv)):
            np.testing.assert_allclose(got, want, rtol=0, atol=atol)
    fin = np.isfinite(f["margin"])
    assert np.array_equal(fin, np.isfinite(w["margin"]))
    np.testing.assert_allclose(w["margin"][fin], f["margin"][fin], rtol=0, atol=1e-11)
    np.testing.assert_array_equal(w["mask"], f["mask"])


def test_windowed_wide_windows_and_ties():
    # all keys equal: every score sits in the window (the widest case), the
    # result is uniform attention; planted duplicates give exact ties
    n, d = 130, 8
    rng = np.random.default_rng(5)
    q = rng.normal(size=(n, d))
    k = np.tile(rng.normal(size=(1, d)), (n, 1))
    v, do = rng.normal(size=(n, d)), rng.normal(size=(n, d))
    for alpha in (1.5, 2.0):
        w = O.attention_windowed(q, k, v, do, alpha, True, 64, workers=2)
        want = np.cumsum(v, axis=0) / np.arange(1, n + 1)[:, None]
        np.testing.assert_allclose(w["out"], want, rtol=0, atol=1e-10)
        dq, dk, dv = O.attention_backward(q, k, v, do, alpha, True)
        np.testing.assert_allclose(w["dv"], dv, rtol=0, atol=1e-10)
        np.testing.assert_allclose(w["dk"], dk, rtol=0, atol=1e-10)
        np.testing.assert_allclose(w["dq"], dq, rtol=0, atol=1e-10)


def test_windowed_pin_catches_a_narrower_window():
    # Mutation check: cutting the window at m - 1/2 instead of m - 1 drops
    # support entries on this wide-support case, and the comparison with the
    # dense definition must notice.
    n, d = 96, 8
    rng = np.random.default_rng(9)
    q = rng.normal(size=(n, d)) * 0.3
    k, v, do = (rng.normal(size=(n, d)) for _ in range(3))
    f = O.attention_forward(q, k, v, 2.0, True, 32)
    good = O.attention_windowed(q, k, v, do, 2.0, True, 32, workers=1)
    bad = O.attention_windowed(q, k, v, do, 2.0, True, 32, workers=1, _window=0.5)
    np.testing.assert_allclose(good["tau"], f["tau"], rtol=0, atol=1e-11)
    assert np.abs(bad["tau"] - f["tau"]).max() > 1e-3
    assert np.abs(bad["out"] - f["out"]).max() > 1e-3
