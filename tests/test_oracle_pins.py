"""Pins for the fp64 oracle: checks against things other than the oracle itself.

Each test is chosen so that a plausible slip in the oracle (a dropped term, a
wrong sign or index, a transposed operand, a missing scale factor, a wrong
causal direction) fails at least one of them:

* brute force: a literal pure-Python triple loop on tiny shapes;
* the online-softmax recurrence (running max m and denominator l, rescaled by
  exp(m_old - m_new) -- explainers.rudrite.com "flash-attention-anatomy", Q&A
  "What is online softmax and how does tiling keep it exact?") written here
  independently, which must equal the two-pass full-row softmax;
* P rows sum to one and are non-negative (chipfoundryservices glossary "flash
  attention": running maximum and normalizer);
* closed forms: constant scores give the mean of V (prefix mean when causal),
  N = 1 gives O = V, the hand-derived cases under tests/golden/;
* invariants: convex hull of V rows, affine equivariance in V, joint
  permutation of K/V rows (non-causal);
* central finite differences of L = sum(dO o O) for every gradient entry;
* the gradient sum identities sum_j dK_j = 0 and sum_j dV_j = sum_i dO_i.
"""
import json
import math
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "tiny_closed_forms.json")


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


# ---------------------------------------------------------------- brute force
def _brute_forward(q, k, v, scale, causal):
    n, d = q.shape
    dv = v.shape[1]
    o = [[0.0] * dv for _ in range(n)]
    lse = [0.0] * n
    for i in range(n):
        s = []
        for j in range(k.shape[0]):
            if causal and j > i:
                continue
            acc = 0.0
            for c in range(d):
                acc += q[i][c] * k[j][c]
            s.append((j, scale * acc))
        mx = max(val for _, val in s)
        z = sum(math.exp(val - mx) for _, val in s)
        lse[i] = mx + math.log(z)
        for j, val in s:
            w = math.exp(val - mx) / z
            for c in range(dv):
                o[i][c] += w * v[j][c]
    return np.array(o), np.array(lse)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("n,d", [(1, 1), (2, 3), (5, 4), (8, 8), (7, 2)])
def test_brute_force_forward(n, d, causal):
    q, k, v = _rand((n, d), 1), _rand((n, d), 2), _rand((n, d), 3)
    scale = 0.7
    o, lse = oracle.head_forward(q, k, v, scale, causal)
    ob, lseb = _brute_forward(q, k, v, scale, causal)
    np.testing.assert_allclose(o, ob, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, lseb, rtol=0, atol=1e-12)


def _brute_backward(q, k, v, do, scale, causal):
    """Gradients by literal loops over the chain rule of the softmax."""
    n, d = q.shape
    o, _ = _brute_forward(q, k, v, scale, causal)
    P = [[0.0] * n for _ in range(n)]
    for i in range(n):
        js = [j for j in range(n) if not (causal and j > i)]
        s = {j: scale * sum(q[i][c] * k[j][c] for c in range(d)) for j in js}
        mx = max(s.values())
        z = sum(math.exp(s[j] - mx) for j in js)
        for j in js:
            P[i][j] = math.exp(s[j] - mx) / z
    dq = np.zeros((n, d))
    dk = np.zeros((n, d))
    dvv = np.zeros((n, d))
    for i in range(n):
        Di = sum(do[i][c] * o[i][c] for c in range(d))
        for j in range(n):
            if P[i][j] == 0.0:
                continue
            dPij = sum(do[i][c] * v[j][c] for c in range(d))
            dSij = P[i][j] * (dPij - Di)
            for c in range(d):
                dvv[j][c] += P[i][j] * do[i][c]
                dq[i][c] += scale * dSij * k[j][c]
                dk[j][c] += scale * dSij * q[i][c]
    return dq, dk, dvv


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("n,d", [(1, 2), (3, 2), (6, 5)])
def test_brute_force_backward(n, d, causal):
    q, k, v, do = (_rand((n, d), s) for s in (4, 5, 6, 7))
    dq, dk, dv, _, _ = oracle.head_backward(q, k, v, do, 0.9, causal)
    bq, bk, bv = _brute_backward(q, k, v, do, 0.9, causal)
    for a, b in ((dq, bq), (dk, bk), (dv, bv)):
        np.testing.assert_allclose(a, b, rtol=0, atol=1e-12)


# ------------------------------------------------------------ online softmax
def _online_forward(q, k, v, scale, causal, tile):
    """Running max m, running denominator l, output rescaled by
    exp(m_old - m_new) whenever a tile raises the max; normalised at the end."""
    n = q.shape[0]
    o = np.zeros((n, v.shape[1]))
    lse = np.zeros(n)
    for i in range(n):
        m = -np.inf
        l = 0.0
        acc = np.zeros(v.shape[1])
        for j0 in range(0, k.shape[0], tile):
            j1 = min(k.shape[0], j0 + tile)
            s = scale * (k[j0:j1] @ q[i])
            if causal:
                s = np.where(np.arange(j0, j1) > i, -np.inf, s)
            m_new = max(m, float(np.max(s)))
            if m_new == -np.inf:
                continue
            alpha = math.exp(m - m_new) if m > -np.inf else 0.0
            p = np.exp(s - m_new)
            l = l * alpha + float(np.sum(p))
            acc = acc * alpha + p @ v[j0:j1]
            m = m_new
        o[i] = acc / l
        lse[i] = m + math.log(l)
    return o, lse


@pytest.mark.parametrize("tile", [1, 2, 3, 7])
@pytest.mark.parametrize("mult", [1.0, 8.0, 64.0])
@pytest.mark.parametrize("causal", [False, True])
def test_online_recurrence_equals_full_softmax(tile, mult, causal):
    n, d = 23, 6
    q = _rand((n, d), 11) * mult
    k, v = _rand((n, d), 12), _rand((n, d), 13)
    o, lse = oracle.head_forward(q, k, v, 0.4, causal)
    oo, lo = _online_forward(q, k, v, 0.4, causal, tile)
    np.testing.assert_allclose(o, oo, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(lse, lo, rtol=1e-12, atol=1e-12)


# ------------------------------------------------------------- softmax facts
@pytest.mark.parametrize("causal", [False, True])
def test_probability_rows(causal):
    q, k = _rand((40, 8), 21) * 3, _rand((40, 8), 22)
    p = oracle.attention_probs(q, k, 0.5, causal)
    assert np.all(p >= 0)
    np.testing.assert_allclose(p.sum(axis=1), 1.0, rtol=0, atol=1e-12)
    if causal:
        assert np.all(np.triu(p, 1) == 0.0)
        assert np.all(np.diag(p) > 0)


def test_constant_scores_give_mean_of_v():
    n, d = 17, 5
    v = _rand((n, d), 31)
    k = np.tile(_rand((1, d), 32), (n, 1))          # all key rows equal
    q = _rand((n, d), 33)
    o, lse = oracle.head_forward(q, k, v, 0.3, False)
    np.testing.assert_allclose(o, np.tile(v.mean(axis=0), (n, 1)), atol=1e-12)
    s = 0.3 * (q @ k[0])
    np.testing.assert_allclose(lse, s + math.log(n), atol=1e-12)
    # Q = 0: every score is 0, LSE = ln N
    o0, l0 = oracle.head_forward(np.zeros((n, d)), _rand((n, d), 34), v, 1.0, False)
    np.testing.assert_allclose(o0, np.tile(v.mean(axis=0), (n, 1)), atol=1e-12)
    np.testing.assert_allclose(l0, math.log(n), atol=1e-12)


def test_constant_scores_causal_prefix_mean():
    n, d = 13, 4
    v = _rand((n, d), 41)
    o, lse = oracle.head_forward(np.zeros((n, d)), _rand((n, d), 42), v, 1.0, True)
    prefix = np.cumsum(v, axis=0) / np.arange(1, n + 1)[:, None]
    np.testing.assert_allclose(o, prefix, atol=1e-12)
    np.testing.assert_allclose(lse, np.log(np.arange(1, n + 1)), atol=1e-12)


def test_single_key_and_causal_row0():
    q, k, v = _rand((1, 6), 51), _rand((1, 6), 52), _rand((1, 6), 53)
    o, lse = oracle.head_forward(q, k, v, 0.8, False)
    np.testing.assert_allclose(o, v, atol=1e-15)
    np.testing.assert_allclose(lse, 0.8 * (q[0] @ k[0]), atol=1e-15)
    q, k, v = _rand((9, 6), 54), _rand((9, 6), 55), _rand((9, 6), 56)
    o, lse = oracle.head_forward(q, k, v, 0.8, True)
    np.testing.assert_allclose(o[0], v[0], atol=1e-15)
    np.testing.assert_allclose(lse[0], 0.8 * (q[0] @ k[0]), atol=1e-14)


def test_convex_hull_affine_permutation():
    n, d = 31, 7
    q, k, v = _rand((n, d), 61) * 4, _rand((n, d), 62), _rand((n, d), 63)
    for causal in (False, True):
        o, _ = oracle.head_forward(q, k, v, 0.6, causal)
        for i in range(n):
            vis = v[: i + 1] if causal else v
            assert np.all(o[i] >= vis.min(axis=0) - 1e-12)
            assert np.all(o[i] <= vis.max(axis=0) + 1e-12)
        oa, la = oracle.head_forward(q, k, 2.5 * v - 1.25, 0.6, causal)
        np.testing.assert_allclose(oa, 2.5 * o - 1.25, atol=1e-12)
    perm = np.random.default_rng(64).permutation(n)
    o, lse = oracle.head_forward(q, k, v, 0.6, False)
    op, lp = oracle.head_forward(q, k[perm], v[perm], 0.6, False)
    np.testing.assert_allclose(op, o, atol=1e-12)
    np.testing.assert_allclose(lp, lse, atol=1e-12)


def test_batched_forward_matches_heads():
    B, H, N, d = 2, 3, 19, 8
    q, k, v = (_rand((B, H, N, d), s) for s in (71, 72, 73))
    o, lse = oracle.attention_forward(q, k, v, 0.35, True)
    for b in range(B):
        for h in range(H):
            ob, lb = _brute_forward(q[b, h], k[b, h], v[b, h], 0.35, True)
            np.testing.assert_allclose(o[b, h], ob, atol=1e-12)
            np.testing.assert_allclose(lse[b, h], lb, atol=1e-12)


def test_row_subset_matches_full():
    q, k, v = (_rand((50, 8), s) for s in (81, 82, 83))
    rows = np.array([0, 7, 31, 49])
    for causal in (False, True):
        o, lse = oracle.head_forward(q, k, v, 0.5, causal)
        os_, ls_ = oracle.head_forward(q, k, v, 0.5, causal, rows=rows)
        np.testing.assert_allclose(os_, o[rows], atol=1e-13)
        np.testing.assert_allclose(ls_, lse[rows], atol=1e-13)


def test_row_blocking_is_transparent(monkeypatch):
    q, k, v, do = (_rand((45, 6), s) for s in (91, 92, 93, 94))
    ref = oracle.head_backward(q, k, v, do, 0.5, True)
    monkeypatch.setattr(oracle, "_MAX_BLOCK_ELEMS", 45 * 4)   # 4-row blocks
    blk = oracle.head_backward(q, k, v, do, 0.5, True)
    for a, b in zip(ref, blk):
        np.testing.assert_allclose(a, b, atol=1e-12)


# ------------------------------------------------------------------ golden
def test_golden_closed_forms():
    cases = json.load(open(GOLDEN))["cases"]
    for c in cases:
        q, k, v, do = (np.array(c[n], dtype=np.float64) for n in ("q", "k", "v", "do"))
        o, lse = oracle.head_forward(q, k, v, c["scale"], c["causal"])
        np.testing.assert_allclose(o, np.array(c["o"]), atol=1e-14, err_msg=c["name"])
        np.testing.assert_allclose(lse, np.array(c["lse"]), atol=1e-14, err_msg=c["name"])
        dq, dk, dv, _, _ = oracle.head_backward(q, k, v, do, c["scale"], c["causal"])
        np.testing.assert_allclose(dq, np.array(c["dq"]), atol=1e-14, err_msg=c["name"])
        np.testing.assert_allclose(dk, np.array(c["dk"]), atol=1e-14, err_msg=c["name"])
        np.testing.assert_allclose(dv, np.array(c["dv"]), atol=1e-14, err_msg=c["name"])


# ------------------------------------------------------- finite differences
def _loss(q, k, v, do, scale, causal):
    o, _ = oracle.head_forward(q, k, v, scale, causal)
    return float(np.sum(do * o))


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("n,d", [(5, 3), (16, 8)])
def test_gradients_central_differences(n, d, causal):
    q, k, v, do = (_rand((n, d), s) for s in (101, 102, 103, 104))
    scale = 0.45
    dq, dk, dv, _, _ = oracle.head_backward(q, k, v, do, scale, causal)
    h = 1e-5
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        fd = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args = {"q": q, "k": k, "v": v}
            args[name] = xp
            lp = _loss(args["q"], args["k"], args["v"], do, scale, causal)
            args[name] = xm
            lm = _loss(args["q"], args["k"], args["v"], do, scale, causal)
            fd[idx] = (lp - lm) / (2 * h)
        err = np.linalg.norm(fd - g) / max(np.linalg.norm(g), 1e-300)
        assert err <= 1e-6, (name, err)


@pytest.mark.parametrize("causal", [False, True])
def test_gradient_sum_identities(causal):
    q, k, v, do = (_rand((64, 16), s) for s in (111, 112, 113, 114))
    dq, dk, dv, _, _ = oracle.head_backward(q, k, v, do, 0.25, causal)
    np.testing.assert_allclose(dk.sum(axis=0), 0.0, atol=1e-12)
    np.testing.assert_allclose(dv.sum(axis=0), do.sum(axis=0), atol=1e-12)


def test_sampled_backward_matches_full():
    q, k, v, do = (_rand((70, 8), s) for s in (121, 122, 123, 124))
    rows = np.array([0, 3, 33, 69])
    cols = np.array([0, 1, 40, 69])
    for causal in (False, True):
        dq, dk, dv, _, _ = oracle.head_backward(q, k, v, do, 0.3, causal)
        sq, sk, sv = oracle.head_backward_sampled(q, k, v, do, 0.3, causal, rows, cols)
        np.testing.assert_allclose(sq, dq[rows], atol=1e-12)
        np.testing.assert_allclose(sk, dk[cols], atol=1e-12)
        np.testing.assert_allclose(sv, dv[cols], atol=1e-12)


def test_batched_backward_matches_heads():
    B, H, N, d = 1, 2, 9, 4
    q, k, v, do = (_rand((B, H, N, d), s) for s in (131, 132, 133, 134))
    dq, dk, dv = oracle.attention_backward(q, k, v, do, 0.5, False)
    for h in range(H):
        bq, bk, bv = _brute_backward(q[0, h], k[0, h], v[0, h], do[0, h], 0.5, False)
        np.testing.assert_allclose(dq[0, h], bq, atol=1e-12)
        np.testing.assert_allclose(dk[0, h], bk, atol=1e-12)
        np.testing.assert_allclose(dv[0, h], bv, atol=1e-12)
