"""Pins for the rectangular (decode) oracle: Nq queries against Nk keys with
causal masking aligned to the end of the keys."""
import math

import numpy as np
import pytest

import oracle


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


@pytest.mark.parametrize("causal", [False, True])
def test_square_case_equals_square_oracle(causal):
    q, k, v = (_rand((37, 8), s) for s in (1, 2, 3))
    o, lse = oracle.head_forward_rect(q, k, v, 0.4, causal)
    o2, lse2 = oracle.head_forward(q, k, v, 0.4, causal)
    np.testing.assert_allclose(o, o2, atol=1e-13)
    np.testing.assert_allclose(lse, lse2, atol=1e-13)


@pytest.mark.parametrize("nq", [1, 3, 16])
def test_decode_rows_are_the_last_rows_of_causal_attention(nq):
    n, d = 50, 6
    q, k, v = (_rand((n, d), s) for s in (4, 5, 6))
    o_full, lse_full = oracle.head_forward(q, k, v, 0.3, True)
    o, lse = oracle.head_forward_rect(q[n - nq:], k, v, 0.3, True)
    np.testing.assert_allclose(o, o_full[n - nq:], atol=1e-13)
    np.testing.assert_allclose(lse, lse_full[n - nq:], atol=1e-13)


def test_brute_force_rect():
    nq, nk, d = 3, 7, 4
    q, k, v = _rand((nq, d), 7), _rand((nk, d), 8), _rand((nk, d), 9)
    for causal in (False, True):
        o, lse = oracle.head_forward_rect(q, k, v, 0.7, causal)
        for i in range(nq):
            js = [j for j in range(nk) if not (causal and j > nk - nq + i)]
            s = [0.7 * sum(q[i][c] * k[j][c] for c in range(d)) for j in js]
            mx = max(s)
            z = sum(math.exp(x - mx) for x in s)
            assert abs(lse[i] - (mx + math.log(z))) < 1e-12
            for c in range(d):
                ref = sum(math.exp(x - mx) / z * v[j][c] for x, j in zip(s, js))
                assert abs(o[i][c] - ref) < 1e-12


def test_lse_merge_of_key_halves_equals_whole():
    """Attention over all keys = merge of attention over two disjoint key sets,
    weighted by exp(LSE_part - LSE_all), with LSE_all = log(sum exp LSE_part)."""
    q, k, v = _rand((4, 8), 10), _rand((90, 8), 11), _rand((90, 8), 12)
    o, lse = oracle.head_forward_rect(q, k, v, 0.5, False)
    oa, la = oracle.head_forward_rect(q, k[:33], v[:33], 0.5, False)
    ob, lb = oracle.head_forward_rect(q, k[33:], v[33:], 0.5, False)
    lm = np.logaddexp(la, lb)
    om = np.exp(la - lm)[:, None] * oa + np.exp(lb - lm)[:, None] * ob
    np.testing.assert_allclose(lm, lse, atol=1e-12)
    np.testing.assert_allclose(om, o, atol=1e-12)


def _literal_rect(qh, kh, vh, scale, causal):
    """Pure-Python loops over one head: Nq rows against Nk keys, causal mask
    aligned to the end of the keys, full-row softmax."""
    nq, nk, d = len(qh), len(kh), len(vh[0])
    o = [[0.0] * d for _ in range(nq)]
    lse = [0.0] * nq
    for i in range(nq):
        js = [j for j in range(nk) if not (causal and j > nk - nq + i)]
        s = [scale * sum(qh[i][c] * kh[j][c] for c in range(d)) for j in js]
        mx = max(s)
        z = sum(math.exp(x - mx) for x in s)
        lse[i] = mx + math.log(z)
        for c in range(d):
            o[i][c] = sum(math.exp(x - mx) / z * vh[j][c] for x, j in zip(s, js))
    return np.array(o), np.array(lse)


@pytest.mark.parametrize("causal", [False, True])
def test_batched_rect_matches_literal_loops_per_head(causal):
    """attention_forward_rect on B=2, H=3, Nq=5 < Nk=11: every (b, h) slice
    equals literal loops over that head's own q, k, v.  The heads are drawn
    with different scales so that a b/h mix-up or a k/v swap cannot pass."""
    B, H, nq, nk, d = 2, 3, 5, 11, 4
    rng = np.random.default_rng(91)
    mult = (1.0 + np.arange(B * H).reshape(B, H, 1, 1))
    q = rng.standard_normal((B, H, nq, d)) * mult
    k = rng.standard_normal((B, H, nk, d))
    v = rng.standard_normal((B, H, nk, d)) * mult + 3.0 * mult
    o, lse = oracle.attention_forward_rect(q, k, v, 0.45, causal)
    assert o.shape == (B, H, nq, d) and lse.shape == (B, H, nq)
    for b in range(B):
        for h in range(H):
            ob, lb = _literal_rect(q[b, h].tolist(), k[b, h].tolist(), v[b, h].tolist(), 0.45, causal)
            np.testing.assert_allclose(o[b, h], ob, atol=1e-12)
            np.testing.assert_allclose(lse[b, h], lb, atol=1e-12)


def test_batched_rect_swapped_kv_is_detected():
    """Sanity of the pin above: exchanging K and V changes the result."""
    B, H, nq, nk, d = 1, 2, 3, 9, 4
    rng = np.random.default_rng(92)
    q, k, v = (rng.standard_normal((B, H, n, d)) for n in (nq, nk, nk))
    o, _ = oracle.attention_forward_rect(q, k, v, 0.5, False)
    o_sw, _ = oracle.attention_forward_rect(q, v, k, 0.5, False)
    assert np.max(np.abs(o - o_sw)) > 1e-3
