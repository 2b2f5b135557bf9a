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
