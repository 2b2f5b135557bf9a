"""Seeded random shapes through every bf16 entry point, against the fp64 oracle.

Each case draws B, H, N (ragged, 1 to a few tiles), d in {64, 128}, the causal
flag and a score multiplier from a fixed seed, runs the forward and the
backward (atomic and deterministic dQ) on the device and compares every output
with the oracle at the stated tolerances.  The shapes are kept small enough for
the oracle to finish in a second or two each.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu

fa = pytest.importorskip("exact_io_aware_55_b200")


def _cases(n, seed=2024):
    rng = np.random.default_rng(seed)
    out = []
    for i in range(n):
        d = int(rng.choice([64, 128]))
        N = int(rng.integers(1, 700))
        B = int(rng.integers(1, 3))
        H = int(rng.integers(1, 4))
        causal = bool(rng.integers(0, 2))
        mult = float(rng.choice([1.0, 1.0, 4.0, 8.0]))
        out.append((B, H, N, d, causal, mult, 3000 + i))
    return out


@pytest.mark.parametrize("case", _cases(16), ids=lambda c: f"B{c[0]}H{c[1]}N{c[2]}d{c[3]}{'c' if c[4] else ''}x{c[5]:g}")
def test_random_shapes_forward_and_both_backwards(case):
    B, H, N, d, causal, mult, seed = case
    inp = synth.attention_inputs(B, H, N, d, seed=seed, q_mult=mult)
    scale = 1.0 / math.sqrt(d)
    q, k, v, do = (gu.dev_bf16(inp[n + "_bits"]) for n in ("q", "k", "v", "do"))
    o, lse = fa.attention_forward(q, k, v, scale=scale, causal=causal)
    torch.cuda.synchronize()
    o_ref, lse_ref = oracle.attention_forward(inp["q"], inp["k"], inp["v"], scale, causal)
    gu.assert_o_lse(gu.to_f64(o), gu.to_f64(lse), o_ref, lse_ref, str(case))
    ref = oracle.attention_backward(inp["q"], inp["k"], inp["v"], inp["do"], scale, causal)
    for det in (False, True):
        got = fa.attention_backward(q, k, v, o, do, lse, scale=scale, causal=causal, deterministic=det)
        torch.cuda.synchronize()
        for name, g, r in zip(("dQ", "dK", "dV"), got, ref):
            g = gu.to_f64(g)
            assert np.all(np.isfinite(g)), (name, det, case)
            e = gu.rel_fro(g, r)
            assert e <= gu.GRAD_REL_FRO, f"{name} rel-Frobenius {e:.3e} det={det} {case}"
    assert fa.fa_device_status() == (0, 0)


def test_ragged_long_causal_d128_sampled():
    """A long ragged sequence (N = 20000 = 156 full tiles + 32 rows), causal,
    d = 128: sampled rows of the forward and of the gradients of two heads,
    sum identities on every head."""
    B, H, N, d = 1, 4, 20000, 128
    inp = synth.attention_inputs(B, H, N, d, seed=3100, want_f64=False)
    scale = 1.0 / math.sqrt(d)
    q, k, v, do = (gu.dev_bf16(inp[n + "_bits"]) for n in ("q", "k", "v", "do"))
    o, lse = fa.attention_forward(q, k, v, scale=scale, causal=True)
    dq, dk, dv = fa.attention_backward(q, k, v, o, do, lse, scale=scale, causal=True)
    torch.cuda.synchronize()
    o, lse, dq, dk, dv = (gu.to_f64(t) for t in (o, lse, dq, dk, dv))
    for h in (0, H - 1):
        rows = gu.sample_rows(N, 12, 3101 + h)
        cols = gu.sample_rows(N, 12, 3111 + h)
        qh, kh, vh, doh = (synth.head_f64(inp, n, 0, h) for n in ("q", "k", "v", "do"))
        o_ref, lse_ref = oracle.head_forward(qh, kh, vh, scale, True, rows=rows)
        gu.assert_o_lse(o[0, h][rows], lse[0, h][rows], o_ref, lse_ref, f"head {h}")
        rq, rk, rv = oracle.head_backward_sampled(qh, kh, vh, doh, scale, True, rows, cols)
        for name, g, r in zip(("dQ", "dK", "dV"), (dq[0, h][rows], dk[0, h][cols], dv[0, h][cols]), (rq, rk, rv)):
            assert gu.rel_fro(g, r) <= gu.GRAD_REL_FRO, (name, h)
    do_sum = np.stack([synth.head_f64(inp, "do", 0, h).sum(axis=0) for h in range(H)])
    assert np.max(np.abs(dk[0].sum(axis=1)) / np.linalg.norm(dk[0].reshape(H, -1), axis=1)[:, None]) <= 1e-2
    assert np.max(np.abs(dv[0].sum(axis=1) - do_sum) / np.linalg.norm(do_sum, axis=1)[:, None]) <= 1e-2
