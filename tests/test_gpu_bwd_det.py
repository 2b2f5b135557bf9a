"""GPU parity of fa_bwd_deterministic (dQ from the query-tile pass, no
atomics) against the fp64 oracle, and its bit-reproducibility."""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu

fa = pytest.importorskip("exact_io_aware_55_b200")


def _run(inp, causal, reps=1):
    B, H, N, d = inp["shape"]
    scale = 1.0 / math.sqrt(d)
    q, k, v, do = (gu.dev_bf16(inp[n + "_bits"]) for n in ("q", "k", "v", "do"))
    o, lse = fa.attention_forward(q, k, v, scale=scale, causal=causal)
    outs = []
    for _ in range(reps):
        gs = [gu.Guarded((B, H, N, d), torch.bfloat16) for _ in range(3)]
        ws = gu.Guarded((max(16, fa.fa_bwd_workspace_size(B, H, N, d)),), torch.uint8)
        fa.fa_bwd_deterministic(q, k, v, o, do, lse, gs[0].view, gs[1].view, gs[2].view, scale, causal, ws.view)
        torch.cuda.synchronize()
        assert all(g.intact() for g in gs) and ws.intact()
        outs.append([g.view.clone() for g in gs])
    assert fa.fa_device_status() == (0, 0)
    return outs, scale, (q, k, v, o, do, lse)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("shape", [(1, 1, 128, 64), (1, 2, 1, 64), (2, 1, 129, 128), (1, 2, 300, 64),
                                   (1, 1, 513, 128), (1, 3, 1000, 64)])
def test_det_small_parity_and_repeatability(shape, causal):
    B, H, N, d = shape
    inp = synth.attention_inputs(B, H, N, d, seed=400 + N + d)
    outs, scale, _ = _run(inp, causal, reps=2)
    for a, b in zip(outs[0], outs[1]):                       # bit-identical across calls
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    ref = oracle.attention_backward(inp["q"], inp["k"], inp["v"], inp["do"], scale, causal)
    for name, g, r in zip(("dQ", "dK", "dV"), outs[0], ref):
        e = gu.rel_fro(gu.to_f64(g), r)
        assert e <= gu.GRAD_REL_FRO, f"{name} {e:.3e} {shape} causal={causal}"


def test_det_matches_atomic_backward():
    inp = synth.attention_inputs(2, 4, 1024, 128, seed=411, q_mult=8.0)
    outs, scale, (q, k, v, o, do, lse) = _run(inp, True)
    ref = fa.attention_backward(q, k, v, o, do, lse, scale=scale, causal=True)
    for g, r in zip(outs[0], ref):
        assert gu.rel_fro(gu.to_f64(g), gu.to_f64(r)) <= 5e-3


def test_det_config_b2_h16_n8192_d128_causal_sampled():
    B, H, N, d = 2, 16, 8192, 128
    inp = synth.attention_inputs(B, H, N, d, seed=1237, want_f64=False)
    outs, scale, _ = _run(inp, True)
    dq = gu.to_f64(outs[0][0])
    for (b, h) in ((0, 0), (1, 15)):
        rows = gu.sample_rows(N, 12, 17 * b + h)
        qh, kh, vh, doh = (synth.head_f64(inp, n, b, h) for n in ("q", "k", "v", "do"))
        rq, _, _ = oracle.head_backward_sampled(qh, kh, vh, doh, scale, True, rows, rows[:2])
        assert gu.rel_fro(dq[b, h][rows], rq) <= gu.GRAD_REL_FRO


def test_det_matches_atomic_partial_head_group_b2_h5_n16384_d128_causal():
    """Ten heads at N=16384: both causal grids order heads in groups of four,
    the last group holding two; the atomic-free dQ pass and the atomic one agree."""
    inp = synth.attention_inputs(2, 5, 16384, 128, seed=412, want_f64=False)
    outs, scale, (q, k, v, o, do, lse) = _run(inp, True)
    ref = fa.attention_backward(q, k, v, o, do, lse, scale=scale, causal=True)
    for g, r in zip(outs[0], ref):
        assert gu.rel_fro(gu.to_f64(g), gu.to_f64(r)) <= 5e-3
