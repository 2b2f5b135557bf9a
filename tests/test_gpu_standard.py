"""GPU parity of the standard (materialising) attention baseline
(fa_fwd_standard) against the fp64 oracle, and agreement with the fused
kernel on the same inputs."""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu

fa = pytest.importorskip("exact_io_aware_55_b200")


def _run(inp, causal, scale=None):
    B, H, N, d = inp["shape"]
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    q, k, v = (gu.dev_bf16(inp[n + "_bits"]) for n in ("q", "k", "v"))
    og = gu.Guarded((B, H, N, d), torch.bfloat16)
    lg = gu.Guarded((B, H, N), torch.float32)
    wg = gu.Guarded((fa.fa_fwd_standard_workspace_size(B, H, N, d),), torch.uint8)
    fa.fa_fwd_standard(q, k, v, og.view, lg.view, scale, causal, wg.view)
    torch.cuda.synchronize()
    assert og.intact() and lg.intact() and wg.intact(), "write outside the output or workspace buffers"
    return gu.to_f64(og.view), gu.to_f64(lg.view), scale, (q, k, v)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("shape", [(1, 1, 1, 64), (1, 2, 17, 128), (2, 1, 128, 64), (1, 1, 129, 128),
                                   (1, 3, 300, 64), (2, 2, 513, 128), (1, 1, 1000, 64)])
def test_standard_parity(shape, causal):
    inp = synth.attention_inputs(*shape, seed=700 + sum(shape), with_grad=False)
    o, lse, scale, _ = _run(inp, causal)
    o_ref, lse_ref = oracle.attention_forward(inp["q"], inp["k"], inp["v"], scale, causal)
    gu.assert_o_lse(o, lse, o_ref, lse_ref, f"{shape} causal={causal}")


@pytest.mark.parametrize("causal", [False, True])
def test_standard_matches_fused_b4_h16_n2048_d64(causal):
    """The bench shape: the baseline and the fused kernel agree with each other
    and, on sampled heads and rows, with the oracle."""
    B, H, N, d = 4, 16, 2048, 64
    inp = synth.attention_inputs(B, H, N, d, seed=710, with_grad=False, want_f64=False)
    o, lse, scale, (q, k, v) = _run(inp, causal)
    of, lf = fa.attention_forward(q, k, v, scale=scale, causal=causal)
    torch.cuda.synchronize()
    of, lf = gu.to_f64(of), gu.to_f64(lf)
    assert gu.rel_fro(o, of) <= 2 * gu.O_REL_FRO and gu.max_abs(lse, lf) <= gu.LSE_MAX_ABS
    for (b, h) in [(0, 0), (3, 15)]:
        rows = gu.sample_rows(N, 16, 711 + h)
        qh, kh, vh = (synth.head_f64(inp, n, b, h) for n in ("q", "k", "v"))
        o_ref, lse_ref = oracle.head_forward(qh, kh, vh, scale, causal, rows=rows)
        gu.assert_o_lse(o[b, h, rows], lse[b, h, rows], o_ref, lse_ref, f"head {(b, h)}")


@pytest.mark.parametrize("causal", [False, True])
def test_standard_scale_zero(causal):
    inp = synth.attention_inputs(1, 2, 300, 64, seed=1248, with_grad=False)
    o, lse, _, _ = _run(inp, causal, scale=0.0)
    o_ref, lse_ref = oracle.attention_forward(inp["q"], inp["k"], inp["v"], 0.0, causal)
    gu.assert_o_lse(o, lse, o_ref, lse_ref, f"scale 0 causal={causal}")
