"""GPU parity of the split-KV decode path (fa_fwd_decode) against the fp64
rectangular oracle: Nq new queries over Nk cached keys, causal masking aligned
to the end of the cache."""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu

fa = pytest.importorskip("exact_io_aware_55_b200")


def _dev(inp):
    return tuple(gu.dev_bf16(inp[n + "_bits"]) for n in ("q", "k", "v"))


def _run(inp, causal, scale=None):
    B, H, Nq, Nk, d = inp["shape"]
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    q, k, v = _dev(inp)
    og = gu.Guarded((B, H, Nq, d), torch.bfloat16)
    lg = gu.Guarded((B, H, Nq), torch.float32)
    wbytes = fa.fa_fwd_decode_workspace_size(B, H, Nq, Nk, d)
    wg = gu.Guarded((max(16, wbytes),), torch.uint8)
    fa.fa_fwd_decode(q, k, v, og.view, lg.view, scale, causal, wg.view)
    torch.cuda.synchronize()
    assert og.intact() and lg.intact() and wg.intact(), "write outside the output or workspace buffers"
    return gu.to_f64(og.view), gu.to_f64(lg.view), scale


# (B, H, Nq, Nk, d): single key, ragged tails, Nq = Nk, one split (many heads)
# and hundreds of splits (one head, long cache)
SHAPES = [(1, 1, 1, 1, 64), (1, 2, 1, 37, 128), (2, 1, 3, 300, 64), (1, 1, 16, 16, 128), (1, 4, 16, 1000, 128),
          (2, 3, 5, 4097, 64), (1, 1, 1, 70001, 128), (4, 8, 1, 2048, 128), (2, 160, 2, 700, 64),
          (1, 1, 7, 257, 128)]


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("shape", SHAPES)
def test_decode_parity(shape, causal):
    B, H, Nq, Nk, d = shape
    inp = synth.decode_inputs(B, H, Nq, Nk, d, seed=500 + Nq + Nk + d)
    o, lse, scale = _run(inp, causal)
    o_ref, lse_ref = oracle.attention_forward_rect(inp["q"], inp["k"], inp["v"], scale, causal)
    gu.assert_o_lse(o, lse, o_ref, lse_ref, f"{shape} causal={causal}")


@pytest.mark.parametrize("mult", [8.0, 64.0])
def test_decode_large_score_range(mult):
    """Peaked softmax: running-max moves inside a tile, across warps and across splits."""
    inp = synth.decode_inputs(1, 2, 4, 5000, 128, seed=91, q_mult=mult)
    for causal in (False, True):
        o, lse, scale = _run(inp, causal)
        o_ref, lse_ref = oracle.attention_forward_rect(inp["q"], inp["k"], inp["v"], scale, causal)
        gu.assert_o_lse(o, lse, o_ref, lse_ref, f"mult={mult} causal={causal}")


def test_decode_rows_match_square_forward():
    """The decode of the last Nq rows equals those rows of the causal square forward."""
    B, H, N, d, nq = 1, 2, 1500, 128, 9
    inp = synth.attention_inputs(B, H, N, d, seed=92, with_grad=False)
    q, k, v = (gu.dev_bf16(inp[n + "_bits"]) for n in ("q", "k", "v"))
    o_sq, lse_sq = fa.attention_forward(q, k, v, causal=True)
    o_dec, lse_dec = fa.attention_decode(q[:, :, N - nq:].contiguous(), k, v, causal=True)
    torch.cuda.synchronize()
    o_ref, lse_ref = oracle.attention_forward_rect(inp["q"][:, :, N - nq:], inp["k"], inp["v"], d ** -0.5, True)
    gu.assert_o_lse(gu.to_f64(o_dec), gu.to_f64(lse_dec), o_ref, lse_ref)
    gu.assert_o_lse(gu.to_f64(o_sq[:, :, N - nq:]), gu.to_f64(lse_sq[:, :, N - nq:]), o_ref, lse_ref)


def test_decode_repeat_is_identical():
    """No atomics: two runs give the same bytes."""
    inp = synth.decode_inputs(2, 4, 3, 9000, 128, seed=93, want_f64=False)
    q, k, v = _dev(inp)
    o1, l1 = fa.attention_decode(q, k, v, causal=True)
    o2, l2 = fa.attention_decode(q, k, v, causal=True)
    torch.cuda.synchronize()
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16)) and torch.equal(l1, l2)


@pytest.mark.parametrize("causal", [False, True])
def test_decode_workload_b8_h32_nk16384_d128_sampled(causal):
    """The decode timing workload (8 x 32 heads, one query, 16384 cached keys,
    d = 128) at full size; a few heads checked against the oracle."""
    B, H, Nq, Nk, d = 8, 32, 1, 16384, 128
    inp = synth.decode_inputs(B, H, Nq, Nk, d, seed=94, want_f64=False)
    q, k, v = _dev(inp)
    o, lse = fa.attention_decode(q, k, v, causal=causal)
    torch.cuda.synchronize()
    o, lse = gu.to_f64(o), gu.to_f64(lse)
    for (b, h) in [(0, 0), (3, 17), (7, 31)]:
        qh, kh, vh = (synth.head_f64(inp, n, b, h) for n in ("q", "k", "v"))
        o_ref, lse_ref = oracle.head_forward_rect(qh, kh, vh, d ** -0.5, causal)
        gu.assert_o_lse(o[b, h], lse[b, h], o_ref, lse_ref, f"head {(b, h)}")


@pytest.mark.parametrize("causal", [False, True])
def test_decode_scale_zero(causal):
    """scale = 0 over several splits: uniform weights over the visible keys."""
    inp = synth.decode_inputs(1, 2, 3, 5000, 128, seed=93)
    o, lse, scale = _run(inp, causal, scale=0.0)
    o_ref, lse_ref = oracle.attention_forward_rect(inp["q"], inp["k"], inp["v"], 0.0, causal)
    gu.assert_o_lse(o, lse, o_ref, lse_ref, f"scale 0 causal={causal}")
