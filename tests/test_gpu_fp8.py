"""GPU parity of the e4m3 forward (fa_fwd_fp8) against the fp64 oracle on the
dequantised inputs (the exact values x8 * descale the kernel sees).

Tolerances: O relative Frobenius <= 3e-2 (P is rounded to e4m3 for the PV
product).  LSE is checked at the bf16 forward's 1e-3: the scores come from
exact e4m3 products summed in fp32, so LSE carries no e4m3 rounding of P.
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


def _run(inp, causal):
    B, H, N, d = inp["shape"]
    scale = 1.0 / math.sqrt(d)
    q8, k8, v8 = (gu.dev_u8(inp[n + "_bits"]) for n in ("q", "k", "v"))
    o, lse = fa.attention_forward_fp8(q8, k8, v8, inp["q_descale"], inp["k_descale"], inp["v_descale"],
                                      scale=scale, causal=causal)
    torch.cuda.synchronize()
    assert fa.fa_device_status() == (0, 0)
    return gu.to_f64(o), gu.to_f64(lse), scale


def _check(o, lse, o_ref, lse_ref, what):
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(lse)), what
    e = gu.rel_fro(o, o_ref)
    assert e <= gu.FP8_O_REL_FRO, f"FP8 O rel-Frobenius {e:.3e} {what}"
    le = gu.max_abs(lse, lse_ref)
    assert le <= gu.LSE_MAX_ABS, f"FP8 LSE max-abs {le:.3e} {what}"


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("shape", [(1, 1, 128, 128), (1, 2, 1, 128), (2, 1, 300, 128), (1, 2, 1000, 128),
                                   (1, 1, 2049, 128)])
def test_fp8_small_parity(shape, causal):
    B, H, N, d = shape
    inp = synth.attention_inputs(B, H, N, d, seed=300 + N, storage="e4m3")
    o, lse, scale = _run(inp, causal)
    o_ref, lse_ref = oracle.attention_forward(inp["q"], inp["k"], inp["v"], scale, causal)
    _check(o, lse, o_ref, lse_ref, f"{shape} causal={causal}")


def test_fp8_config_b2_h16_n16384_d128_sampled():
    B, H, N, d = 2, 16, 16384, 128
    inp = synth.attention_inputs(B, H, N, d, seed=1239, storage="e4m3", want_f64=False)
    o, lse, scale = _run(inp, False)
    for (b, h) in ((0, 0), (1, 15), (0, 7)):
        rows = gu.sample_rows(N, 24, 5 + b * 16 + h)
        qh, kh, vh = (synth.head_f64(inp, n, b, h) for n in ("q", "k", "v"))
        o_ref, lse_ref = oracle.head_forward(qh, kh, vh, scale, False, rows=rows)
        _check(o[b, h][rows], lse[b, h][rows], o_ref, lse_ref, f"head ({b},{h})")
    assert np.all(np.isfinite(o))


def test_fp8_rejects_d64():
    x = torch.zeros((1, 1, 16, 64), dtype=torch.uint8, device="cuda")
    with pytest.raises(fa.FAError) as e:
        fa.attention_forward_fp8(x, x, x, 1.0, 1.0, 1.0)
    assert e.value.status == fa.STATUS_CODES["FA_ERR_UNSUPPORTED"]


def test_fp8_mixed_pair_single_grid_b4_h16_n2048_d128():
    """The e4m3 forward on the mixed grid (444 pair blocks, then 136 single
    Q-tile blocks on 148 SMs): every head in full against the oracle."""
    B, H, N, d = 4, 16, 2048, 128
    if torch.cuda.get_device_properties(0).multi_processor_count == 148:
        assert fa.fa_fwd_plan(B, H, N, d, False) == (580, 580, 444)
    inp = synth.attention_inputs(B, H, N, d, seed=1246, storage="e4m3")
    o, lse, scale = _run(inp, False)
    o_ref, lse_ref = oracle.attention_forward(inp["q"], inp["k"], inp["v"], scale, False)
    _check(o, lse, o_ref, lse_ref, "mixed grid")


@pytest.mark.parametrize("causal", [False, True])
def test_fp8_scale_zero_gives_the_mean_of_v(causal):
    B, H, N, d = 1, 2, 300, 128
    inp = synth.attention_inputs(B, H, N, d, seed=1247, storage="e4m3")
    q8, k8, v8 = (gu.dev_u8(inp[n + "_bits"]) for n in ("q", "k", "v"))
    o, lse = fa.attention_forward_fp8(q8, k8, v8, inp["q_descale"], inp["k_descale"], inp["v_descale"],
                                      scale=0.0, causal=causal)
    torch.cuda.synchronize()
    o_ref, lse_ref = oracle.attention_forward(inp["q"], inp["k"], inp["v"], 0.0, causal)
    _check(gu.to_f64(o), gu.to_f64(lse), o_ref, lse_ref, f"scale 0 causal={causal}")
