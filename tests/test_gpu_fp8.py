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


# ------------------------------------------------------------ FP8 backward
def _fp8_bwd_inputs(B, H, N, d, seed):
    inp = synth.attention_inputs(B, H, N, d, seed=seed, storage="e4m3")
    do_bits = synth.to_bf16_bits(synth.normal_f32(seed, synth.TENSOR_IDS["do"], (B, H, N, d)))
    return inp, do_bits, synth.bf16_bits_to_f64(do_bits)


def _run_bwd_fp8(inp, do_bits, o, lse, causal, guarded=True):
    B, H, N, d = inp["shape"]
    scale = 1.0 / math.sqrt(d)
    q8, k8, v8 = (gu.dev_u8(inp[n + "_bits"]) for n in ("q", "k", "v"))
    do = gu.dev_bf16(do_bits)
    gs = [gu.Guarded((B, H, N, d), torch.bfloat16) for _ in range(3)]
    wg = gu.Guarded((fa.fa_bwd_fp8_workspace_size(B, H, N, d),), torch.uint8)
    fa.fa_bwd_fp8(q8, k8, v8, inp["q_descale"], inp["k_descale"], inp["v_descale"], o, do, lse,
                  gs[0].view, gs[1].view, gs[2].view, scale, causal, wg.view)
    torch.cuda.synchronize()
    assert all(g.intact() for g in gs) and wg.intact(), "write outside the output/workspace buffers"
    assert fa.fa_device_status() == (0, 0)
    return [gu.to_f64(g.view) for g in gs], scale


def test_fp8_bwd_single_key():
    """N = 1: P = 1, so dS = dO.V - dO.O vanishes and the exact dQ and dK are 0;
    a relative comparison is meaningless there.  The kernel's dS is then only
    the bf16 rounding of O (O = V * v_descale is not a bf16 value), so |dQ|
    and |dK| are bounded by scale * 2^-8 |dO||V| |K| (and |Q|); dV = dO."""
    B, H, N, d = 1, 2, 1, 128
    inp, do_bits, do = _fp8_bwd_inputs(B, H, N, d, seed=1251)
    scale = 1.0 / math.sqrt(d)
    o_ref, lse_ref = oracle.attention_forward(inp["q"], inp["k"], inp["v"], scale, False)
    o = torch.from_numpy(o_ref.astype(np.float32)).to(torch.bfloat16).cuda()
    lse = torch.from_numpy(lse_ref.astype(np.float32)).cuda()
    (dq, dk, dv), _ = _run_bwd_fp8(inp, do_bits, o, lse, False)
    ref = oracle.attention_backward(inp["q"], inp["k"], inp["v"], do, scale, False)
    assert np.all(ref[0] == 0.0) and np.all(ref[1] == 0.0)
    assert gu.rel_fro(dv, ref[2]) <= gu.GRAD_REL_FRO
    nrm = lambda x: np.linalg.norm(x, axis=-1)  # noqa: E731
    bound = scale * 2.0 ** -8 * nrm(do) * nrm(inp["v"])
    assert np.all(nrm(dq) <= bound * nrm(inp["k"]) + 1e-6)
    assert np.all(nrm(dk) <= bound * nrm(inp["q"]) + 1e-6)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("shape", [(1, 1, 128, 128), (1, 2, 7, 128), (2, 1, 300, 128), (1, 2, 1000, 128)])
def test_fp8_bwd_given_exact_forward_outputs(shape, causal):
    """The e4m3 backward on the oracle's own O (rounded to bf16) and LSE: what
    remains is the backward's arithmetic (bf16 P and dS, fp32 accumulation),
    held to the bf16 gradient tolerance against the oracle on the dequantised
    inputs."""
    B, H, N, d = shape
    inp, do_bits, do = _fp8_bwd_inputs(B, H, N, d, seed=1250 + N)
    scale = 1.0 / math.sqrt(d)
    o_ref, lse_ref = oracle.attention_forward(inp["q"], inp["k"], inp["v"], scale, causal)
    o = torch.from_numpy(o_ref.astype(np.float32)).to(torch.bfloat16).cuda()
    lse = torch.from_numpy(lse_ref.astype(np.float32)).cuda()
    got, _ = _run_bwd_fp8(inp, do_bits, o, lse, causal)
    ref = oracle.attention_backward(inp["q"], inp["k"], inp["v"], do, scale, causal)
    for name, g, r in zip(("dQ", "dK", "dV"), got, ref):
        assert np.all(np.isfinite(g)), name
        e = gu.rel_fro(g, r)
        assert e <= gu.GRAD_REL_FRO, f"{name} rel-Frobenius {e:.3e} {shape} causal={causal}"


@pytest.mark.parametrize("causal", [False, True])
def test_fp8_forward_then_backward(causal):
    """End to end: fa_fwd_fp8's O and LSE feed fa_bwd_fp8.  dV = P^T dO needs
    only LSE (accurate to 1e-3), so it keeps the bf16 gradient tolerance; dQ
    and dK see the forward's e4m3 P rounding through D = rowsum(dO o O), and
    take the FP8 output tolerance, 3e-2."""
    B, H, N, d = 2, 3, 1000, 128
    inp, do_bits, do = _fp8_bwd_inputs(B, H, N, d, seed=1251)
    q8, k8, v8 = (gu.dev_u8(inp[n + "_bits"]) for n in ("q", "k", "v"))
    o, lse = fa.attention_forward_fp8(q8, k8, v8, inp["q_descale"], inp["k_descale"], inp["v_descale"],
                                      causal=causal)
    got, scale = _run_bwd_fp8(inp, do_bits, o, lse, causal)
    ref = oracle.attention_backward(inp["q"], inp["k"], inp["v"], do, scale, causal)
    for name, g, r, tol in zip(("dQ", "dK", "dV"), got, ref, (gu.FP8_O_REL_FRO, gu.FP8_O_REL_FRO, gu.GRAD_REL_FRO)):
        e = gu.rel_fro(g, r)
        assert e <= tol, f"{name} rel-Frobenius {e:.3e} causal={causal}"


def test_fp8_bwd_config_b2_h16_n16384_d128_sampled():
    """The FP8 configuration's shape: sampled dQ rows and dK/dV columns of
    three heads against the oracle, and the gradient sum identities on all 32
    heads (sum_j dK_j = 0, sum_j dV_j = sum_i dO_i)."""
    B, H, N, d = 2, 16, 16384, 128
    inp = synth.attention_inputs(B, H, N, d, seed=1252, storage="e4m3", want_f64=False)
    do_bits = synth.to_bf16_bits(synth.normal_f32(1252, synth.TENSOR_IDS["do"], (B, H, N, d)))
    q8, k8, v8 = (gu.dev_u8(inp[n + "_bits"]) for n in ("q", "k", "v"))
    o, lse = fa.attention_forward_fp8(q8, k8, v8, inp["q_descale"], inp["k_descale"], inp["v_descale"])
    (dq, dk, dv), scale = _run_bwd_fp8(inp, do_bits, o, lse, False, guarded=True)
    do_sum = np.stack([synth.bf16_bits_to_f64(do_bits[b, h]).sum(axis=0) for b in range(B) for h in range(H)])
    dk_sum = dk.sum(axis=2).reshape(B * H, d)
    dv_sum = dv.sum(axis=2).reshape(B * H, d)
    dk_norm = np.linalg.norm(dk.reshape(B * H, -1), axis=1)[:, None]
    assert np.max(np.abs(dk_sum) / dk_norm) <= 1e-2
    assert np.max(np.abs(dv_sum - do_sum) / np.linalg.norm(do_sum, axis=1)[:, None]) <= 1e-2
    for (b, h) in ((0, 0), (1, 15), (0, 9)):
        rows = gu.sample_rows(N, 12, 3 + b * 16 + h)
        cols = gu.sample_rows(N, 12, 4 + b * 16 + h)
        qh, kh, vh = (synth.head_f64(inp, n, b, h) for n in ("q", "k", "v"))
        doh = synth.bf16_bits_to_f64(do_bits[b, h])
        rq, rk, rv = oracle.head_backward_sampled(qh, kh, vh, doh, scale, False, rows, cols)
        for name, g, r, tol in zip(("dQ", "dK", "dV"), (dq[b, h][rows], dk[b, h][cols], dv[b, h][cols]),
                                   (rq, rk, rv), (gu.FP8_O_REL_FRO, gu.FP8_O_REL_FRO, gu.GRAD_REL_FRO)):
            e = gu.rel_fro(g, r)
            assert e <= tol, f"{name} rel-Frobenius {e:.3e} head ({b},{h})"


def test_fp8_bwd_rejects_d64_and_bad_descales():
    x8 = torch.zeros((1, 1, 16, 64), dtype=torch.uint8, device="cuda")
    with pytest.raises(fa.FAError):
        fa.fa_bwd_fp8_workspace_size(1, 1, 16, 64)
    y8 = torch.zeros((1, 1, 16, 128), dtype=torch.uint8, device="cuda")
    y = torch.zeros((1, 1, 16, 128), dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros((1, 1, 16), dtype=torch.float32, device="cuda")
    outs = [torch.empty_like(y) for _ in range(3)]
    w = torch.empty(fa.fa_bwd_fp8_workspace_size(1, 1, 16, 128), dtype=torch.uint8, device="cuda")
    with pytest.raises(fa.FAError) as e:
        fa.fa_bwd_fp8(y8, y8, y8, 1.0, 0.0, 1.0, y, y, lse, *outs, 0.1, False, w)
    assert e.value.status == fa.STATUS_CODES["FA_ERR_INVALID_ARG"]
    small = torch.empty(fa.fa_bwd_workspace_size(1, 1, 16, 128), dtype=torch.uint8, device="cuda")
    with pytest.raises(fa.FAError) as e:
        fa.fa_bwd_fp8(y8, y8, y8, 1.0, 1.0, 1.0, y, y, lse, *outs, 0.1, False, small)
    assert e.value.status == fa.STATUS_CODES["FA_ERR_WORKSPACE"]
    del x8


@pytest.mark.parametrize("mult", [8.0, 64.0])
def test_fp8_large_score_range(mult):
    """Q scaled by a power of two before quantisation: peaked rows and frequent
    running-max moves.  The e4m3 forward takes its exponentials in half
    precision, so LSE is checked here at 1e-3 where the largest terms dominate
    the row sum."""
    inp = synth.attention_inputs(1, 2, 1024, 128, seed=77, q_mult=mult, storage="e4m3")
    for causal in (False, True):
        o, lse, scale = _run(inp, causal)
        o_ref, lse_ref = oracle.attention_forward(inp["q"], inp["k"], inp["v"], scale, causal)
        _check(o, lse, o_ref, lse_ref, f"mult={mult} causal={causal}")


def test_fp8_causal_forward_and_backward_b2_h16_n8192_d128_sampled():
    """Causal e4m3 forward and its backward at B2 H16 N8192: sampled rows of O
    and LSE, sampled dQ rows and dK/dV columns of two heads, and the gradient
    sum identities on all 32 heads."""
    B, H, N, d = 2, 16, 8192, 128
    inp = synth.attention_inputs(B, H, N, d, seed=1253, storage="e4m3", want_f64=False)
    do_bits = synth.to_bf16_bits(synth.normal_f32(1253, synth.TENSOR_IDS["do"], (B, H, N, d)))
    q8, k8, v8 = (gu.dev_u8(inp[n + "_bits"]) for n in ("q", "k", "v"))
    o, lse = fa.attention_forward_fp8(q8, k8, v8, inp["q_descale"], inp["k_descale"], inp["v_descale"], causal=True)
    (dq, dk, dv), scale = _run_bwd_fp8(inp, do_bits, o, lse, True)
    o64, lse64 = gu.to_f64(o), gu.to_f64(lse)
    do_sum = np.stack([synth.bf16_bits_to_f64(do_bits[b, h]).sum(axis=0) for b in range(B) for h in range(H)])
    dk_sum = dk.sum(axis=2).reshape(B * H, d)
    dv_sum = dv.sum(axis=2).reshape(B * H, d)
    assert np.max(np.abs(dk_sum) / np.linalg.norm(dk.reshape(B * H, -1), axis=1)[:, None]) <= 1e-2
    assert np.max(np.abs(dv_sum - do_sum) / np.linalg.norm(do_sum, axis=1)[:, None]) <= 1e-2
    for (b, h) in ((0, 0), (1, 15)):
        rows = gu.sample_rows(N, 12, 5 + b * 16 + h)
        cols = gu.sample_rows(N, 12, 6 + b * 16 + h)
        qh, kh, vh = (synth.head_f64(inp, n, b, h) for n in ("q", "k", "v"))
        doh = synth.bf16_bits_to_f64(do_bits[b, h])
        o_ref, lse_ref = oracle.head_forward(qh, kh, vh, scale, True, rows=rows)
        _check(o64[b, h][rows], lse64[b, h][rows], o_ref, lse_ref, f"head ({b},{h})")
        rq, rk, rv = oracle.head_backward_sampled(qh, kh, vh, doh, scale, True, rows, cols)
        for name, g, r, tol in zip(("dQ", "dK", "dV"), (dq[b, h][rows], dk[b, h][cols], dv[b, h][cols]),
                                   (rq, rk, rv), (gu.FP8_O_REL_FRO, gu.FP8_O_REL_FRO, gu.GRAD_REL_FRO)):
            e = gu.rel_fro(g, r)
            assert e <= tol, f"{name} rel-Frobenius {e:.3e} head ({b},{h})"
