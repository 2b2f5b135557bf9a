"""GPU parity of the bf16 backward (fa_bwd) against the fp64 oracle.

The device backward consumes the device forward's O and LSE, as a caller
would; the oracle computes everything from the same rounded Q, K, V, dO.
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


def _device_inputs(inp):
    return tuple(gu.dev_bf16(inp[n + "_bits"]) for n in ("q", "k", "v", "do"))


def _run(inp, causal, scale=None, guarded=False):
    B, H, N, d = inp["shape"]
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    q, k, v, do = _device_inputs(inp)
    o, lse = fa.attention_forward(q, k, v, scale=scale, causal=causal)
    if guarded:
        gs = [gu.Guarded((B, H, N, d), torch.bfloat16) for _ in range(3)]
        wsz = fa.fa_bwd_workspace_size(B, H, N, d)
        wg = gu.Guarded((max(wsz, 16),), torch.uint8)
        fa.fa_bwd(q, k, v, o, do, lse, gs[0].view, gs[1].view, gs[2].view, scale, causal, wg.view)
        torch.cuda.synchronize()
        assert all(g.intact() for g in gs) and wg.intact(), "write outside the output/workspace buffers"
        dq, dk, dv = (g.view for g in gs)
    else:
        dq, dk, dv = fa.attention_backward(q, k, v, o, do, lse, scale=scale, causal=causal)
        torch.cuda.synchronize()
    assert fa.fa_device_status() == (0, 0)
    return tuple(gu.to_f64(t) for t in (dq, dk, dv)), scale


def _assert_grads(got, ref, what=""):
    for name, g, r in zip(("dQ", "dK", "dV"), got, ref):
        assert np.all(np.isfinite(g)), f"non-finite {name} {what}"
        e = gu.rel_fro(g, r)
        assert e <= gu.GRAD_REL_FRO, f"{name} rel-Frobenius {e:.3e} > {gu.GRAD_REL_FRO} {what}"


SMALL = [(1, 1, 128, 64), (1, 2, 1, 64), (1, 1, 17, 128), (2, 1, 127, 64), (1, 1, 129, 128),
         (1, 2, 300, 64), (1, 1, 300, 128), (2, 2, 513, 128), (1, 3, 1000, 64), (1, 1, 640, 128)]


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("shape", SMALL)
def test_bwd_small_parity(shape, causal):
    B, H, N, d = shape
    inp = synth.attention_inputs(B, H, N, d, seed=200 + N + d)
    got, scale = _run(inp, causal, guarded=True)
    ref = oracle.attention_backward(inp["q"], inp["k"], inp["v"], inp["do"], scale, causal)
    _assert_grads(got, ref, f"{shape} causal={causal}")


def test_bwd_pr1_reference_case():
    inp = synth.attention_inputs_f32_to_bf16(1, 1, 128, 64, seed=1234)
    got, scale = _run(inp, False, scale=1.0 / 8.0)
    ref = oracle.attention_backward(inp["q"], inp["k"], inp["v"], inp["do"], scale, False)
    _assert_grads(got, ref)


@pytest.mark.parametrize("mult", [8.0])
def test_bwd_large_score_range(mult):
    inp = synth.attention_inputs(1, 2, 1024, 128, seed=78, q_mult=mult)
    for causal in (False, True):
        got, scale = _run(inp, causal)
        ref = oracle.attention_backward(inp["q"], inp["k"], inp["v"], inp["do"], scale, causal)
        _assert_grads(got, ref, f"mult={mult} causal={causal}")


def test_bwd_config_b4_h16_n2048_d64_full():
    inp = synth.attention_inputs(4, 16, 2048, 64, seed=1236)
    got, scale = _run(inp, False)
    ref = oracle.attention_backward(inp["q"], inp["k"], inp["v"], inp["do"], scale, False)
    _assert_grads(got, ref)


def _sampled(B, H, N, d, causal, seed, q_mult=1.0, n_heads=2, n_rows=16):
    inp = synth.attention_inputs(B, H, N, d, seed=seed, q_mult=q_mult, want_f64=False)
    (dq, dk, dv), scale = _run(inp, causal)
    # sum identities on every head: sum_j dK_j = 0 and sum_j dV_j = sum_i dO_i
    do_sum = np.stack([synth.head_f64(inp, "do", b, h).sum(axis=0) for b in range(B) for h in range(H)])
    dk_sum = dk.sum(axis=2).reshape(B * H, d)
    dv_sum = dv.sum(axis=2).reshape(B * H, d)
    dk_norm = np.linalg.norm(dk.reshape(B * H, -1), axis=1)[:, None]
    assert np.max(np.abs(dk_sum) / dk_norm) <= 1e-2
    assert np.max(np.abs(dv_sum - do_sum) / np.linalg.norm(do_sum, axis=1)[:, None]) <= 1e-2
    rng = np.random.default_rng(seed)
    heads = {(0, 0), (B - 1, H - 1)}
    while len(heads) < min(n_heads, B * H):
        heads.add((int(rng.integers(B)), int(rng.integers(H))))
    for (b, h) in sorted(heads):
        rows = gu.sample_rows(N, n_rows, seed + 7 * b + h)
        cols = gu.sample_rows(N, n_rows, seed + 11 * b + h + 1)
        qh, kh, vh, doh = (synth.head_f64(inp, n, b, h) for n in ("q", "k", "v", "do"))
        rq, rk, rv = oracle.head_backward_sampled(qh, kh, vh, doh, scale, causal, rows, cols)
        _assert_grads((dq[b, h][rows], dk[b, h][cols], dv[b, h][cols]), (rq, rk, rv), f"head ({b},{h})")


@pytest.mark.parametrize("q_mult", [1.0, 8.0])
def test_bwd_config_b2_h16_n8192_d128_causal_sampled(q_mult):
    _sampled(2, 16, 8192, 128, True, seed=1237, q_mult=q_mult)


def test_bwd_config_b1_h32_n32768_d128_causal_sampled():
    _sampled(1, 32, 32768, 128, True, seed=1238, n_heads=1, n_rows=12)


def test_bwd_causal_partial_head_group_b2_h5_n16384_d128_sampled():
    """Ten heads at N=16384, d=128: the causal grid orders heads in groups of
    four (Q, dO and the fp32 dQ rows of a head are 16 MiB against a 64 MiB
    budget), so the last group holds two heads."""
    _sampled(2, 5, 16384, 128, True, seed=1240, n_heads=3, n_rows=12)


def test_bwd_workspace_checks():
    x = torch.zeros((1, 1, 64, 64), dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros((1, 1, 64), dtype=torch.float32, device="cuda")
    outs = [torch.empty_like(x) for _ in range(3)]
    small = torch.empty(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(fa.FAError) as e:
        fa.fa_bwd(x, x, x, x, x, lse, *outs, 0.125, False, small)
    assert e.value.status == fa.STATUS_CODES["FA_ERR_WORKSPACE"]
    assert fa.fa_bwd_workspace_size(1, 1, 0, 64) == 0


def test_bwd_noncausal_b1_h32_n8192_d128_sampled():
    """The non-causal d = 128 backward at N = 8192 (the long-sequence shape
    the benchmark's backward fraction is quoted on): sampled dQ rows and
    dK/dV columns of four heads against the oracle, sum identities on all 32."""
    _sampled(1, 32, 8192, 128, False, seed=1244, n_heads=4, n_rows=16)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_bwd_scale_zero(d, causal):
    """scale = 0: S does not depend on Q or K, so dQ = dK = 0 exactly, and
    dV = P^T dO with P the uniform (prefix-uniform when causal) weights."""
    inp = synth.attention_inputs(1, 2, 300, d, seed=1245 + d)
    (dq, dk, dv), _ = _run(inp, causal, scale=0.0, guarded=True)
    assert np.all(dq == 0.0) and np.all(dk == 0.0)
    ref = oracle.attention_backward(inp["q"], inp["k"], inp["v"], inp["do"], 0.0, causal)
    assert np.all(ref[0] == 0.0) and np.all(ref[1] == 0.0)
    e = gu.rel_fro(dv, ref[2])
    assert e <= gu.GRAD_REL_FRO, e


@pytest.mark.parametrize("d,causal", [(64, False), (128, True)])
def test_bwd_events_matches_fa_bwd_and_orders_its_events(d, causal):
    """fa_bwd_events computes what fa_bwd computes (dK, dV byte for byte; dQ
    within the tolerance, its fp32 atomics reorder) and its four events bound
    the preprocess, the main kernel and the dQ conversion in that order."""
    B, H, N = 2, 3, 1000
    inp = synth.attention_inputs(B, H, N, d, seed=1249 + d, want_f64=False)
    q, k, v, do = _device_inputs(inp)
    scale = 1.0 / math.sqrt(d)
    o, lse = fa.attention_forward(q, k, v, scale=scale, causal=causal)
    ref = fa.attention_backward(q, k, v, o, do, lse, scale=scale, causal=causal)
    outs = [torch.empty_like(q) for _ in range(3)]
    work = torch.empty(fa.fa_bwd_workspace_size(B, H, N, d), dtype=torch.uint8, device="cuda")
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
    fa.fa_bwd_events(q, k, v, o, do, lse, *outs, scale, causal, work, ev)
    torch.cuda.synchronize()
    assert torch.equal(outs[1].view(torch.int16), ref[1].view(torch.int16))
    assert torch.equal(outs[2].view(torch.int16), ref[2].view(torch.int16))
    assert gu.rel_fro(gu.to_f64(outs[0]), gu.to_f64(ref[0])) <= 1e-3
    parts = [ev[i].elapsed_time(ev[i + 1]) for i in range(3)]
    assert all(p >= 0.0 for p in parts) and parts[1] > 0.0
    assert fa.fa_device_status() == (0, 0)


def _bf16_round(x):
    """Round float64 values to bf16 (through float32, round to nearest even)."""
    b = np.asarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    b = ((b + 0x7FFF + ((b >> 16) & 1)) >> 16) << 16
    return b.astype(np.uint32).view(np.float32).astype(np.float64)


def _bf16_rounding_reference(inp, o_dev, lse_dev, scale, causal):
    """The backward's definition with P and dS rounded to bf16 where the
    kernels round them (P for dV; dS, formed from the unrounded P, for dQ and
    dK), from the device's own O and LSE.  Test-only: it pins where the device
    path rounds, on problems where the fp64 result is not well conditioned."""
    q, k, v, do = (inp[n] for n in ("q", "k", "v", "do"))
    B, H, N, d = q.shape
    dq, dk, dv = np.zeros_like(q), np.zeros_like(q), np.zeros_like(q)
    for b in range(B):
        for h in range(H):
            s = scale * q[b, h] @ k[b, h].T
            if causal:
                s = np.where(np.tril(np.ones((N, N), bool)), s, -np.inf)
            p = np.exp(s - lse_dev[b, h][:, None])
            dvec = (do[b, h] * o_dev[b, h]).sum(1, keepdims=True)
            dv[b, h] = _bf16_round(p).T @ do[b, h]
            ds = _bf16_round(p * (do[b, h] @ v[b, h].T - dvec))
            dq[b, h] = scale * ds @ k[b, h]
            dk[b, h] = scale * ds.T @ q[b, h]
    return dq, dk, dv


# Tiny, peaked problems (from a seeded random sweep) where dP - D cancels: the
# gradients were 1.1e-2 to 3.4e-2 from the fp64 oracle, all of it the bf16
# rounding of dS, which every bf16 implementation of the method performs.
TINY_PEAKED = [(2, 1, 4, 64, False, 8.0, 986825433), (1, 1, 2, 128, True, 1.0, 87362969),
               (1, 1, 8, 128, False, 8.0, 714526692)]


@pytest.mark.parametrize("deterministic", [False, True])
@pytest.mark.parametrize("case", TINY_PEAKED)
def test_bwd_tiny_peaked_matches_bf16_rounding_reference(case, deterministic):
    B, H, N, d, causal, mult, seed = case
    inp = synth.attention_inputs(B, H, N, d, seed=seed, q_mult=mult)
    q, k, v, do = _device_inputs(inp)
    scale = 1.0 / math.sqrt(d)
    o, lse = fa.attention_forward(q, k, v, scale=scale, causal=causal)
    dq, dk, dv = (torch.empty_like(q) for _ in range(3))
    work = torch.empty(max(16, fa.fa_bwd_workspace_size(B, H, N, d)), dtype=torch.uint8, device="cuda")
    (fa.fa_bwd_deterministic if deterministic else fa.fa_bwd)(q, k, v, o, do, lse, dq, dk, dv, scale, causal, work)
    torch.cuda.synchronize()
    ref = _bf16_rounding_reference(inp, gu.to_f64(o), gu.to_f64(lse), scale, causal)
    for name, g, r in zip(("dQ", "dK", "dV"), (dq, dk, dv), ref):
        e = gu.rel_fro(gu.to_f64(g), r)
        assert e <= 5e-3, f"{name} {e:.3e} against the bf16-rounding reference {case}"
    assert fa.fa_device_status() == (0, 0)
