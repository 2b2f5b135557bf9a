"""GPU parity of the bf16 forward (fa_fwd) against the fp64 oracle."""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu

fa = pytest.importorskip("exact_io_aware_55_b200")


def _run_fwd(inp, causal, scale=None, guarded=False):
    B, H, N, d = inp["shape"]
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    q, k, v = (gu.dev_bf16(inp[n + "_bits"]) for n in ("q", "k", "v"))
    if guarded:
        og = gu.Guarded((B, H, N, d), torch.bfloat16)
        lg = gu.Guarded((B, H, N), torch.float32)
        fa.fa_fwd(q, k, v, og.view, lg.view, scale, causal)
        torch.cuda.synchronize()
        assert og.intact() and lg.intact(), "write outside the output buffers"
        return gu.to_f64(og.view), gu.to_f64(lg.view), scale
    o, lse = fa.attention_forward(q, k, v, scale=scale, causal=causal)
    torch.cuda.synchronize()
    return gu.to_f64(o), gu.to_f64(lse), scale


SMALL = [(1, 1, 128, 64), (1, 2, 1, 64), (1, 1, 17, 128), (2, 1, 127, 64), (1, 1, 129, 128),
         (1, 2, 300, 64), (1, 1, 300, 128), (2, 2, 513, 128), (1, 3, 1000, 64), (1, 1, 640, 128)]


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("shape", SMALL)
def test_fwd_small_parity(shape, causal):
    B, H, N, d = shape
    inp = synth.attention_inputs(B, H, N, d, seed=100 + N + d, with_grad=False)
    o, lse, scale = _run_fwd(inp, causal, guarded=True)
    o_ref, lse_ref = oracle.attention_forward(inp["q"], inp["k"], inp["v"], scale, causal)
    gu.assert_o_lse(o, lse, o_ref, lse_ref, f"{shape} causal={causal}")


def test_fwd_pr1_reference_case():
    """Single head, B=1 H=1 N=128 d=64, fp32 N(0,1) draws rounded to bf16."""
    inp = synth.attention_inputs_f32_to_bf16(1, 1, 128, 64, seed=1234)
    o, lse, scale = _run_fwd(inp, False, scale=1.0 / 8.0)
    o_ref, lse_ref = oracle.attention_forward(inp["q"], inp["k"], inp["v"], scale, False)
    gu.assert_o_lse(o, lse, o_ref, lse_ref)


@pytest.mark.parametrize("mult", [8.0, 64.0])
def test_fwd_large_score_range(mult):
    """Q scaled by a power of two: frequent running-max moves and rescales."""
    inp = synth.attention_inputs(1, 2, 1024, 128, seed=77, q_mult=mult, with_grad=False)
    for causal in (False, True):
        o, lse, scale = _run_fwd(inp, causal)
        o_ref, lse_ref = oracle.attention_forward(inp["q"], inp["k"], inp["v"], scale, causal)
        gu.assert_o_lse(o, lse, o_ref, lse_ref, f"mult={mult} causal={causal}")


def test_fwd_config_b4_h16_n2048_d64_full():
    inp = synth.attention_inputs(4, 16, 2048, 64, seed=1236, with_grad=False)
    o, lse, scale = _run_fwd(inp, False)
    o_ref, lse_ref = oracle.attention_forward(inp["q"], inp["k"], inp["v"], scale, False)
    gu.assert_o_lse(o, lse, o_ref, lse_ref)


def test_fwd_d64_persistent_items_ragged_b2_h40_n1000():
    """d = 64, non-causal: 80 heads x 4 Q-tile pairs = 320 pairs on 148 SMs.
    The last 24 pairs are split into 48 single-tile items (344 items), so each
    persistent CTA takes two or three items, single tiles among them.  Every
    head's last Q tile and last K/V tile are ragged (104 of 128 rows), and the
    output buffers are guarded against writes outside them."""
    inp = synth.attention_inputs(2, 40, 1000, 64, seed=1241, with_grad=False)
    o, lse, scale = _run_fwd(inp, False, guarded=True)
    o_ref, lse_ref = oracle.attention_forward(inp["q"], inp["k"], inp["v"], scale, False)
    gu.assert_o_lse(o, lse, o_ref, lse_ref)


def _sampled_check(B, H, N, d, causal, seed, q_mult=1.0, n_heads=3, n_rows=24):
    inp = synth.attention_inputs(B, H, N, d, seed=seed, q_mult=q_mult, with_grad=False, want_f64=False)
    o, lse, scale = _run_fwd(inp, causal)
    rng = np.random.default_rng(seed)
    heads = {(0, 0), (B - 1, H - 1)}
    while len(heads) < min(n_heads, B * H):
        heads.add((int(rng.integers(B)), int(rng.integers(H))))
    for (b, h) in sorted(heads):
        rows = gu.sample_rows(N, n_rows, seed + 31 * b + h)
        qh, kh, vh = (synth.head_f64(inp, n, b, h) for n in ("q", "k", "v"))
        o_ref, lse_ref = oracle.head_forward(qh, kh, vh, scale, causal, rows=rows)
        gu.assert_o_lse(o[b, h][rows], lse[b, h][rows], o_ref, lse_ref, f"head ({b},{h})")
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(lse))


@pytest.mark.parametrize("q_mult", [1.0, 8.0])
def test_fwd_config_b2_h16_n8192_d128_causal_sampled(q_mult):
    _sampled_check(2, 16, 8192, 128, True, seed=1237, q_mult=q_mult)


def test_fwd_config_b2_h16_n8192_d128_causal_q8_every_head():
    """The large-score-range run of the causal B2 H16 N8192 d128 configuration
    (Q x 8) against the oracle on every element of every head, not a sample:
    with a peaked softmax, O sits next to single V rows, so this is where the
    O max-abs bound is tightest (about 30 s of oracle time)."""
    B, H, N, d = 2, 16, 8192, 128
    inp = synth.attention_inputs(B, H, N, d, seed=1237, q_mult=8.0, with_grad=False, want_f64=False)
    o, lse, scale = _run_fwd(inp, True)
    for b in range(B):
        for h in range(H):
            qh, kh, vh = (synth.head_f64(inp, n, b, h) for n in ("q", "k", "v"))
            o_ref, lse_ref = oracle.head_forward(qh, kh, vh, scale, True)
            gu.assert_o_lse(o[b, h], lse[b, h], o_ref, lse_ref, f"head ({b},{h})")


def test_fwd_config_b1_h32_n32768_d128_causal_sampled():
    _sampled_check(1, 32, 32768, 128, True, seed=1238, n_heads=2, n_rows=16)


def test_fwd_causal_partial_head_group_b2_h5_n16384_d128_sampled():
    """Ten heads at N=16384, d=128: K and V of a head are 8 MiB, so the causal
    grid orders heads in groups of eight and the last group holds two."""
    _sampled_check(2, 5, 16384, 128, True, seed=1240, n_heads=3, n_rows=16)


def test_fwd_noncausal_n8192_d128_sampled():
    _sampled_check(1, 32, 8192, 128, False, seed=1239, n_heads=6)


def test_fwd_empty_and_errors():
    q = torch.zeros((1, 1, 0, 64), dtype=torch.bfloat16, device="cuda")
    o, lse = fa.attention_forward(q, q, q)
    assert o.shape == (1, 1, 0, 64)
    x = torch.zeros((1, 1, 8, 96), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(fa.FAError) as e:
        fa.attention_forward(x, x, x)
    assert e.value.status == fa.STATUS_CODES["FA_ERR_UNSUPPORTED"]
    y = torch.zeros((1, 1, 8, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(fa.FAError) as e:
        fa.attention_forward(y, y, y, scale=-1.0)
    assert e.value.status == fa.STATUS_CODES["FA_ERR_INVALID_ARG"]
    assert fa.lib.fa_get_device_status(None) == 0
    assert fa.fa_device_status() == (0, 0)


def test_watchdog_selftest_times_out_cleanly():
    fa.fa_device_status()                      # clear
    fa.fa_watchdog_selftest(2000)              # 2 ms wait that nobody satisfies
    st, where = fa.fa_device_status()
    assert st == fa.STATUS_CODES["FA_ERR_DEVICE_TIMEOUT"] and where == 99
    assert fa.fa_device_status() == (0, 0)     # cleared, context still usable
    inp = synth.attention_inputs(1, 1, 64, 64, seed=5, with_grad=False)
    o, lse, scale = _run_fwd(inp, False)
    o_ref, lse_ref = oracle.attention_forward(inp["q"], inp["k"], inp["v"], scale, False)
    gu.assert_o_lse(o, lse, o_ref, lse_ref)


def test_fwd_mixed_pair_single_grid_b4_h16_n2048_d128_full():
    """d = 128 non-causal at B4 H16 N2048: 512 Q-tile pairs on 148 SMs leave a
    last round of 68 pairs, which the forward splits into 136 single-tile
    blocks dispatched after 444 pair blocks.  Every head is checked in full, so
    both kinds of block are covered."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    ctas, items, pair_items = fa.fa_fwd_plan(4, 16, 2048, 128, False)
    rem = 512 % sms
    if 0 < 2 * rem <= sms:
        assert (ctas, items, pair_items) == (512 + rem, 512 + rem, 512 - rem)
    if sms == 148:
        assert pair_items == 444 and items == 580
    inp = synth.attention_inputs(4, 16, 2048, 128, seed=1242, with_grad=False)
    o, lse, scale = _run_fwd(inp, False, guarded=True)
    o_ref, lse_ref = oracle.attention_forward(inp["q"], inp["k"], inp["v"], scale, False)
    gu.assert_o_lse(o, lse, o_ref, lse_ref)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_fwd_scale_zero_gives_the_mean_of_v(d, causal):
    """scale = 0: every visible key has the same weight, so O_i is the mean of
    the visible V rows (the prefix mean when causal) and LSE_i = ln(count)."""
    B, H, N = 1, 2, 300
    inp = synth.attention_inputs(B, H, N, d, seed=1243 + d, with_grad=False)
    o, lse, _ = _run_fwd(inp, causal, scale=0.0, guarded=True)
    v = inp["v"]
    if causal:
        cnt = np.arange(1, N + 1, dtype=np.float64)
        o_ref = np.cumsum(v, axis=2) / cnt[None, None, :, None]
        lse_ref = np.broadcast_to(np.log(cnt), (B, H, N))
    else:
        o_ref = np.broadcast_to(v.mean(axis=2, keepdims=True), v.shape)
        lse_ref = np.full((B, H, N), np.log(N))
    gu.assert_o_lse(o, lse, o_ref, lse_ref, f"scale 0 d={d} causal={causal}")
    o2, l2 = oracle.attention_forward(inp["q"], inp["k"], inp["v"], 0.0, causal)
    gu.assert_o_lse(o, lse, o2, l2, "against the oracle")


def test_fwd_noncausal_n8192_d128_every_head_in_the_convex_hull():
    """All 32 heads of B1 H32 N8192 d128 non-causal: each O entry lies between
    the smallest and largest V entry of its column (a softmax average), up to
    the bf16 rounding of O, and LSE_i >= max_j s_ij (checked on the sampled
    rows of three heads against the oracle in the test above)."""
    B, H, N, d = 1, 32, 8192, 128
    inp = synth.attention_inputs(B, H, N, d, seed=1239, with_grad=False, want_f64=False)
    q, k, v = (gu.dev_bf16(inp[n + "_bits"]) for n in ("q", "k", "v"))
    o, lse = fa.attention_forward(q, k, v, scale=1.0 / math.sqrt(d), causal=False)
    torch.cuda.synchronize()
    of, vf = o.float(), v.float()
    vmin, vmax = vf.amin(dim=2, keepdim=True), vf.amax(dim=2, keepdim=True)
    slack = 2.0 ** -8 * torch.maximum(vmin.abs(), vmax.abs())
    assert bool(torch.all(of >= vmin - slack)) and bool(torch.all(of <= vmax + slack))
    assert bool(torch.all(torch.isfinite(lse)))
    # LSE lies in [max_j s_ij, max_j s_ij + ln N]; the row max from a bf16-exact
    # fp32 product on the device (test-side check, one head at a time)
    for h in range(H):
        s = (q[0, h].float() @ k[0, h].float().T) / math.sqrt(d)
        m = s.amax(dim=1)
        assert bool(torch.all(lse[0, h] >= m - 1e-3)) and bool(torch.all(lse[0, h] <= m + math.log(N) + 1e-3)), h
