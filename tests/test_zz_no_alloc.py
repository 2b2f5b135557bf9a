"""fa_bwd_noalloc: the backward for callers that cannot allocate device memory.

Such callers -- a plugin running inside a framework that owns every device
allocation, or a serving loop that reserves all its memory at start-up and
must not call cudaMalloc afterwards -- get the same backward with no caller
workspace: the scratch is a fixed array inside the library.  These tests call
the entry point through the C ABI (raw pointers via ctypes) and check, on two
calls in a row, that it returns what fa_bwd returns with a caller workspace:
dK and dV byte for byte, dQ (fp32 atomics) within the gradient tolerance the
parity tests use.  The file is named to be
collected last.
"""
import ctypes
import math

import numpy as np
import pytest
import torch

import synth
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu

fa = pytest.importorskip("exact_io_aware_55_b200")


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def _call_noalloc(q, k, v, o, do, lse, dq, dk, dv, scale, causal):
    B, H, N, d = q.shape
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return fa.lib.fa_bwd_noalloc(_p(q), _p(k), _p(v), _p(o), _p(do), _p(lse), _p(dq), _p(dk), _p(dv),
                                 B, H, N, d, ctypes.c_float(scale), int(causal), stream)


def _case(shape, causal, seed):
    B, H, N, d = shape
    assert fa.fa_bwd_workspace_size(B, H, N, d) <= fa.lib.fa_bwd_noalloc_max_bytes()
    inp = synth.attention_inputs(B, H, N, d, seed=seed, want_f64=False)
    q, k, v, do = (gu.dev_bf16(inp[n + "_bits"]) for n in ("q", "k", "v", "do"))
    scale = 1.0 / math.sqrt(d)
    o, lse = fa.attention_forward(q, k, v, scale=scale, causal=causal)
    ref = fa.attention_backward(q, k, v, o, do, lse, scale=scale, causal=causal)
    torch.cuda.synchronize()
    return (q, k, v, o, do, lse, scale, causal), ref


def _check(args, ref):
    q = args[0]
    outs = [torch.full_like(q, float("nan")) for _ in range(3)]
    st = _call_noalloc(*args[:6], *outs, args[6], args[7])
    assert st == 0, fa.strerror(st)
    torch.cuda.synchronize()
    # dQ goes through fp32 atomics in both calls: equal within the gradient tolerance
    g, r = gu.to_f64(outs[0]), gu.to_f64(ref[0])
    assert np.all(np.isfinite(g)) and gu.rel_fro(g, r) <= gu.GRAD_REL_FRO, "dQ"
    # dK and dV are summed in a fixed order on chip: identical bytes, so any
    # stale scratch content (row statistics of an earlier call) would show
    for name, got, want in zip(("dK", "dV"), outs[1:], ref[1:]):
        assert torch.equal(got.view(torch.int16), want.view(torch.int16)), name


def test_noalloc_matches_fa_bwd_on_two_calls_larger_then_smaller():
    """A shape that fills most of the scratch, then smaller ones (one causal,
    one with a ragged last tile) right after it, each twice: every call must
    equal fa_bwd with a caller workspace on the same inputs."""
    big = _case((2, 8, 7600, 128), False, 901)      # 60.3 MiB of the 64 MiB scratch
    small = [_case((2, 4, 1000, 64), False, 902), _case((1, 3, 777, 128), True, 903)]
    for _ in range(2):
        _check(*big)
        for c in small:
            _check(*c)
    assert fa.fa_device_status() == (0, 0)


def test_noalloc_checks_arguments_before_the_size_limit():
    B, H, N, d = 1, 32, 4096, 128
    assert fa.fa_bwd_workspace_size(B, H, N, d) > fa.lib.fa_bwd_noalloc_max_bytes()
    x = torch.empty((B, H, N, d), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, H, N), dtype=torch.float32, device="cuda")
    outs = [torch.empty_like(x) for _ in range(3)]
    for scale, causal in ((float("nan"), False), (-1.0, False), (0.125, 2)):
        st = _call_noalloc(x, x, x, x, x, lse, *outs, scale, causal)
        assert st == fa.STATUS_CODES["FA_ERR_INVALID_ARG"], (scale, causal, st)


def test_noalloc_rejects_shapes_beyond_its_scratch():
    B, H, N, d = 1, 32, 4096, 128          # needs 64 MiB of dQ accumulator plus row statistics
    limit = fa.lib.fa_bwd_noalloc_max_bytes()
    assert fa.fa_bwd_workspace_size(B, H, N, d) > limit
    x = torch.empty((B, H, N, d), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, H, N), dtype=torch.float32, device="cuda")
    outs = [torch.empty_like(x) for _ in range(3)]
    st = _call_noalloc(x, x, x, x, x, lse, *outs, 1.0 / math.sqrt(d), False)
    assert st == fa.STATUS_CODES["FA_ERR_SCRATCH_LIMIT"]
    assert "fixed array" in fa.strerror(st)
