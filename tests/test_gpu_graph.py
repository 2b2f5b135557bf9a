"""The forward and the backward inside a CUDA graph.

fa_fwd, fa_bwd, fa_bwd_deterministic and fa_fwd_fp8 only launch kernels on
the caller's stream (the tensor maps are built on the host and passed by
value; nothing is allocated or synchronised), so a caller can capture a whole
step once and replay it.  This test captures forward + backward with
torch.cuda.CUDAGraph, replays it on new inputs copied into the captured
buffers, checks the replay against eager calls on the same inputs, and checks the
last replay against the fp64 oracle.
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


@pytest.mark.parametrize("d,causal", [(64, False), (128, True)])
def test_capture_and_replay_forward_backward(d, causal):
    B, H, N = 2, 3, 777
    scale = 1.0 / math.sqrt(d)
    bufs = {n: torch.empty((B, H, N, d), dtype=torch.bfloat16, device="cuda") for n in ("q", "k", "v", "do")}
    o = torch.empty_like(bufs["q"])
    lse = torch.empty((B, H, N), dtype=torch.float32, device="cuda")
    dq, dk, dv = (torch.empty_like(bufs["q"]) for _ in range(3))
    work = torch.empty(fa.fa_bwd_workspace_size(B, H, N, d), dtype=torch.uint8, device="cuda")

    def load(seed):
        inp = synth.attention_inputs(B, H, N, d, seed=seed)
        for n in bufs:
            bufs[n].copy_(gu.dev_bf16(inp[n + "_bits"]))
        return inp

    def step(stream):
        fa.fa_fwd(bufs["q"], bufs["k"], bufs["v"], o, lse, scale, causal, stream)
        fa.fa_bwd(bufs["q"], bufs["k"], bufs["v"], o, bufs["do"], lse, dq, dk, dv, scale, causal, work, stream)

    load(4000)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):                 # warm-up (configures the kernels) off the capture
        step(side)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step(torch.cuda.current_stream())
    for seed in (4001, 4002):
        inp = load(seed)
        graph.replay()
        torch.cuda.synchronize()
        got = [t.clone() for t in (o, lse, dq, dk, dv)]
        step(torch.cuda.current_stream())         # eager, same inputs
        torch.cuda.synchronize()
        want = (o, lse, dq, dk, dv)
        for name, g, w in zip(("O", "LSE", "dK", "dV"), (got[0], got[1], got[3], got[4]), (want[0], want[1], want[3], want[4])):
            assert torch.equal(g, w), name       # no atomics: identical bytes
        assert gu.rel_fro(gu.to_f64(got[2]), gu.to_f64(want[2])) <= 1e-3   # dQ: fp32 atomics reorder
    o_ref, lse_ref = oracle.attention_forward(inp["q"], inp["k"], inp["v"], scale, causal)
    gu.assert_o_lse(gu.to_f64(got[0]), gu.to_f64(got[1]), o_ref, lse_ref, "graph replay")
    ref = oracle.attention_backward(inp["q"], inp["k"], inp["v"], inp["do"], scale, causal)
    for name, g, r in zip(("dQ", "dK", "dV"), got[2:], ref):
        assert gu.rel_fro(gu.to_f64(g), r) <= gu.GRAD_REL_FRO, name
    assert fa.fa_device_status() == (0, 0)
