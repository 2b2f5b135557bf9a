"""The C ABI without a GPU: every symbol declared in include/fa.h is exported
by libfa.so, and argument errors come back as status codes before anything
touches a device (so these calls are safe on any host)."""
import ctypes
import os
import re

import pytest

import exact_io_aware_55_b200 as fa

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "fa.h")
F = ctypes.c_float
C = fa.STATUS_CODES


def declared_functions():
    text = open(HEADER).read()
    return re.findall(r"^FA_API\s+[\w\s\*]+?\b(fa_\w+)\s*\(", text, flags=re.M)


def test_every_declared_symbol_is_exported():
    names = declared_functions()
    # the boundary's method calls, named as the hot-path scope lists them
    assert {"fa_fwd", "fa_bwd", "fa_fwd_fp8", "fa_bwd_workspace_size", "fa_strerror",
            "fa_get_device_status"} <= set(names)
    lib = ctypes.CDLL(fa.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n


def test_status_texts():
    assert fa.strerror(0) == "ok"
    for code in range(1, 9):
        assert len(fa.strerror(code)) > 5
    assert "unknown" in fa.strerror(99)
    assert fa.lib.fa_version() >= 100


def test_workspace_size_formula():
    # rows padded to 128: (-D, -LSE2) fp32, each rounded up to 256 B, then the fp32 dQ accumulator
    def expect(B, H, N, d):
        rows = B * H * ((N + 127) // 128 * 128)
        stat = (rows * 4 + 255) // 256 * 256
        return 2 * stat + B * H * N * d * 4
    for shape in [(1, 1, 128, 64), (2, 3, 1000, 128), (4, 16, 2048, 64), (1, 1, 1, 64)]:
        assert fa.fa_bwd_workspace_size(*shape) == expect(*shape)
    assert fa.fa_bwd_workspace_size(1, 1, 0, 64) == 0
    with pytest.raises(fa.FAError):
        fa.fa_bwd_workspace_size(1, 1, 16, 96)
    assert fa.lib.fa_bwd_workspace_size(-1, 1, 16, 64) == ctypes.c_size_t(-1).value


def fwd(q, o, lse, B=1, H=1, N=128, d=64, scale=0.125, causal=0):
    return fa.lib.fa_fwd(q, q, q, o, lse, B, H, N, d, F(scale), causal, None)


def test_forward_argument_errors_launch_nothing():
    assert fwd(None, None, None) == C["FA_ERR_INVALID_ARG"]
    assert fwd(4096, 4096, 4096, d=96) == C["FA_ERR_UNSUPPORTED"]
    assert fwd(4096, 4096, 4096, scale=-0.125) == C["FA_ERR_INVALID_ARG"]
    assert fwd(4096, 4096, 4096, scale=float("inf")) == C["FA_ERR_INVALID_ARG"]
    assert fwd(4096, 4096, 4096, scale=float("nan")) == C["FA_ERR_INVALID_ARG"]
    assert fwd(4096, 4096, 4096, causal=2) == C["FA_ERR_INVALID_ARG"]
    assert fwd(4096, 4096, 4096, N=-5) == C["FA_ERR_INVALID_ARG"]
    assert fwd(4104, 4096, 4096) == C["FA_ERR_ALIGNMENT"]          # 8-byte aligned only
    assert fwd(4096, 4096, 4098) == C["FA_ERR_ALIGNMENT"]          # lse needs 4 bytes
    assert fwd(None, None, None, N=0) == C["FA_OK"]                # empty: nothing to do
    assert fwd(None, None, None, B=0) == C["FA_OK"]
    assert fa.lib.fa_fwd_fp8(4096, 4096, 4096, F(1), F(1), F(1), 4096, 4096, 1, 1, 16, 64, F(0.1), 0,
                             None) == C["FA_ERR_UNSUPPORTED"]         # e4m3 path needs d = 128
    assert fa.lib.fa_fwd_fp8(4096, 4096, 4096, F(0), F(1), F(1), 4096, 4096, 1, 1, 16, 128, F(0.1), 0,
                             None) == C["FA_ERR_INVALID_ARG"]


def test_backward_argument_errors_launch_nothing():
    p = 4096
    args = [p] * 6 + [p] * 3
    assert fa.lib.fa_bwd(*args, 1, 1, 64, 64, F(0.125), 0, None, 0, None) == C["FA_ERR_WORKSPACE"]
    assert fa.lib.fa_bwd(*args, 1, 1, 64, 64, F(0.125), 0, p, 16, None) == C["FA_ERR_WORKSPACE"]
    need = fa.fa_bwd_workspace_size(1, 1, 64, 64)
    assert fa.lib.fa_bwd(*([p] * 5 + [p + 2] + [p] * 3), 1, 1, 64, 64, F(0.125), 0, p, need,
                         None) == C["FA_ERR_ALIGNMENT"]
    assert fa.lib.fa_bwd(*([None] + [p] * 8), 1, 1, 64, 64, F(0.125), 0, p, need, None) == C["FA_ERR_INVALID_ARG"]
    assert fa.lib.fa_bwd(*args, 1, 1, 0, 64, F(0.125), 0, None, 0, None) == C["FA_OK"]


def test_noalloc_limit_is_checked_first():
    limit = fa.lib.fa_bwd_noalloc_max_bytes()
    assert limit == 64 << 20
    assert fa.fa_bwd_workspace_size(1, 32, 4096, 128) > limit
    st = fa.lib.fa_bwd_noalloc(*([4096] * 9), 1, 32, 4096, 128, F(0.1), 0, None)
    assert st == C["FA_ERR_SCRATCH_LIMIT"]
    assert fa.lib.fa_bwd_noalloc(*([4096] * 9), 1, 1, 16, 96, F(0.1), 0, None) == C["FA_ERR_UNSUPPORTED"]


def decode_plan(B, H, Nq, Nk, d):
    """Items per head and workspace bytes of the decode path: a head's cache is
    cut into items of whole key tiles (128 keys at d=128, 256 at d=64); with
    one persistent CTA per SM (148 SMs) the time is about ceil(items / 148) x
    (tiles per item + 1/2 + Nq/64), and the balanced tiles-per-item value with
    the smallest such cost wins."""
    BH, T = B * H, -(-Nk // (256 if d == 64 else 128))
    best, plan = None, (1, max(T, 1))
    for tps in range(1, T + 1):
        ns = -(-T // tps)
        if -(-T // ns) != tps or BH * ns > 1 << 30:
            continue
        cost = -(-(BH * ns) // 148) * (tps + 0.5 + Nq / 64)
        if best is None or cost < best - 1e-9:
            best, plan = cost, (ns, tps)
    ns = plan[0]
    parts = BH * ns * Nq
    total = (parts * d * 4 + 255) // 256 * 256 + (parts * 4 + 255) // 256 * 256 if ns > 1 else 0
    return ns, total


def test_decode_workspace_size_formula():
    for shape in [(1, 1, 1, 64, 64), (1, 1, 1, 4096, 128), (8, 32, 1, 16384, 128), (2, 3, 16, 1000, 64),
                  (1, 1, 5, 70000, 128), (64, 32, 1, 4096, 128)]:
        assert fa.fa_fwd_decode_workspace_size(*shape) == decode_plan(*shape)[1]
    assert decode_plan(1, 1, 1, 64, 64) == (1, 0)                # one tile: one item, no workspace
    assert decode_plan(1, 1, 1, 4096 * 37, 128)[0] == 148        # one head: an item per SM
    assert decode_plan(8, 32, 1, 16384, 128)[0] == 4             # 1024 items of 32 tiles
    assert decode_plan(64, 32, 1, 4096, 128)[0] == 1             # enough heads: no split
    assert fa.fa_fwd_decode_workspace_size(1, 1, 0, 64, 64) == 0
    with pytest.raises(fa.FAError):
        fa.fa_fwd_decode_workspace_size(1, 1, 17, 64, 64)
    with pytest.raises(fa.FAError):
        fa.fa_fwd_decode_workspace_size(1, 1, 1, 64, 96)


def test_decode_argument_errors_launch_nothing():
    p = 4096

    def dec(Nq=1, Nk=64, d=64, causal=0, ws=None, wbytes=0, q=p, o=p, lse=p, scale=0.125):
        return fa.lib.fa_fwd_decode(q, p, p, o, lse, 1, 1, Nq, Nk, d, F(scale), causal, ws, wbytes, None)

    assert dec(Nq=17) == C["FA_ERR_UNSUPPORTED"]
    assert dec(d=96) == C["FA_ERR_UNSUPPORTED"]
    assert dec(Nk=0) == C["FA_ERR_INVALID_ARG"]                     # queries with nothing to attend to
    assert dec(Nq=8, Nk=4, causal=1) == C["FA_ERR_INVALID_ARG"]     # causal needs Nk >= Nq
    assert dec(scale=-1.0) == C["FA_ERR_INVALID_ARG"]
    assert dec(q=None) == C["FA_ERR_INVALID_ARG"]
    assert dec(q=p + 8) == C["FA_ERR_ALIGNMENT"]
    assert dec(Nk=4096) == C["FA_ERR_WORKSPACE"]                    # 16 splits need a workspace
    need = fa.fa_fwd_decode_workspace_size(1, 1, 1, 4096, 64)
    assert dec(Nk=4096, ws=p, wbytes=need - 1) == C["FA_ERR_WORKSPACE"]
    assert dec(Nk=4096, ws=p + 4, wbytes=need) == C["FA_ERR_ALIGNMENT"]
    assert dec(Nq=0, q=None, o=None, lse=None) == C["FA_OK"]        # empty: nothing to do


def test_standard_workspace_and_errors():
    # S fp32 then P bf16, both [B,H,N,Np] with Np = N rounded up to 128; S rounded up to 256 bytes
    def expect(B, H, N, d):
        cells = B * H * N * (-(-N // 128) * 128)
        return (cells * 4 + 255) // 256 * 256 + cells * 2
    for shape in [(1, 1, 1, 64), (2, 3, 300, 128), (4, 16, 2048, 64)]:
        assert fa.fa_fwd_standard_workspace_size(*shape) == expect(*shape)
    assert fa.fa_fwd_standard_workspace_size(1, 1, 0, 64) == 0
    p = 4096
    need = fa.fa_fwd_standard_workspace_size(1, 1, 64, 64)

    def std(ws=p, wbytes=need, d=64, q=p):
        return fa.lib.fa_fwd_standard(q, p, p, p, p, 1, 1, 64, d, F(0.125), 0, ws, wbytes, None)

    assert std(ws=None, wbytes=0) == C["FA_ERR_WORKSPACE"]
    assert std(wbytes=need - 1) == C["FA_ERR_WORKSPACE"]
    assert std(ws=p + 16) == C["FA_ERR_ALIGNMENT"]            # workspace must be 256-byte aligned
    assert std(q=p + 8) == C["FA_ERR_ALIGNMENT"]
    assert std(d=96) == C["FA_ERR_UNSUPPORTED"]
    assert std(q=None) == C["FA_ERR_INVALID_ARG"]


def test_scale_zero_passes_the_argument_checks():
    # scale = 0 is a valid (uniform-weight) softmax: the call gets past every
    # host check and stops only at the device query on a host without a GPU
    st = fwd(4096, 4096, 4096, scale=0.0)
    assert st in (C["FA_ERR_ARCH"], C["FA_OK"], C["FA_ERR_LAUNCH"])
    assert st != C["FA_ERR_INVALID_ARG"]


def test_forward_plan_on_the_mixed_grid():
    """B4 H16 N2048 d128 non-causal: 512 Q-tile pairs on 148 SMs leave a last
    round of 68, which is split into 136 single-tile items dispatched last."""
    if fa.lib.fa_get_device_status(None) != C["FA_ERR_ARCH"]:
        pytest.skip("a GPU is visible; the GPU test checks the plan with its SM count")
    assert fa.fa_fwd_plan(4, 16, 2048, 128, False) == (580, 580, 444)
    assert fa.fa_fwd_plan(4, 16, 2048, 64, False) == (148, 580, 444)     # persistent CTAs
    assert fa.fa_fwd_plan(4, 16, 2048, 128, True) == (512, 512, 512)     # causal: pairs only
    assert fa.fa_fwd_plan(1, 32, 8192, 128, False) == (1024, 1024, 1024)  # 1024 = 148 * 6 + 136: no split
    assert fa.fa_fwd_plan(1, 1, 0, 128, False) == (0, 0, 0)
    with pytest.raises(fa.FAError):
        fa.fa_fwd_plan(1, 1, 16, 96, False)


def test_bwd_events_needs_four_events():
    p = 4096
    args = [p] * 9
    need = fa.fa_bwd_workspace_size(1, 1, 64, 64)
    assert fa.lib.fa_bwd_events(*args, 1, 1, 64, 64, F(0.125), 0, p, need, None, None) == C["FA_ERR_INVALID_ARG"]
    ev = (ctypes.c_void_p * 4)(p, p, None, p)
    assert fa.lib.fa_bwd_events(*args, 1, 1, 64, 64, F(0.125), 0, p, need, ev, None) == C["FA_ERR_INVALID_ARG"]


def test_get_device_status_without_a_gpu():
    if fa.lib.fa_get_device_status(None) == C["FA_OK"]:
        pytest.skip("a GPU is visible")
    assert fa.lib.fa_get_device_status(None) == C["FA_ERR_ARCH"]


def test_fp8_backward_argument_errors_launch_nothing():
    p = 4096
    need = fa.fa_bwd_fp8_workspace_size(1, 1, 64, 128)
    assert need > fa.fa_bwd_workspace_size(1, 1, 64, 128)
    # bf16 workspace + three widened [BH, N, d] bf16 tensors
    base = (fa.fa_bwd_workspace_size(1, 1, 64, 128) + 255) // 256 * 256
    assert need == base + 2 * ((64 * 128 * 2 + 255) // 256 * 256) + 64 * 128 * 2
    assert fa.lib.fa_bwd_fp8_workspace_size(1, 1, 64, 64) == ctypes.c_size_t(-1).value

    def call(d=128, qd=1.0, ws=need, N=64):
        return fa.lib.fa_bwd_fp8(p, p, p, F(qd), F(1.0), F(1.0), p, p, p, p, p, p, 1, 1, N, d, F(0.125), 0,
                                 p, ws, None)
    assert call(d=64) == C["FA_ERR_UNSUPPORTED"]
    assert call(qd=0.0) == C["FA_ERR_INVALID_ARG"]
    assert call(qd=float("nan")) == C["FA_ERR_INVALID_ARG"]
    assert call(ws=need - 1) == C["FA_ERR_WORKSPACE"]
    assert call(N=0) == C["FA_OK"]
