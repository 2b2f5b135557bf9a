"""The N > 1 path on CPU: two gloo ranks split the heads with head_range, each
computes its heads (here with the fp64 oracle; on GPUs each rank calls the
library on its slice), and the gathered result equals the single-process one.
Also checks the max-over-ranks timing reduction used by bench.py."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from exact_io_aware_55_b200.dist import head_range, max_over_ranks


def test_head_range_partitions():
    for n in (0, 1, 5, 64, 65):
        for w in (1, 2, 3, 8):
            spans = [head_range(n, w, r) for r in range(w)]
            assert spans[0][0] == 0 and spans[-1][1] == n
            assert all(a[1] == b[0] for a, b in zip(spans, spans[1:]))
            sizes = [e - s for s, e in spans]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        head_range(4, 2, 2)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import oracle
    import synth
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        B, H, N, d = 1, 5, 40, 8
        inp = synth.attention_inputs(B, H, N, d, seed=77, with_grad=False)
        q, k, v = (inp[n].reshape(B * H, N, d) for n in ("q", "k", "v"))
        s, e = head_range(B * H, world, rank)
        o_part = np.zeros((B * H, N, d))
        for h in range(s, e):
            o_part[h], _ = oracle.head_forward(q[h], k[h], v[h], 0.3, True)
        t = torch.from_numpy(o_part)
        dist.all_reduce(t)                 # disjoint slices: the sum assembles the whole
        full = np.stack([oracle.head_forward(q[h], k[h], v[h], 0.3, True)[0] for h in range(B * H)])
        ok_parity = bool(np.allclose(t.numpy(), full, atol=0, rtol=0))
        times = max_over_ranks(dist, [1.0 + rank, 5.0 - rank])
        out.put((rank, ok_parity, times))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_shard_heads_and_take_max_time():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ok_parity, times in res:
        assert ok_parity
        assert times == [2.0, 5.0]


def test_max_over_ranks_without_group():
    assert max_over_ranks(None, [1, 2]) == [1.0, 2.0]


def _bench_shard_worker(rank, world, port, out):
    """One rank of the bench's sharding: its slice of the flattened heads, cut
    from the full seeded problem with bench.head_slice, run as a [1, nh, N, d]
    problem (here by the oracle; on GPUs by the library)."""
    import bench
    import oracle
    import synth
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        B, H, N, d = 2, 3, 24, 8
        inp = synth.attention_inputs(B, H, N, d, seed=78, with_grad=False, want_f64=False)
        h0, h1 = bench.rank_heads(B, H, world, rank)
        parts = {n: bench.head_slice(inp[n + "_bits"], B, H, h0, h1) for n in ("q", "k", "v")}
        full = np.zeros((B * H, N, d))
        for j in range(h1 - h0):
            qh, kh, vh = (synth.bf16_bits_to_f64(parts[n][0, j]) for n in ("q", "k", "v"))
            full[h0 + j], _ = oracle.head_forward(qh, kh, vh, 0.35, True)
        t = torch.from_numpy(full)
        dist.all_reduce(t)
        ref = oracle.attention_forward(synth.bf16_bits_to_f64(inp["q_bits"]), synth.bf16_bits_to_f64(inp["k_bits"]),
                                       synth.bf16_bits_to_f64(inp["v_bits"]), 0.35, True)[0].reshape(B * H, N, d)
        out.put((rank, (h0, h1), bool(np.array_equal(t.numpy(), ref))))
    finally:
        dist.destroy_process_group()


def test_bench_shards_one_problem_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_bench_shard_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[1] for r in res] == [(0, 3), (3, 6)]       # 6 heads split 3 + 3, across the batch boundary
    assert all(r[2] for r in res)


def test_bench_gpus_flag_launches_that_many_ranks():
    """`bench.py --gpus 2` outside torchrun re-launches itself under
    torch.distributed.run with two ranks; the reference arm needs no GPU, so
    the launcher path runs here: rank 0 prints one line with n_gpus = 2."""
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = {k: v for k, v in os.environ.items() if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK")}
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--gpus", "2", "--impl", "reference",
                        "--shape", "1,2,256,64", "--causal", "--steps", "1", "--warmup", "3",
                        "--ref-step-budget", "0"], capture_output=True, text=True, timeout=300, env=env, cwd=root)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [json.loads(x) for x in r.stdout.splitlines() if x.startswith("{")]
    assert len(lines) == 1, r.stdout
    assert lines[0]["n_gpus"] == 2 and lines[0]["impl"] == "reference"
