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
