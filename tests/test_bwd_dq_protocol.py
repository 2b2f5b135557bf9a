"""CPU model of the synchronisation protocol of the deterministic dQ kernel.

``bwd_dq_kernel<D, CAUSAL>`` (csrc/fa_bwd_dq.cu) keeps one query tile per
CTA and walks the key tiles: S = Q K_j^T and dP = dO V_j^T into TMEM, the
elementwise warpgroups turn them into dS (bf16, in TMEM), and dQ += dS K_j
accumulates in TMEM.  The model runs the producer (Q and dO once, K/V through
the ring), the MMA warp, the elementwise warps (one role), the TMA engine and
the in-order tensor pipe as coroutines under random interleavings with random
role speeds.  It checks for deadlock, exact parity phases, and that no TMEM
region or ring stage is rewritten while a read of it is pending: S_(j+1) and
dP_(j+1) only after the elementwise warps hold S_j and dP_j, dS_j only after
dQ += dS_(j-1) K_(j-1) executed, the dQ readout only after the last product,
a K/V stage only after every product that reads it.  A planted mistake must
be caught.
"""
import random

import pytest


import kernel_constants as kc

K = kc.barrier_counts("fa_bwd_dq.cu")
WARPS_PER_GROUP = 4      # a model agent for an elementwise group stands for its 4 warps


class Bar:
    def __init__(self, name, count):
        self.name, self.count, self.arrivals, self.completed = name, count, 0, 0

    def arrive(self):
        self.arrivals += 1
        assert self.arrivals <= self.count
        if self.arrivals == self.count:
            self.arrivals = 0
            self.completed += 1

    def passes(self, k):
        return (self.completed & 1) != (k & 1)


class Violation(Exception):
    pass


class Model:
    def __init__(self, T, nst, rng, plant=None):
        self.T, self.nst, self.rng, self.plant = T, nst, rng, plant
        B = Bar
        g = lambda n: kc.per_agent(K[n], 2 * WARPS_PER_GROUP, n)  # noqa: E731  (one agent: both groups)
        self.qdo_full = B("qdo_full", K["qdo_full"])
        self.k_full = [B(f"k_full{s}", K["k_full"]) for s in range(nst)]
        self.v_full = [B(f"v_full{s}", K["v_full"]) for s in range(nst)]
        self.kv_empty = [B(f"kv_empty{s}", K["kv_empty"]) for s in range(nst)]
        self.s_full, self.dp_full = B("s_full", K["s_full"]), B("dp_full", K["dp_full"])
        self.s_free, self.dp_free = B("s_free", g("s_free")), B("dp_free", g("dp_free"))
        self.ds_full, self.ds_free = B("ds_full", g("ds_full")), B("ds_free", K["ds_free"])
        self.final_ = B("final", K["final_"])
        self.speeds = {}
        self.pipe, self.tma = [], []
        self.exec = {"S": 0, "dP": 0, "dQ": 0}
        self.s_read = self.dp_read = self.ds_written = 0
        self.kv_reads = {}

    def wait(self, bar, k):
        return ("wait", bar, k)

    def speed(self, actor):
        if actor not in self.speeds:
            self.speeds[actor] = 10.0 ** self.rng.uniform(-3.0, 0.0)
        return self.speeds[actor]

    def producer(self):
        self.tma.append(self.qdo_full)
        for j in range(self.T):
            s = j % self.nst
            if j >= self.nst:
                yield self.wait(self.kv_empty[s], j // self.nst - 1)
                if self.kv_reads.get(j - self.nst, 0) != 3:
                    raise Violation(f"K/V stage {s} refilled while tile {j - self.nst} is still read")
            self.tma.append(self.k_full[s])
            self.tma.append(self.v_full[s])

    def mma(self):
        T, nst = self.T, self.nst
        yield self.wait(self.qdo_full, 0)
        yield self.wait(self.k_full[0], 0)
        yield self.wait(self.v_full[0], 0)
        self.pipe += [("S", 0), ("commit", self.s_full), ("dP", 0), ("commit", self.dp_full)]
        for j in range(T):
            s = j % nst
            if j + 1 < T:
                if self.plant != "no_s_free":
                    yield self.wait(self.s_free, j)
                yield self.wait(self.k_full[(j + 1) % nst], (j + 1) // nst)
                self.pipe += [("S", j + 1), ("commit", self.s_full)]
            yield self.wait(self.ds_full, j)
            self.pipe += [("dQ", j), ("commit", self.ds_free)]
            if j + 1 < T:
                yield self.wait(self.dp_free, j)
                yield self.wait(self.v_full[(j + 1) % nst], (j + 1) // nst)
                self.pipe += [("dP", j + 1), ("commit", self.dp_full)]
            self.pipe.append(("commit", self.kv_empty[s]))
        self.pipe.append(("commit", self.final_))
        yield self.wait(self.final_, 0)

    def elementwise(self):
        for j in range(self.T):
            yield self.wait(self.s_full, j)
            if self.exec["S"] < j + 1:
                raise Violation(f"S_{j} read before it was computed")
            self.s_read += 1
            self.s_free.arrive()
            yield self.wait(self.dp_full, j)
            self.dp_read += 1
            self.dp_free.arrive()
            if j > 0:
                yield self.wait(self.ds_free, j - 1)
            if self.exec["dQ"] < j:
                raise Violation(f"dS_{j} written before dQ += dS_{j - 1} K read the previous one")
            self.ds_written += 1
            self.ds_full.arrive()
        yield self.wait(self.final_, 0)
        if self.exec["dQ"] != self.T:
            raise Violation("dQ read out before its last product")

    def exec_pipe(self):
        entry = self.pipe.pop(0)
        if entry[0] == "commit":
            entry[1].arrive()
            return
        op, j = entry
        if op == "S" and j > 0 and self.s_read < j:
            raise Violation(f"S_{j} overwrote S_{j - 1} before it was read")
        if op == "dP" and j > 0 and self.dp_read < j:
            raise Violation(f"dP_{j} overwrote dP_{j - 1} before it was read")
        if op == "dQ" and self.ds_written < j + 1:
            raise Violation(f"dQ += dS_{j} K read dS before it was written")
        self.exec[op] += 1
        self.kv_reads[j] = self.kv_reads.get(j, 0) + 1

    def run(self, max_steps=100000):
        roles = {"producer": self.producer(), "mma": self.mma(), "ew": self.elementwise()}
        pending = {}
        for nm, gen in list(roles.items()):
            pending[nm] = next(gen, None)
            if pending[nm] is None:
                del roles[nm]
        for _ in range(max_steps):
            rdy = [nm for nm in roles if pending[nm][1].passes(pending[nm][2])]
            choices = rdy + (["tma"] if self.tma else []) + (["pipe"] if self.pipe else [])
            if not choices:
                if not roles:
                    return
                raise Violation(f"deadlock: { {nm: (pending[nm][1].name, pending[nm][2]) for nm in roles} }")
            c = self.rng.choices(choices, weights=[self.speed(x) for x in choices])[0]
            if c == "tma":
                self.tma.pop(self.rng.randrange(len(self.tma))).arrive()
            elif c == "pipe":
                self.exec_pipe()
            else:
                _, bar, k = pending[c]
                if bar.completed != k + 1:
                    raise Violation(f"{c}: wait on {bar.name} for completion {k} passed at {bar.completed}")
                nxt = next(roles[c], None)
                if nxt is None:
                    del roles[c]
                else:
                    pending[c] = nxt
        raise Violation("step limit")


@pytest.mark.parametrize("nst", [kc.ring_depth("fa_bwd_dq.cu", "kNST", 128),
                                 kc.ring_depth("fa_bwd_dq.cu", "kNST", 64)])   # ring depth at d = 128, 64
@pytest.mark.parametrize("T", [1, 2, 3, 5, 16])
def test_protocol_holds_under_random_interleavings(T, nst):
    for seed in range(60):
        Model(T, nst, random.Random(seed)).run()


def test_protocol_model_catches_a_planted_missing_wait():
    # Without the s_free wait, S_(j+1) can overwrite S_j before it was read.
    caught = 0
    for seed in range(200):
        try:
            Model(4, 2, random.Random(seed), plant="no_s_free").run()
        except Violation:
            caught += 1
    assert caught > 0


def test_model_counts_are_the_kernels():
    """One arrive per warp of both elementwise groups on s_free, dp_free and
    ds_full (the model's single elementwise agent), one per commit elsewhere."""
    assert K["s_free"] == K["dp_free"] == K["ds_full"] == 2 * WARPS_PER_GROUP
    assert all(K[n] == 1 for n in ("qdo_full", "k_full", "v_full", "kv_empty", "s_full", "dp_full", "ds_free",
                                   "final_"))
