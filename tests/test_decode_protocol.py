"""CPU model of the synchronisation protocol of the split-KV decode kernel.

The model runs the roles of ``decode_kernel`` (csrc/fa_decode.cu) as
coroutines: the TMA producer (Q once per work item, K/V tiles through a
3-stage ring), the MMA warp (S^T of each tile into one of two S buffers, and
O^T += V^T P^T one tile behind into one of two O buffers), the softmax warps
(one role: their max exchange is internal to the role), the epilogue warps,
the TMA engine (loads complete asynchronously) and the in-order tensor pipe.
A random scheduler with per-run random speeds interleaves them.  Every wait
names the completion it intends (the kernel's parity expression), and the
model checks for deadlock, exact phases, and that no buffer is rewritten while
a read of it is pending: S buffers, the two shared-memory P^T buffers, the two
O^T buffers in TMEM (first product of an item, rescales), the per-item
statistics the epilogue reads, the K/V stages and the Q buffers.
A planted mistake must be caught, so the checks are not vacuous.
"""
import random

import pytest

import kernel_constants as kc

NS = kc.ring_depth("fa_decode.cu", "kNS")   # K/V ring depth of the decode kernel
K = kc.barrier_counts("fa_decode.cu")
WARPS_PER_ROLE = 4      # a model agent for the softmax or epilogue role stands for its 4 warps


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
    def __init__(self, nts, rescale, rng, plant=None):
        self.nts, self.rescale, self.rng, self.plant = nts, rescale, rng, plant
        B = Bar
        g = lambda n: kc.per_agent(K[n], WARPS_PER_ROLE, n)  # noqa: E731
        two = lambda n, c: [B(f"{n}{i}", c) for i in range(2)]  # noqa: E731
        self.q_full, self.q_empty = two("q_full", K["q_full"]), two("q_empty", K["q_empty"])
        self.kv_full = [B(f"kv_full{s}", K["kv_full"]) for s in range(NS)]
        self.kv_empty = [B(f"kv_empty{s}", K["kv_empty"]) for s in range(NS)]
        self.s_full, self.s_free = two("s_full", K["s_full"]), two("s_free", g("s_free"))
        self.p_full, self.pv_done = two("p_full", g("p_full")), two("pv_done", K["pv_done"])
        self.o_full, self.o_free = two("o_full", K["o_full"]), two("o_free", g("o_free"))
        self.stats_full = two("stats_full", g("stats_full"))
        self.speeds = {}
        self.pipe, self.tma = [], []
        self.s_exec = 0            # S^T products executed (ring index order)
        self.pv_exec = 0           # PV products executed
        self.s_read = 0            # S tiles read by the softmax
        self.epi_done = 0          # items read out by the epilogue
        self.item_last_g = []      # ring index of each item's last tile
        g = 0
        for nt in nts:
            g += nt
            self.item_last_g.append(g - 1)

    def wait(self, bar, k):
        return ("wait", bar, k)

    def speed(self, actor):
        if actor not in self.speeds:
            self.speeds[actor] = 10.0 ** self.rng.uniform(-3.0, 0.0)
        return self.speeds[actor]

    # ------------------------------------------------------------------ roles
    def producer(self):
        g = 0
        for it, nt in enumerate(self.nts):
            qb = it & 1
            if it >= 2:
                yield self.wait(self.q_empty[qb], (it >> 1) - 1)
                if self.s_exec < self.item_last_g[it - 2] + 1:
                    raise Violation(f"Q buffer {qb} refilled while item {it - 2}'s S^T is pending")
            self.tma.append(self.q_full[qb])
            for _ in range(nt):
                s = g % NS
                if g >= NS:
                    yield self.wait(self.kv_empty[s], g // NS - 1)
                    if self.s_exec < g - NS + 1 or self.pv_exec < g - NS + 1:
                        raise Violation(f"K/V stage {s} refilled while tile {g - NS} is still read")
                self.tma.append(self.kv_full[s])
                g += 1

    def mma(self):
        g = 0
        for it, nt in enumerate(self.nts):
            qb = ob = it & 1

            def issue_pv(gg, first):
                pb = gg & 1
                if first and it >= 2 and self.plant != "no_o_free":
                    yield self.wait(self.o_free[ob], (it >> 1) - 1)
                yield self.wait(self.p_full[pb], gg >> 1)
                self.pipe.append(("PV", gg, it if first else None))
                self.pipe.append(("commit", self.pv_done[pb]))
                self.pipe.append(("commit", self.kv_empty[gg % NS]))

            yield self.wait(self.q_full[qb], it >> 1)
            for j in range(nt):
                s, sb = g % NS, g & 1
                yield self.wait(self.kv_full[s], g // NS)
                if g >= 2:
                    yield self.wait(self.s_free[sb], (g >> 1) - 1)
                self.pipe.append(("S", g, None))
                self.pipe.append(("commit", self.s_full[sb]))
                if j == nt - 1:
                    self.pipe.append(("commit", self.q_empty[qb]))
                if j > 0:
                    yield from issue_pv(g - 1, j == 1)
                g += 1
            yield from issue_pv(g - 1, nt == 1)
            self.pipe.append(("commit", self.o_full[ob]))

    def softmax(self):
        g = 0
        for it, nt in enumerate(self.nts):
            ob = it & 1
            for j in range(nt):
                sb = g & 1
                yield self.wait(self.s_full[sb], g >> 1)
                self.s_read += 1
                self.s_free[sb].arrive()
                if j > 0 and self.rescale(it, j):
                    yield self.wait(self.pv_done[(g - 1) & 1], (g - 1) >> 1)
                    if self.pv_exec < g:
                        raise Violation(f"O^T {ob} rescaled before PV {g - 1} executed")
                pb = g & 1
                if g >= 2:
                    yield self.wait(self.pv_done[pb], (g - 2) >> 1)
                if self.pv_exec < g - 1:
                    raise Violation(f"P^T buffer {pb} rewritten before PV {g - 2} read it")
                self.p_full[pb].arrive()
                g += 1
            yield self.wait(self.pv_done[(g - 1) & 1], (g - 1) >> 1)
            if self.epi_done < it - 1:
                raise Violation(f"statistics {ob} rewritten before the epilogue of item {it - 2} read them")
            self.stats_full[ob].arrive()

    def epilogue(self):
        for it in range(len(self.nts)):
            ob = it & 1
            yield self.wait(self.o_full[ob], it >> 1)
            yield self.wait(self.stats_full[ob], it >> 1)
            if self.pv_exec < self.item_last_g[it] + 1:
                raise Violation(f"epilogue read O^T of item {it} before its last product")
            self.epi_done += 1
            self.o_free[ob].arrive()

    # -------------------------------------------------------------- execution
    def exec_pipe(self):
        entry = self.pipe.pop(0)
        if entry[0] == "commit":
            entry[1].arrive()
            return
        op, x, first_item = entry
        if op == "S":
            if x >= 2 and self.s_read < x - 1:
                raise Violation(f"S^T {x} overwrote S buffer {x & 1} before the softmax read it")
            if self.s_exec != x:
                raise Violation("S^T products out of order")
            self.s_exec += 1
        else:
            if first_item is not None and self.epi_done < first_item - 1:
                raise Violation(f"first PV of item {first_item} overwrote O^T before the epilogue read it")
            if self.pv_exec != x:
                raise Violation("PV products out of order")
            self.pv_exec += 1

    def run(self, max_steps=200000):
        roles = {"producer": self.producer(), "mma": self.mma(), "softmax": self.softmax(),
                 "epilogue": self.epilogue()}
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


CASES = [[1], [1, 1, 1, 1], [3], [2, 5, 1, 4, 2], [4, 4, 4, 3], [1, 6, 1, 6, 1]]


@pytest.mark.parametrize("nts", CASES)
@pytest.mark.parametrize("rescale_mode", ["never", "always", "random"])
def test_protocol_holds_under_random_interleavings(nts, rescale_mode):
    for seed in range(40):
        rng = random.Random(seed)
        pick = random.Random(seed + 1000)
        rescale = {"never": lambda it, j: False, "always": lambda it, j: True,
                   "random": lambda it, j: pick.random() < 0.3}[rescale_mode]
        Model(nts, rescale, rng).run()


def test_protocol_model_catches_a_planted_missing_wait():
    # Without the o_free wait, the first product of an item can overwrite the
    # O^T buffer before the epilogue has read the item two before it.
    caught = 0
    for seed in range(200):
        try:
            Model([1, 1, 1, 2, 1], lambda it, j: False, random.Random(seed), plant="no_o_free").run()
        except Violation:
            caught += 1
    assert caught > 0


def test_model_counts_are_the_kernels():
    """One arrive per warp of the softmax role (s_free, p_full, red) and of the
    epilogue role (o_free, stats_full), one per commit or TMA elsewhere."""
    assert K["s_free"] == K["p_full"] == K["red"] == K["o_free"] == K["stats_full"] == WARPS_PER_ROLE
    assert all(K[n] == 1 for n in ("q_full", "q_empty", "kv_full", "kv_empty", "s_full", "pv_done", "o_full"))
