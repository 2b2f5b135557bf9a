"""CPU model of the synchronisation protocol of the persistent d = 64 forward.

The model runs the roles of ``fwd64_kernel`` (csrc/fa_fwd64.cu) as coroutines:
the TMA producer, one MMA-issuing warp per Q-tile slot, the two softmax
warpgroups, the TMA engine (loads complete asynchronously) and the in-order
tensor pipe (MMAs and ``tcgen05.commit`` arrivals execute in issue order).
A random scheduler with per-run random speeds interleaves them.  Each mbarrier
wait names the completion it intends (the kernel's parity expression); the
model applies the hardware rule (a parity wait passes once the barrier's phase
parity differs) and checks:

* no deadlock;
* every wait that passes sees exactly its intended completion (no parity
  aliasing: neither before it nor two phases after it);
* no buffer is overwritten while a read of its previous contents is pending:
  the producer refills a K/V stage or a Q buffer only after every MMA that
  reads the old contents has executed, a softmax warpgroup writes P_g only
  after the previous O_g += P_g V has executed, and the first O_g += P_g V of
  an item (which overwrites O_g) executes only after the previous item's
  epilogue has read O_g.

Items follow the kernel's numbering: non-causal Q-tile pairs, the split
single-tile items of an uneven last round, and causal pairs with T_0 < T_1.
A planted mistake (a slot with no work on a tile releasing the stage without
waiting for its load) must be caught, so the checks are not vacuous.
"""
import random

import pytest

import kernel_constants as kc

NST = kc.ring_depth("fa_fwd64.cu", "kD64NST")   # K/V ring depth of the d = 64 kernel
K = kc.barrier_counts("fa_fwd64.cu")
WARPS_PER_GROUP = 4      # a model agent for a softmax group stands for its 4 warps


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
        """Hardware rule for a wait on the phase with the parity of completion k."""
        return (self.completed & 1) != (k & 1)


class Violation(Exception):
    pass


class Model:
    def __init__(self, items, rng, planted_bug=False):
        self.items, self.rng, self.bug = items, rng, planted_bug
        B = Bar
        g = lambda n: kc.per_agent(K[n], WARPS_PER_GROUP, n)  # noqa: E731
        two = lambda n, c: [B(f"{n}{i}", c) for i in range(2)]  # noqa: E731
        self.q_full, self.q_empty = two("q_full", K["q_full"]), two("q_empty", K["q_empty"])  # both MMA warps
        self.k_full = [B(f"k_full{s}", K["k_full"]) for s in range(NST)]
        self.v_full = [B(f"v_full{s}", K["v_full"]) for s in range(NST)]
        self.kv_empty = [B(f"kv_empty{s}", K["kv_empty"]) for s in range(NST)]   # both MMA warps
        self.s_full, self.s_free = two("s_full", K["s_full"]), two("s_free", g("s_free"))
        self.p_full, self.pv_done = two("p_full", g("p_full")), two("pv_done", K["pv_done"])
        self.o_final = two("o_final", K["o_final"])
        self.speeds = {}
        self.pipe = []          # in-order tensor pipe: ("mma", info) | ("commit", bar)
        self.tma = []           # outstanding loads: bars to arrive on
        # buffer bookkeeping
        self.kv_reads_needed, self.kv_reads_done = {}, {}
        self.q_reads_needed, self.q_reads_done = {}, {}
        self.pv_exec = [0, 0]   # O_g += P_g V executed, per slot
        self.epi_done = [0, 0]  # epilogues finished, per slot

    # ------------------------------------------------------------------ roles
    def wait(self, bar, k):
        return ("wait", bar, k)

    def speed(self, actor):
        """Per-run random speed of each role and engine (log-uniform over three
        decades), so that some runs starve one of them for long stretches."""
        if actor not in self.speeds:
            self.speeds[actor] = 10.0 ** self.rng.uniform(-3.0, 0.0)
        return self.speeds[actor]

    def producer(self):
        kv_c = 0
        for n, (T0, T1) in enumerate(self.items):
            Tmax, qb = max(T0, T1), n & 1
            if n >= 2:
                yield self.wait(self.q_empty[qb], (n >> 1) - 1)
                key = (qb, n - 2)
                if self.q_reads_done.get(key, 0) != self.q_reads_needed.get(key, 0):
                    raise Violation(f"Q buffer {qb} refilled while item {n - 2} still reads it")
            self.q_reads_needed[(qb, n)] = T0 + T1
            self.tma.append(self.q_full[qb])
            for j in range(Tmax):
                s, u = kv_c % NST, kv_c // NST
                if kv_c >= NST:
                    yield self.wait(self.kv_empty[s], u - 1)
                    key = (s, u - 1)
                    if self.kv_reads_done.get(key, 0) != self.kv_reads_needed[key]:
                        raise Violation(f"K/V stage {s} refilled while use {u - 1} is still read")
                self.kv_reads_needed[(s, u)] = 2 * ((j < T0) + (j < T1))   # S reads K, PV reads V
                self.tma.append(self.k_full[s])
                self.tma.append(self.v_full[s])
                kv_c += 1

    def mma_warp(self, g):
        kv_c = n_s = n_p = 0
        m = 0                   # items of this slot so far
        n = 0
        for n, (T0, T1) in enumerate(self.items):
            Tg, Tmax, qb = (T0, T1)[g], max(T0, T1), n & 1
            yield self.wait(self.q_full[qb], n >> 1)
            if Tg > 0:
                yield self.wait(self.k_full[kv_c % NST], kv_c // NST)
                if n_s > 0:
                    yield self.wait(self.s_free[g], n_s - 1)
                self.pipe.append(("mma", ("S", g, (kv_c % NST, kv_c // NST), (qb, n), None)))
                self.pipe.append(("commit", self.s_full[g]))
                n_s += 1
            for j in range(Tmax):
                s, u = kv_c % NST, kv_c // NST
                if j < Tg:
                    if j + 1 < Tg:
                        c1 = kv_c + 1
                        yield self.wait(self.s_free[g], n_s - 1)
                        yield self.wait(self.k_full[c1 % NST], c1 // NST)
                        self.pipe.append(("mma", ("S", g, (c1 % NST, c1 // NST), (qb, n), None)))
                        self.pipe.append(("commit", self.s_full[g]))
                        n_s += 1
                    yield self.wait(self.v_full[s], u)
                    yield self.wait(self.p_full[g], n_p)
                    self.pipe.append(("mma", ("PV", g, (s, u), None, m if j == 0 else None)))
                    self.pipe.append(("commit", self.pv_done[g]))
                    n_p += 1
                    if j + 1 == Tg:
                        self.pipe.append(("commit", self.o_final[g]))
                    self.pipe.append(("commit", self.kv_empty[s]))
                else:
                    if not self.bug:
                        yield self.wait(self.v_full[s], u)
                    self.kv_empty[s].arrive()
                kv_c += 1
            if Tg > 0:
                self.pipe.append(("commit", self.q_empty[qb]))
                m += 1
            else:
                self.q_empty[qb].arrive()
        if self.items:
            yield self.wait(self.kv_empty[(kv_c - 1) % NST], (kv_c - 1) // NST)
            yield self.wait(self.q_empty[n & 1], n >> 1)

    def softmax(self, g):
        n_t = n_o = 0
        for (T0, T1) in self.items:
            Tg = (T0, T1)[g]
            if Tg == 0:
                continue
            for j in range(Tg):
                yield self.wait(self.s_full[g], n_t)
                self.s_free[g].arrive()               # S_g(j) is in registers
                if j > 0:
                    yield self.wait(self.pv_done[g], n_t - 1)
                if self.pv_exec[g] < n_t:
                    raise Violation(f"P_{g} written while O_{g} += P_{g} V of tile {n_t - 1} is pending")
                self.p_full[g].arrive()
                n_t += 1
            yield self.wait(self.o_final[g], n_o)
            if self.pv_exec[g] != n_t:
                raise Violation(f"epilogue {n_o} of slot {g} read O_{g} before its last product")
            self.epi_done[g] += 1                     # O_g read out
            n_o += 1

    # -------------------------------------------------------------- execution
    def exec_pipe(self):
        kind, x = self.pipe.pop(0)
        if kind == "commit":
            x.arrive()
            return
        op, g, kv, q, first_of_item = x
        self.kv_reads_done[kv] = self.kv_reads_done.get(kv, 0) + 1
        if op == "S":
            self.q_reads_done[q] = self.q_reads_done.get(q, 0) + 1
        else:
            if first_of_item is not None and self.epi_done[g] != first_of_item:
                raise Violation(f"O_{g} overwritten before the epilogue of item {first_of_item - 1}")
            self.pv_exec[g] += 1

    def run(self, max_steps=200000):
        roles = {"producer": self.producer(), "mma0": self.mma_warp(0), "mma1": self.mma_warp(1),
                 "sm0": self.softmax(0), "sm1": self.softmax(1)}
        pending = {}
        for name, gen in list(roles.items()):
            pending[name] = next(gen, None)
            if pending[name] is None:
                del roles[name]
        for _ in range(max_steps):
            ready = [nm for nm in roles if pending[nm][1].passes(pending[nm][2])]
            choices = ready + (["tma"] if self.tma else []) + (["pipe"] if self.pipe else [])
            if not choices:
                if not roles:
                    return
                waits = {nm: (pending[nm][1].name, pending[nm][2]) for nm in roles}
                raise Violation(f"deadlock: {waits}")
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


def kernel_items(BH, N, causal, sms, cta):
    """The (T_0, T_1) of the items CTA `cta` takes, as fwd_item / fwd_slot and
    the API's pair split compute them."""
    n_kv = (N + 127) // 128
    n_qt = n_kv
    n_pairs = (N + 255) // 256
    pairs = n_pairs * BH
    rem = pairs % sms
    pair_blocks = pairs if (causal or n_qt % 2 or rem == 0 or 2 * rem > sms) else pairs - rem
    n_items = pairs if causal else pair_blocks + 2 * (pairs - pair_blocks)
    grid = n_items if causal else min(n_items, sms)
    out = []
    if cta >= grid:
        return out
    for w in range(cta, n_items, grid):
        only = -1
        if causal:
            pair = n_pairs - 1 - (w % n_pairs)   # any pair order: only T matters here
        else:
            p = w
            if p >= pair_blocks:
                u = p - pair_blocks
                p, only = pair_blocks + (u >> 1), u & 1
            pair = p % n_pairs
        T = []
        for g in range(2):
            q0 = pair * 256 + (only if only >= 0 else g) * 128
            ok = q0 < N and (only < 0 or g == 0)
            T.append((min(n_kv, q0 // 128 + 1) if causal else n_kv) if ok else 0)
        out.append(tuple(T))
    return out


CASES = [
    # (BH, N, causal, SMs, CTA): several items per CTA, split single tiles, causal pairs
    (64, 2048, False, 148, 0),      # bench shape: 3 pairs then one single tile
    (64, 2048, False, 148, 140),    # a CTA without a single-tile item
    (80, 1000, False, 148, 10),     # ragged N, singles among pairs
    (3, 300, False, 2, 1),          # odd tile count: no split, a pair with one tile
    (1, 640, False, 1, 0),          # one CTA takes every item
    (4, 2048, True, 148, 5),        # causal: T_0 < T_1
    (1, 200, True, 148, 0),         # causal, a single pair with one tile each
]


@pytest.mark.parametrize("case", CASES)
def test_protocol_holds_under_random_interleavings(case):
    items = kernel_items(*case)
    assert items, case
    for seed in range(60):
        Model(items, random.Random(seed)).run()


def test_protocol_model_catches_a_planted_release_race():
    # An idle slot that releases a K/V stage without waiting for its load can
    # complete the stage's previous phase early; the model must notice.
    items = [(4, 0), (4, 0), (4, 4), (4, 0)]
    caught = 0
    for seed in range(200):
        try:
            Model(items, random.Random(seed), planted_bug=True).run()
        except Violation:
            caught += 1
    assert caught > 0


def test_kernel_items_cover_every_q_tile_once():
    for BH, N, causal, sms in [(64, 2048, False, 148), (80, 1000, False, 148), (3, 300, False, 2),
                               (4, 2048, True, 148)]:
        n_qt = (N + 127) // 128
        n_items = None
        tiles = 0
        for cta in range(sms if not causal else BH * ((N + 255) // 256)):
            its = kernel_items(BH, N, causal, sms, cta)
            tiles += sum((T0 > 0) + (T1 > 0) for T0, T1 in its)
        assert tiles == BH * n_qt, (BH, N, causal, sms, tiles)


def test_model_counts_are_the_kernels():
    """Each K/V stage and Q buffer is released by both MMA-issuing warps (one
    per Q-tile slot); S is freed and P published by the 4 warps of a group."""
    assert K["kv_empty"] == K["q_empty"] == 2
    assert K["s_free"] == K["p_full"] == WARPS_PER_GROUP
    assert all(K[n] == 1 for n in ("q_full", "k_full", "v_full", "s_full", "pv_done", "o_final"))
