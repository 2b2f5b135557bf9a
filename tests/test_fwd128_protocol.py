"""CPU model of the synchronisation protocol of the d = 128 forward kernel.

``fwd_kernel<128, CAUSAL, FP8>`` (csrc/fa_fwd.cu) takes one Q-tile pair per
CTA.  The model runs its roles as coroutines: the TMA producer (both Q tiles
once, K/V through a 2-stage ring), the single MMA warp (for each K/V tile, per
slot: O_g += P_g V, then S_g of the next tile written over P_g), the two
softmax warpgroups (P_g written over S_g in TMEM, O_g rescaled in place), the
TMA engine (loads complete asynchronously) and the in-order tensor pipe.  A
random scheduler with per-run random speeds interleaves them.  Every wait
names the completion it intends (the kernel's parity expression), and the
model checks for deadlock, exact phases, and that no buffer is rewritten while
a read of it is pending: S_g(j+1) over P_g(j) only after O_g += P_g(j) V
executed, O_g rescaled only after the previous product on it executed, the
epilogue only after the last product, K/V stages refilled only after every
product that reads them executed.  A planted mistake must be caught.
"""
import random

import pytest

import kernel_constants as kc

NST = kc.ring_depth("fa_fwd.cu", "kNST", 128)   # K/V ring depth at d = 128 (32 KB tiles)
K = kc.barrier_counts("fa_fwd.cu")
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
        return (self.completed & 1) != (k & 1)


class Violation(Exception):
    pass


class Model:
    def __init__(self, T, rescale, rng, plant=None):
        self.T, self.rescale, self.rng, self.plant = T, rescale, rng, plant
        B = Bar
        self.q = B("q", K["q"])
        self.k_full = [B(f"k_full{s}", K["k_full"]) for s in range(NST)]
        self.v_full = [B(f"v_full{s}", K["v_full"]) for s in range(NST)]
        self.kv_empty = [B(f"kv_empty{s}", K["kv_empty"]) for s in range(NST)]
        self.s_full = [B(f"s_full{g}", K["s_full"]) for g in range(2)]
        self.p_full = [B(f"p_full{g}", kc.per_agent(K["p_full"], WARPS_PER_GROUP, "p_full")) for g in range(2)]
        self.o_final = [B(f"o_final{g}", K["o_final"]) for g in range(2)]
        self.speeds = {}
        self.pipe, self.tma = [], []
        self.s_exec = [0, 0]        # S_g tiles executed
        self.pv_exec = [0, 0]       # O_g += P_g V executed
        self.p_written = [0, 0]     # P_g tiles written by the softmax
        self.kv_reads = {}          # tile -> products done reading it

    def wait(self, bar, k):
        return ("wait", bar, k)

    def speed(self, actor):
        if actor not in self.speeds:
            self.speeds[actor] = 10.0 ** self.rng.uniform(-3.0, 0.0)
        return self.speeds[actor]

    def readers(self, j):
        return 2 * sum(1 for g in range(2) if j < self.T[g])   # S reads K, PV reads V

    # ------------------------------------------------------------------ roles
    def producer(self):
        self.tma.append(self.q)
        for j in range(max(self.T)):
            s = j % NST
            if j >= NST:
                yield self.wait(self.kv_empty[s], j // NST - 1)
                if self.kv_reads.get(j - NST, 0) != self.readers(j - NST):
                    raise Violation(f"K/V stage {s} refilled while tile {j - NST} is still read")
            self.tma.append(self.k_full[s])
            self.tma.append(self.v_full[s])

    def mma(self):
        T, Tmax = self.T, max(self.T)
        yield self.wait(self.q, 0)
        yield self.wait(self.k_full[0], 0)
        for g in range(2):
            if T[g] > 0:
                self.pipe.append(("S", g, 0))
                self.pipe.append(("commit", self.s_full[g]))
        for j in range(Tmax):
            s = j % NST
            yield self.wait(self.v_full[s], j // NST)
            k_next_ready = False
            for g in range(2):
                if j >= T[g]:
                    continue
                if self.plant != "no_p_full":
                    yield self.wait(self.p_full[g], j)
                self.pipe.append(("PV", g, j))
                if j + 1 < T[g]:
                    if not k_next_ready:
                        yield self.wait(self.k_full[(j + 1) % NST], (j + 1) // NST)
                        k_next_ready = True
                    self.pipe.append(("S", g, j + 1))
                    self.pipe.append(("commit", self.s_full[g]))
                else:
                    self.pipe.append(("commit", self.o_final[g]))
            self.pipe.append(("commit", self.kv_empty[s]))
        if Tmax > 0:
            yield self.wait(self.kv_empty[(Tmax - 1) % NST], (Tmax - 1) // NST)

    def softmax(self, g):
        for j in range(self.T[g]):
            yield self.wait(self.s_full[g], j)
            if self.s_exec[g] < j + 1:
                raise Violation(f"S_{g}({j}) read before it was computed")
            # P_g(j) over S_g(j); O_g rescaled in place when the reference max moves
            if self.rescale(g, j) and self.pv_exec[g] < j:
                raise Violation(f"O_{g} rescaled before O_{g} += P_{g}({j - 1}) V executed")
            self.p_written[g] += 1
            self.p_full[g].arrive()
        if self.T[g] > 0:
            yield self.wait(self.o_final[g], 0)
            if self.pv_exec[g] != self.T[g]:
                raise Violation(f"epilogue of slot {g} before its last product")

    # -------------------------------------------------------------- execution
    def exec_pipe(self):
        entry = self.pipe.pop(0)
        if entry[0] == "commit":
            entry[1].arrive()
            return
        op, g, j = entry
        if op == "S":
            if j > 0 and self.pv_exec[g] < j:
                raise Violation(f"S_{g}({j}) overwrote P_{g}({j - 1}) before its product")
            self.s_exec[g] += 1
        else:
            if self.p_written[g] < j + 1:
                raise Violation(f"O_{g} += P_{g}({j}) V read P before it was written")
            self.pv_exec[g] += 1
        self.kv_reads[j] = self.kv_reads.get(j, 0) + 1

    def run(self, max_steps=100000):
        roles = {"producer": self.producer(), "mma": self.mma(), "sm0": self.softmax(0), "sm1": self.softmax(1)}
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


# (T_0, T_1): non-causal pairs, a pair with one tile (odd tile count), the
# single-tile blocks of the split tail, causal pairs (T_0 = T_1 - 1).
CASES = [(1, 1), (4, 4), (16, 16), (3, 0), (5, 0), (1, 2), (7, 8), (15, 16)]


@pytest.mark.parametrize("T", CASES)
@pytest.mark.parametrize("rescale_mode", ["never", "always", "random"])
def test_protocol_holds_under_random_interleavings(T, rescale_mode):
    for seed in range(40):
        pick = random.Random(seed + 1000)
        rescale = {"never": lambda g, j: False, "always": lambda g, j: j > 0,
                   "random": lambda g, j: j > 0 and pick.random() < 0.3}[rescale_mode]
        Model(T, rescale, random.Random(seed)).run()


def test_protocol_model_catches_a_planted_missing_wait():
    # Without the p_full wait, O_g += P_g V would read P_g before the softmax
    # wrote it (and S_g(j+1) would overwrite S_g(j) before it was read).
    caught = 0
    for seed in range(100):
        try:
            Model((4, 4), lambda g, j: False, random.Random(seed), plant="no_p_full").run()
        except Violation:
            caught += 1
    assert caught > 0


def test_model_counts_are_the_kernels():
    assert K["p_full"] == WARPS_PER_GROUP
    assert all(K[n] == 1 for n in ("q", "k_full", "v_full", "kv_empty", "s_full", "o_final"))
    assert NST == kc.ring_depth("fa_fwd.cu", "kNST", 128)
