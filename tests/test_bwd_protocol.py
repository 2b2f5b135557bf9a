"""CPU model of the synchronisation protocol of the backward main kernel.

The model runs the roles of ``bwd_kernel<D, CAUSAL, dQ>`` (csrc/fa_bwd.cu,
the path with the fp32 dQ accumulator), for d = 64 and d = 128, as
coroutines: the TMA producer, the MMA warp, the two P/dS warpgroups, the dQ
warpgroup (d = 64: TMA bulk reductions through two staging tiles; d = 128:
dQ^T read from R2 and added with red.global.add), the TMA engine (loads and reduction reads complete
asynchronously, reductions in issue order) and the in-order tensor pipe (MMAs
and ``tcgen05.commit`` arrivals execute in issue order).  A random scheduler
with per-run random speeds interleaves them.  Each mbarrier wait names the
completion it intends (the kernel's parity expression), and the model checks:

* no deadlock, and every wait that passes sees exactly its intended completion;
* no TMEM region, shared-memory buffer or ring stage is rewritten while a read
  of its previous contents is pending, and no product reads a region before
  its contents are written: K and V copied into TMEM before the first S^T
  (d = 64); at d = 128, dQ^T_i over dS^T_i in R2 only after dK_i used it, and
  dP^T_(i+1) over dQ^T_i only after the dQ group read it;
  S^T_(i+1) over P^T_i only after dV used it; dP^T_(i+1) over dS^T_i only
  after dK used it; P^T_i and dS^T_i written only after their TMEM columns
  were read; dS^T_i in shared memory only after dQ_(i-1) read it; dQ_i into
  TMEM only after the dQ group read dQ_(i-1); a dQ staging tile only after
  the reduction that read it completed its read; a Q/dO stage only after all
  four products and both groups are done with it.
A planted mistake must be caught, so the checks are not vacuous.
"""
import random

import pytest

import kernel_constants as kc

NST = kc.ring_depth("fa_bwd.cu", "kNST")   # Q / dO / statistics ring depth of the backward
# Arrive counts of the kernel's barriers.  A model agent for a P/dS group or
# the dQ group stands for that group's 4 warps, each of which arrives once.
K = kc.barrier_counts("fa_bwd.cu")
WARPS_PER_GROUP = 4


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
    def __init__(self, n_iter, rng, plant=None, d=64):
        self.n, self.rng, self.plant, self.d = n_iter, rng, plant, d
        B = Bar
        g = lambda n: kc.per_agent(K[n], WARPS_PER_GROUP, n)  # noqa: E731
        self.kv_full = B("kv_full", K["kv_full"])
        self.kv_tmem = B("kv_tmem", g("kv_tmem"))
        self.qdo_full = [B(f"qdo_full{s}", K["qdo_full"]) for s in range(NST)]
        # MMA commit + the P/dS groups
        self.qdo_empty = [B(f"qdo_empty{s}", 1 + kc.per_agent(K["qdo_empty"] - 1, WARPS_PER_GROUP, "qdo_empty"))
                          for s in range(NST)]
        self.s_ready, self.dp_ready = B("s_ready", K["s_ready"]), B("dp_ready", K["dp_ready"])
        self.p_ready, self.ds_ready = B("p_ready", g("p_ready")), B("ds_ready", g("ds_ready"))
        self.ds_free, self.dq_ready = B("ds_free", K["ds_free"]), B("dq_ready", K["dq_ready"])
        self.dq_free = B("dq_free", g("dq_free"))
        self.dq_staged = [B(f"dq_staged{b}", g("dq_staged")) for b in range(2)]
        self.dq_stage_free = [B(f"dq_stage_free{b}", K["dq_stage_free"]) for b in range(2)]
        self.final_ = B("final", K["final_"])
        self.speeds = {}
        self.pipe, self.tma, self.reduce_reads = [], [], []
        self.exec = {k: 0 for k in ("S", "dP", "dV", "dK", "dQ")}   # products executed
        self.p_done = [0, 0]      # P^T tiles written, per group
        self.ds_done = [0, 0]     # dS^T tiles written (TMEM and smem), per group
        self.kv_copied = 0
        self.dq_read = 0          # dQ tiles read out of TMEM
        self.reads_done = 0       # reductions whose shared-memory read has completed
        self.stage_reads = {}     # (stage, tile) -> products done with it

    def wait(self, bar, k):
        return ("wait", bar, k)

    def speed(self, actor):
        """Per-run random speed of each role and engine (log-uniform over three
        decades), so that some runs starve one of them for long stretches."""
        if actor not in self.speeds:
            self.speeds[actor] = 10.0 ** self.rng.uniform(-3.0, 0.0)
        return self.speeds[actor]

    # ------------------------------------------------------------------ roles
    def producer(self):
        self.tma.append(self.kv_full)
        for it in range(self.n):
            s = it % NST
            if it >= NST:
                yield self.wait(self.qdo_empty[s], it // NST - 1)
                if self.stage_reads.get((s, it - NST), 0) != 4 or min(self.ds_done) < it - NST + 1:
                    raise Violation(f"Q/dO stage {s} refilled while tile {it - NST} is still read")
            self.tma.append(self.qdo_full[s])

    def mma(self):
        yield self.wait(self.kv_full, 0)
        yield self.wait(self.qdo_full[0], 0)
        if self.d == 64:
            yield self.wait(self.kv_tmem, 0)
        self.pipe.append(("S", 0))
        self.pipe.append(("commit", self.s_ready))
        for it in range(self.n):
            s = it % NST
            if self.d == 128 and it > 0 and self.plant != "no_dq_free":
                yield self.wait(self.dq_free, it - 1)     # dP^T reuses R2, where dQ^T was
            self.pipe.append(("dP", it))
            self.pipe.append(("commit", self.dp_ready))
            yield self.wait(self.p_ready, it)
            self.pipe.append(("dV", it))
            if it + 1 < self.n:
                yield self.wait(self.qdo_full[(it + 1) % NST], (it + 1) // NST)
                self.pipe.append(("S", it + 1))
                self.pipe.append(("commit", self.s_ready))
            yield self.wait(self.ds_ready, it)
            self.pipe.append(("dK", it))
            if self.d == 64 and it > 0 and self.plant != "no_dq_free":
                yield self.wait(self.dq_free, it - 1)
            self.pipe.append(("dQ", it))
            self.pipe.append(("commit", self.dq_ready))
            self.pipe.append(("commit", self.ds_free))
            self.pipe.append(("commit", self.qdo_empty[s]))
        self.pipe.append(("commit", self.final_))
        yield self.wait(self.final_, 0)

    def pds(self, h):
        if self.d == 64:
            yield self.wait(self.kv_full, 0)
            self.kv_copied += 1
            self.kv_tmem.arrive()
        for it in range(self.n):
            s = it % NST
            yield self.wait(self.qdo_full[s], it // NST)
            yield self.wait(self.s_ready, it)
            # P^T_it over the S^T columns just read: dV_(it-1) must have read P^T_(it-1)
            if self.exec["dV"] < it:
                raise Violation(f"P^T_{it} written before dV_{it - 1} read P^T_{it - 1}")
            self.p_done[h] += 1
            self.p_ready.arrive()
            yield self.wait(self.dp_ready, it)
            if it > 0:
                yield self.wait(self.ds_free, it - 1)
            # dS^T_it over the dP^T columns (dK_(it-1) read the previous dS^T there)
            # and into shared memory (dQ_(it-1) read the previous one)
            if self.exec["dK"] < it or self.exec["dQ"] < it:
                raise Violation(f"dS^T_{it} written before dK/dQ of tile {it - 1} read the previous one")
            self.ds_done[h] += 1
            self.ds_ready.arrive()
            self.qdo_empty[s].arrive()
        yield self.wait(self.final_, 0)
        if min(self.exec.values()) < self.n:
            raise Violation("epilogue before every product executed")

    def dq_group(self):
        if self.d == 128:                                # dQ^T from R2, then red.global.add
            for it in range(self.n):
                yield self.wait(self.dq_ready, it)
                self.dq_read += 1
                self.dq_free.arrive()
            return
        for it in range(self.n):
            b = it & 1
            yield self.wait(self.dq_ready, it)
            self.dq_read += 1
            self.dq_free.arrive()
            if it >= 2:
                yield self.wait(self.dq_stage_free[b], (it >> 1) - 1)
                if self.reads_done < it - 1:
                    raise Violation(f"dQ staging tile {b} rewritten before reduction {it - 2} read it")
            self.dq_staged[b].arrive()
            yield self.wait(self.dq_staged[b], it >> 1)
            self.reduce_reads.append(it)                 # TMA reduction of tile it issued
            # wait_group_read<1>: every reduction but the newest has read its tile
            while self.reads_done < it:
                yield ("poll", lambda it=it: self.reads_done >= it)
            if it >= 1:
                self.dq_stage_free[b ^ 1].arrive()
        while self.reads_done < self.n:
            yield ("poll", lambda: self.reads_done >= self.n)

    # -------------------------------------------------------------- execution
    def exec_pipe(self):
        op, x = self.pipe.pop(0)
        if op == "commit":
            x.arrive()
            return
        it = x
        s = it % NST
        if op == "S":
            if self.d == 64 and self.kv_copied < 2:
                raise Violation("S^T issued before K and V were copied into TMEM")
            if it > 0 and (self.exec["dV"] < it or min(self.p_done) < it):
                raise Violation(f"S^T_{it} overwrote P^T_{it - 1} before it was used")
        elif op == "dP":
            if it > 0 and (self.exec["dK"] < it or min(self.ds_done) < it):
                raise Violation(f"dP^T_{it} overwrote dS^T_{it - 1} before it was used")
            if self.d == 128 and self.dq_read < it:
                raise Violation(f"dP^T_{it} overwrote dQ^T_{it - 1} before the dQ group read it")
        elif op == "dV":
            if min(self.p_done) < it + 1:
                raise Violation(f"dV_{it} read P^T before it was written")
        elif op in ("dK", "dQ"):
            if min(self.ds_done) < it + 1:
                raise Violation(f"{op}_{it} read dS^T before it was written")
            if op == "dQ" and self.dq_read < it:
                raise Violation(f"dQ_{it} overwrote dQ_{it - 1} before the dQ group read it")
            if op == "dQ" and self.d == 128 and self.exec["dK"] < it + 1:
                raise Violation(f"dQ^T_{it} overwrote dS^T_{it} in R2 before dK_{it} read it")
        self.exec[op] += 1
        if op in ("S", "dP", "dV", "dK"):
            self.stage_reads[(s, it)] = self.stage_reads.get((s, it), 0) + 1

    def run(self, max_steps=100000):
        roles = {"producer": self.producer(), "mma": self.mma(), "pds0": self.pds(0), "pds1": self.pds(1),
                 "dq": self.dq_group()}
        pending = {}
        for nm, gen in list(roles.items()):
            pending[nm] = next(gen, None)
            if pending[nm] is None:
                del roles[nm]

        def ready(nm):
            p = pending[nm]
            return p[1]() if p[0] == "poll" else p[1].passes(p[2])

        for _ in range(max_steps):
            rdy = [nm for nm in roles if ready(nm)]
            choices = rdy + (["tma"] if self.tma else []) + (["pipe"] if self.pipe else []) + \
                (["red"] if self.reduce_reads else [])
            if not choices:
                if not roles:
                    return
                raise Violation(f"deadlock: { {nm: pending[nm][1:] for nm in roles} }")
            c = self.rng.choices(choices, weights=[self.speed(x) for x in choices])[0]
            if c == "tma":
                self.tma.pop(self.rng.randrange(len(self.tma))).arrive()
            elif c == "pipe":
                self.exec_pipe()
            elif c == "red":
                self.reduce_reads.pop(0)
                self.reads_done += 1
            else:
                p = pending[c]
                if p[0] == "wait" and p[1].completed != p[2] + 1:
                    raise Violation(f"{c}: wait on {p[1].name} for completion {p[2]} passed at {p[1].completed}")
                nxt = next(roles[c], None)
                if nxt is None:
                    del roles[c]
                else:
                    pending[c] = nxt
        raise Violation("step limit")


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("n_iter", [1, 2, 3, 5, 16])
def test_protocol_holds_under_random_interleavings(n_iter, d):
    for seed in range(80):
        Model(n_iter, random.Random(seed), d=d).run()


@pytest.mark.parametrize("d", [64, 128])
def test_protocol_model_catches_a_planted_missing_wait(d):
    # Without its dq_free wait the MMA warp may overwrite dQ_(i-1) in TMEM
    # (d = 64) or dQ^T_(i-1) in R2 (d = 128) before the dQ group has read it.
    caught = 0
    for seed in range(200):
        try:
            Model(4, random.Random(seed), plant="no_dq_free", d=d).run()
        except Violation:
            caught += 1
    assert caught > 0


def test_model_counts_are_the_kernels():
    """The kernel's counts map onto the model's agents: one arrive per warp of
    the two P/dS groups (and of the dQ group), one for each commit."""
    assert K["p_ready"] == K["ds_ready"] == K["kv_tmem"] == 2 * WARPS_PER_GROUP
    assert K["qdo_empty"] == 1 + 2 * WARPS_PER_GROUP
    assert K["dq_free"] == K["dq_staged"] == WARPS_PER_GROUP
    assert all(K[n] == 1 for n in ("kv_full", "qdo_full", "s_ready", "dp_ready", "ds_free", "dq_ready",
                                   "final_", "dq_stage_free"))
    assert NST >= 2
