"""CPU model of the mbarrier protocol of the tensor-core kernels.

Every role of one CTA (TMA warp, producer warps, MMA issuers, the tensor core
completing what they issued, drain and pool warps) is an agent that waits on
and arrives at mbarriers with the parities and counts the kernels in
csrc/conv2d_tc.cuh (both conv2d kernels), csrc/conv1d_tcx.cuh and
csrc/conv1d_tc2.cuh (two CTAs of a cluster) use.  The agents run in many random interleavings; for each
shape of the work (tiles per CTA, input-channel chunks, accumulator buffers)
the model checks:

* no deadlock: some agent can always move until all have finished;
* no stale wait: a parity wait only passes once the phase the agent needs has
  really completed (an mbarrier answers from the parity of its current phase,
  so a waiter two phases behind would pass on an old phase);
* no early arrival: every arrival lands in the phase it belongs to;
* no overwrite in use: a buffer (halo, A stage, accumulator, transposed
  buffer) is written only after the readers of its previous contents have
  released it.

A tcgen05.commit arrives when the MMAs before it complete, which the model
lets happen at any time after their issue, in issue order per issuing thread.
"""
import random

import pytest


class Barrier:
    def __init__(self, name, count):
        self.name, self.count = name, count
        self.phase = 0       # index of the current (incomplete) phase
        self.pending = 0

    def passes(self, parity):
        # mbarrier.try_wait.parity: true once the phase with this parity is the
        # last completed one, i.e. the current phase has the other parity
        return (self.phase & 1) != parity

    def arrive(self, use, who):
        assert use == self.phase, f"{who}: arrival for use {use} of {self.name} in phase {self.phase}"
        self.pending += 1
        if self.pending == self.count:
            self.pending = 0
            self.phase += 1


class Sim:
    """Barriers plus agents; an agent is a list of steps run in order:
    ("wait", barrier, parity, phases that must be done, who),
    ("arrive", barrier, use, arrivals, who),
    ("issue", counter), ("issued", counter, k)  -- ordering of a commit after its issue,
    ("owns", barrier, phases done, who)  -- a write that needs the buffer released,
    ("release", key), ("owns_all", keys, releases done, who)  -- the same with
    explicit per-buffer release counts, for buffers in several CTAs."""

    def __init__(self):
        self.bars, self.agents, self.counters = {}, [], {}

    def bar(self, name, count):
        self.bars[name] = Barrier(name, count)

    def can_run(self, st):
        if st[0] == "wait":
            _, name, parity, need, who = st
            bar = self.bars[name]
            if not bar.passes(parity):
                return False
            assert bar.phase >= need, (f"{who}: wait on {name} parity {parity} passed in phase "
                                       f"{bar.phase}, needs {need} phases done")
            return True
        if st[0] == "issued":
            return self.counters.get(st[1], 0) > st[2]
        return True

    def step(self, st):
        if st[0] == "arrive":
            _, name, use, n, who = st
            for _ in range(n):
                self.bars[name].arrive(use, who)
        elif st[0] == "issue":
            self.counters[st[1]] = self.counters.get(st[1], 0) + 1
        elif st[0] == "release":
            self.counters[st[1]] = self.counters.get(st[1], 0) + 1
        elif st[0] == "owns_all":
            _, keys, need, who = st
            for key in keys:
                assert self.counters.get(key, 0) >= need, (f"{who}: writes {key} with "
                                                           f"{self.counters.get(key, 0)} of {need} releases done")
        elif st[0] == "owns":
            _, name, need, who = st
            assert self.bars[name].phase >= need, (f"{who}: writes the buffer of {name} with "
                                                   f"{self.bars[name].phase} of {need} releases done")

    def run(self, seed):
        rng = random.Random(seed)
        pcs = [0] * len(self.agents)
        while True:
            ready = [i for i, a in enumerate(self.agents) if pcs[i] < len(a) and self.can_run(a[pcs[i]])]
            if not ready:
                left = [a[pcs[i]] for i, a in enumerate(self.agents) if pcs[i] < len(a)]
                assert not left, f"deadlock at {left}"
                break
            i = rng.choice(ready)
            self.step(self.agents[i][pcs[i]])
            pcs[i] += 1
        for bar in self.bars.values():
            assert bar.pending == 0, f"{bar.name}: {bar.pending} arrivals left over"


def add_tma_and_epilogue(sim, T, C, A, hempty_count):
    """TMA warp (halo ring of 2), drain warps (4) and pool warps (8), shared by both kernels."""
    for h in range(2):
        sim.bar(f"hfull{h}", 1)
        sim.bar(f"hempty{h}", hempty_count)
        sim.bar(f"tfull{h}", 4)
        sim.bar(f"tempty{h}", 8)
    for a in range(A):
        sim.bar(f"accfull{a}", 1)
        sim.bar(f"accempty{a}", 4)
    tma = []
    for seq in range(T * C):
        b, k = seq & 1, seq >> 1
        tma += [("wait", f"hempty{b}", (k & 1) ^ 1, k, "tma"), ("owns", f"hempty{b}", k, "tma"),
                ("arrive", f"hfull{b}", k, 1, "tma")]
    drain, pool = [], []
    for t in range(T):
        buf, rnd = t % A, t // A
        tb, tk = t & 1, t >> 1
        drain += [("wait", f"accfull{buf}", rnd & 1, rnd + 1, "drain"),
                  ("wait", f"tempty{tb}", (tk & 1) ^ 1, tk, "drain"),
                  ("owns", f"tempty{tb}", tk, "drain"),
                  ("arrive", f"accempty{buf}", rnd, 4, "drain"),
                  ("arrive", f"tfull{tb}", tk, 4, "drain")]
        pool += [("wait", f"tfull{tb}", tk & 1, tk + 1, "pool"), ("arrive", f"tempty{tb}", tk, 8, "pool")]
    sim.agents += [tma, drain, pool]


def add_issuers(sim, T, C, A, subs, stage_of):
    """Two MMA issuers (even / odd tiles); each waits "A full" of every
    sub-chunk of every chunk, and its commits (stage free per sub-chunk,
    accumulator full per tile) complete later, in order."""
    for par in range(2):
        issue, complete = [], []
        n = 0
        for t in range(par, T, 2):
            for ch in range(C):
                use = (t >> 1) * C + ch
                for sub in range(subs):
                    stage = stage_of(t, sub)
                    issue.append(("wait", f"afull{stage}", use & 1, use + 1, f"issuer{par}"))
                    if ch == 0 and sub == 0:
                        issue.append(("owns", f"accempty{t % A}", t // A, f"issuer{par}"))
                    issue.append(("issue", par))
                    complete += [("issued", par, n), ("arrive", f"aempty{stage}", use, 1, f"mma{par}")]
                    n += 1
            complete.append(("arrive", f"accfull{t % A}", t // A, 1, f"mma{par}"))
        sim.agents += [issue, complete]


def sub_chunk_kernel(T, C, A, stage_of=lambda t, g: 2 * (t & 1) + g):
    """conv2d_tc4_kernel: two producer groups of 4 warps, one per K sub-chunk;
    A stage 2 * (tile parity) + sub-chunk; group 0 also waits for the
    accumulator before a tile's first chunk."""
    sim = Sim()
    for s in range(4):
        sim.bar(f"afull{s}", 4)
        sim.bar(f"aempty{s}", 1)
    add_tma_and_epilogue(sim, T, C, A, hempty_count=8)
    for g in range(2):
        st = []
        for seq in range(T * C):
            t, ch = divmod(seq, C)
            stage, use = stage_of(t, g), (t >> 1) * C + ch
            b, k = seq & 1, seq >> 1
            st += [("wait", f"aempty{stage}", (use & 1) ^ 1, use, f"group{g}"),
                   ("wait", f"hfull{b}", k & 1, k + 1, f"group{g}")]
            if g == 0 and ch == 0:
                st.append(("wait", f"accempty{t % A}", ((t // A) & 1) ^ 1, t // A, f"group{g}"))
            st += [("owns", f"aempty{stage}", use, f"group{g}"),
                   ("arrive", f"hempty{b}", k, 4, f"group{g}"), ("arrive", f"afull{stage}", use, 4, f"group{g}")]
        sim.agents.append(st)
    add_issuers(sim, T, C, A, 2, stage_of)
    return sim


def full_chunk_kernel(T, C, A):
    """conv2d_tc_kernel: 8 producer warps (thread 0 waits for all) build a
    whole chunk into A stage (tile parity); before a tile's first chunk they
    also wait for its accumulator."""
    sim = Sim()
    for s in range(2):
        sim.bar(f"afull{s}", 8)
        sim.bar(f"aempty{s}", 1)
    add_tma_and_epilogue(sim, T, C, A, hempty_count=8)
    st = []
    for seq in range(T * C):
        t, ch = divmod(seq, C)
        stage, use = t & 1, (t >> 1) * C + ch
        b, k = seq & 1, seq >> 1
        st.append(("wait", f"aempty{stage}", (use & 1) ^ 1, use, "producers"))
        if ch == 0:
            st.append(("wait", f"accempty{t % A}", ((t // A) & 1) ^ 1, t // A, "producers"))
        st += [("wait", f"hfull{b}", k & 1, k + 1, "producers"), ("owns", f"aempty{stage}", use, "producers"),
               ("arrive", f"hempty{b}", k, 8, "producers"), ("arrive", f"afull{stage}", use, 8, "producers")]
    sim.agents.append(st)
    add_issuers(sim, T, C, A, 1, lambda t, sub: t & 1)
    return sim


def conv1d_tma_halo_kernel(T, NK, stages=2):
    """dwsep_conv1d_tcx_kernel: T tiles per CTA, NK 32-channel chunks per tile.

    `stages` smem stages (seq % stages; two for 256-wide tiles, three for
    128-wide ones) hold the pw chunk and the x halo, which the TMA warp loads
    once the MMAs that read the stage are done ("empty", a commit); 8 producer
    warps wait for the loads ("tma"), turn the halo into the A operand in place
    and arrive at "full"; one issuer waits for "full" per chunk and for the
    accumulator (local & 1) to be drained ("aempty", 4 epilogue warps) per
    tile, and commits "empty" per chunk and "afull" per tile.  The
    register-halo kernel (dwsep_conv1d_tc_kernel) has the same protocol with
    two stages: its TMA brings only the pw chunk, and its halo goes through a
    buffer only the producers use, ordered by their own group barrier."""
    sim = Sim()
    for s in range(stages):
        sim.bar(f"full{s}", 8)
        sim.bar(f"empty{s}", 1)
        sim.bar(f"tma{s}", 1)
    for b in range(2):
        sim.bar(f"afull{b}", 1)
        sim.bar(f"aempty{b}", 4)
    tma, prod = [], []
    for seq in range(T * NK):
        st, k = seq % stages, seq // stages
        tma += [("wait", f"empty{st}", (k & 1) ^ 1, k, "tma"), ("owns", f"empty{st}", k, "tma"),
                ("arrive", f"tma{st}", k, 1, "tma")]
        prod += [("wait", f"tma{st}", k & 1, k + 1, "producers"), ("owns", f"empty{st}", k, "producers"),
                 ("arrive", f"full{st}", k, 8, "producers")]
    issue, complete, epi = [], [], []
    n = 0
    for t in range(T):
        buf, bk = t & 1, t >> 1
        issue += [("wait", f"aempty{buf}", (bk & 1) ^ 1, bk, "issuer"), ("owns", f"aempty{buf}", bk, "issuer")]
        for c in range(NK):
            seq = t * NK + c
            st, k = seq % stages, seq // stages
            issue += [("wait", f"full{st}", k & 1, k + 1, "issuer"), ("issue", 0)]
            complete += [("issued", 0, n), ("arrive", f"empty{st}", k, 1, "mma")]
            n += 1
        complete.append(("arrive", f"afull{buf}", bk, 1, "mma"))
        epi += [("wait", f"afull{buf}", bk & 1, bk + 1, "epilogue"), ("arrive", f"aempty{buf}", bk, 4, "epilogue")]
    sim.agents += [tma, prod, issue, complete, epi]
    return sim


def conv1d_pair_kernel(T, NK, stages=3, relay=True, split=2, npw=8):
    """dwsep_conv1d_tc2_kernel: a cluster of two CTAs (rank 0 leads) shares
    every MMA (cta_group::2).  Each CTA's TMA warp fills its own stage once
    the MMAs that read it are done (its "empty", which the leader's
    multicast commit completes in both CTAs).  The leader's 8 producer warps
    arrive at its "full" directly; the other CTA's 8 arrive at a local "lfull",
    and one relay thread there forwards a single cluster arrival to the
    leader's "full" (9 arrivals; relay=False: all 16 producer warps arrive at
    the leader's "full" themselves).  The leader's issuer waits for "full" per
    chunk and for the accumulator to be drained by both CTAs' epilogues (its
    "aempty", 8 arrivals) per tile; its multicast commits complete "empty"
    and "afull" in both CTAs.  `split` more warps per CTA (one agent) form
    the pw lo part of each chunk and arrive beside the producers."""
    sim = Sim()
    for r in range(2):
        for s_ in range(stages):
            sim.bar(f"empty{s_}@{r}", 1)
            sim.bar(f"tma{s_}@{r}", 1)
        for b_ in range(2):
            sim.bar(f"afull{b_}@{r}", 1)
    for s_ in range(stages):
        sim.bar(f"full{s_}@0", npw + split + 1 if relay else 2 * (npw + split))
        if relay:
            sim.bar(f"lfull{s_}@1", npw + split)
    for b_ in range(2):
        sim.bar(f"aempty{b_}@0", 8)
    for r in range(2):
        sim.bar(f"last@{r}", 4)
    for r in range(2):
        tma, prod, spl = [], [], []
        for seq in range(T * NK):
            st, k = seq % stages, seq // stages
            tma += [("wait", f"empty{st}@{r}", (k & 1) ^ 1, k, f"tma{r}"), ("owns", f"empty{st}@{r}", k, f"tma{r}"),
                    ("arrive", f"tma{st}@{r}", k, 1, f"tma{r}")]
            target = f"lfull{st}@1" if (relay and r == 1) else f"full{st}@0"
            prod += [("wait", f"tma{st}@{r}", k & 1, k + 1, f"producers{r}"),
                     ("owns", f"empty{st}@{r}", k, f"producers{r}"),
                     ("arrive", target, k, npw, f"producers{r}")]
            spl += [("wait", f"tma{st}@{r}", k & 1, k + 1, f"split{r}"),
                    ("owns", f"empty{st}@{r}", k, f"split{r}"),
                    ("arrive", target, k, split, f"split{r}")]
        # the producers help drain the last tile once the epilogue warps have
        # seen it complete (a barrier used once)
        prod.append(("wait", f"last@{r}", 0, 1, f"producers{r}"))
        epi = []
        for t in range(T):
            buf, bk = t & 1, t >> 1
            epi += [("wait", f"afull{buf}@{r}", bk & 1, bk + 1, f"epilogue{r}")]
            if t == T - 1:
                epi.append(("arrive", f"last@{r}", 0, 4, f"epilogue{r}"))
            epi += [("release", f"acc{buf}@{r}"),
                    ("arrive", f"aempty{buf}@0", bk, 4, f"epilogue{r}")]
        sim.agents += [tma, prod, epi] + ([spl] if split else [])
    if relay:
        rel = []
        for seq in range(T * NK):
            st, k = seq % stages, seq // stages
            rel += [("wait", f"lfull{st}@1", k & 1, k + 1, "relay"), ("arrive", f"full{st}@0", k, 1, "relay")]
        sim.agents.append(rel)
    issue, complete = [], []
    n = 0
    for t in range(T):
        buf, bk = t & 1, t >> 1
        issue += [("wait", f"aempty{buf}@0", (bk & 1) ^ 1, bk, "issuer"),
                  ("owns_all", [f"acc{buf}@0", f"acc{buf}@1"], bk, "issuer")]
        for c in range(NK):
            seq = t * NK + c
            st, k = seq % stages, seq // stages
            issue += [("wait", f"full{st}@0", k & 1, k + 1, "issuer"), ("issue", 0)]
            complete += [("issued", 0, n), ("arrive", f"empty{st}@0", k, 1, "mma"), ("arrive", f"empty{st}@1", k, 1, "mma")]
            n += 1
        complete += [("arrive", f"afull{buf}@0", bk, 1, "mma"), ("arrive", f"afull{buf}@1", bk, 1, "mma")]
    sim.agents += [issue, complete]
    return sim


@pytest.mark.parametrize("T", [1, 2, 3, 5, 8])
@pytest.mark.parametrize("NK", [1, 2, 3, 4, 8])
def test_conv1d_pair_kernel_protocol(T, NK):
    for seed in range(30):
        conv1d_pair_kernel(T, NK).run(seed)
        conv1d_pair_kernel(T, NK, relay=False).run(seed)
        conv1d_pair_kernel(T, NK, split=0).run(seed)


@pytest.mark.parametrize("stages", [2, 3])
@pytest.mark.parametrize("T", [1, 2, 3, 5, 8])
@pytest.mark.parametrize("NK", [1, 2, 3, 8])
def test_conv1d_tma_halo_kernel_protocol(T, NK, stages):
    for seed in range(30):
        conv1d_tma_halo_kernel(T, NK, stages).run(seed)


SHAPES = [(T, C, A) for T in (1, 2, 3, 4, 7) for C in (1, 2, 3) for A in (2, 3)]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "T%d_C%d_A%d" % s)
def test_sub_chunk_kernel_protocol(shape):
    for seed in range(30):
        sub_chunk_kernel(*shape).run(seed)


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "T%d_C%d_A%d" % s)
def test_full_chunk_kernel_protocol(shape):
    for seed in range(30):
        full_chunk_kernel(*shape).run(seed)


def test_model_catches_shared_stages():
    """Plant the mistake the stage-per-tile-parity rule prevents: both issuers
    (even and odd tiles) on the same two A stages, with the use count still
    advancing every other tile.  The model must report it."""
    failures = 0
    for seed in range(50):
        try:
            sub_chunk_kernel(6, 2, 3, stage_of=lambda t, g: g).run(seed)
        except AssertionError:
            failures += 1
    assert failures > 0


def test_model_catches_a_missing_accumulator_wait():
    """Plant a data race: the producers stop waiting for the drained
    accumulator, so an issuer may start a tile on one still being read."""
    failures = 0
    for seed in range(100):
        sim = sub_chunk_kernel(7, 1, 2)
        for a in sim.agents:
            a[:] = [st for st in a if not (st[0] == "wait" and st[1].startswith("accempty"))]
        try:
            sim.run(seed)
        except AssertionError as e:
            failures += "releases done" in str(e)
    assert failures > 0


def test_model_catches_a_missing_conv1d_accumulator_wait():
    """Plant a data race in the conv1d protocol: the issuer stops waiting for
    the drained accumulator."""
    failures = 0
    for seed in range(100):
        sim = conv1d_tma_halo_kernel(6, 2)
        sim.agents[2] = [st for st in sim.agents[2] if not (st[0] == "wait" and st[1].startswith("aempty"))]
        try:
            sim.run(seed)
        except AssertionError as e:
            failures += "releases done" in str(e)
    assert failures > 0


def test_model_catches_a_leader_that_ignores_the_peer_epilogue():
    """Plant a cluster race: the leader's "accumulator drained" barrier counts
    only its own epilogue warps, so an MMA may overwrite the peer CTA's
    accumulator rows while the peer still reads them."""
    failures = 0
    for seed in range(100):
        sim = conv1d_pair_kernel(5, 3)
        for b in range(2):
            sim.bars[f"aempty{b}@0"].count = 4
        peer_epilogue = next(a for a in sim.agents if any(st[-1] == "epilogue1" for st in a))
        peer_epilogue[:] = [st for st in peer_epilogue if st[0] != "arrive"]
        try:
            sim.run(seed)
        except AssertionError as e:
            failures += "releases done" in str(e)
    assert failures > 0



# ------------------------------------------------------------------------------
# conv2d_tcs_kernel (csrc/conv2d_tcs.cuh): the input rows of a CTA's contiguous
# range of units stream through NSTG staging buffers (loader -> producers) and
# NSLOT row slots (producers -> MMA issuer); the issuer releases a slot after
# the last conv row that reads it and hands two accumulators to the epilogue.
# The abort model lets any main-loop wait give up (a timeout): every role then
# leaves its loop, the loader waits for the last box it issued on each staging
# buffer, the issuer commits a drain barrier and waits for it, and the CTA
# leaves.  At that point no TMA box and no MMA may still be in flight.


def shifted_walk(u, PH, CT, PHB):
    """(ph, first pooled row of its block, block height) of unit u: image groups,
    then blocks of PHB pooled rows, then column tiles, then pooled rows."""
    r = u % (CT * PH)
    blk = r // (PHB * CT)
    b0 = blk * PHB
    bh = min(PHB, PH - b0)
    return b0 + (r - blk * PHB * CT) % bh, b0, bh


def shifted_units(P, u0, u1, PH, CT=1, PHB=1 << 30):
    """(base row sequence number, continues into the next unit) per unit, and
    the number of rows loaded, as every role of the kernel derives them."""
    units, s = [], 0
    for u in range(u0, u1):
        ph, b0, bh = shifted_walk(u, PH, CT, PHB)
        fj = 2 if (u > u0 and ph > b0) else 0
        units.append((s - fj, u + 1 < u1 and ph + 1 < b0 + bh))
        s += P + 2 - fj
    return units, s


class AbortSim(Sim):
    """Sim whose role agents are (loop steps, steps after the loop).  A "wait"
    inside the loop may give up once the abort flag is set, or start the abort
    with probability p_abort; the role then runs its after-loop steps, whose
    waits always end (drain waits).  Asynchronous work (TMA boxes, MMAs with
    their commits) goes into FIFO queues, one per unit, which complete in order
    at any later time.

    Extra steps: ("enqueue", queue, actions) issues asynchronous work whose
    completion runs `actions`; ("mark", s, nstg) records the last box issued on
    a staging buffer; ("tma_drain", nstg, who) passes once the last box issued
    on every staging buffer has landed; ("write", buf, use) fills a buffer and
    ("read", buf, use, who) -- run when an MMA completes, i.e. at the end of its
    asynchronous read -- checks that the buffer still holds that use."""

    def __init__(self):
        super().__init__()
        self.roles, self.queues, self.done, self.last_issue, self.content = [], {}, {}, {}, {}

    def can_run(self, st):
        if st[0] in ("write", "read"):
            return True
        if st[0] == "tma_drain":
            _, nstg, _who = st
            for b in range(nstg):
                last = self.last_issue.get(b)
                if last is not None and self.bars[f"stgf{b}"].phase < last // nstg + 1:
                    return False
            return True
        if st[0] in ("enqueue", "mark", "end_loop"):
            return True
        return super().can_run(st)

    def step(self, st):
        if st[0] == "enqueue":
            self.queues.setdefault(st[1], []).append(st[2])
            self.counters[st[1]] = self.counters.get(st[1], 0) + 1
        elif st[0] == "mark":
            self.last_issue[st[1] % st[2]] = st[1]
        elif st[0] == "write":
            self.content[st[1]] = st[2]
        elif st[0] == "read":
            _, buf, use, who = st
            assert self.content.get(buf) == use, (f"{who}: {buf} use {use} overwritten by use "
                                                  f"{self.content.get(buf)} before the read completed")
        elif st[0] in ("tma_drain", "end_loop"):
            pass
        else:
            super().step(st)

    def complete(self, q):
        self.done[q] = self.done.get(q, 0) + 1
        for act in self.queues[q].pop(0):
            self.step(act)

    def run(self, seed, p_abort=0.0):
        rng = random.Random(seed)
        steps = [list(m) + [("end_loop",)] + list(post) for m, post in self.roles]
        post_at = [len(m) for m, _ in self.roles]
        pcs = [0] * len(steps)
        aborted = False
        while True:
            if all(pcs[i] >= len(a) for i, a in enumerate(steps)):
                # The CTA leaves (__syncthreads, TMEM dealloc, exit): nothing it
                # issued may still be in flight.
                for q, n in self.counters.items():
                    assert self.done.get(q, 0) == n, f"{q}: {n - self.done.get(q, 0)} still in flight at exit"
                break
            moves = []
            for i, a in enumerate(steps):
                if pcs[i] >= len(a):
                    continue
                st = a[pcs[i]]
                if st[0] == "wait" and pcs[i] < post_at[i] and (aborted or p_abort > 0):
                    moves.append(("giveup", i))
                if self.can_run(st):
                    moves.append(("role", i))
            for q, items in self.queues.items():
                if items:
                    moves.append(("complete", q))
            assert moves, "deadlock at " + str([a[pcs[i]] for i, a in enumerate(steps) if pcs[i] < len(a)])
            kind, i = rng.choice(moves)
            if kind == "giveup":
                if not aborted and rng.random() > p_abort:
                    continue
                aborted = True
                pcs[i] = post_at[i] + 1
            elif kind == "role":
                self.step(steps[i][pcs[i]])
                pcs[i] += 1
            else:
                self.complete(i)
        if not aborted:
            for bar in self.bars.values():
                assert bar.pending == 0, f"{bar.name}: {bar.pending} arrivals left over"
        return aborted


def shifted_kernel(P, u0, u1, PH, nslot, nstg, nprod=4, planted=None, CT=1, PHB=1 << 30):
    """The roles of conv2d_tcs_kernel for one CTA with units [u0, u1) of strips of
    PH pooled rows.  `planted` names a mistake to plant: "drain_only_if_aborted"
    (the loader skips its drain when its own loop ended normally), "early_release"
    (a slot is released one conv row early), "no_acc_wait" (the issuer does not
    wait for a drained accumulator)."""
    units, S = shifted_units(P, u0, u1, PH, CT, PHB)
    sim = AbortSim()
    for b in range(nstg):
        sim.bar(f"stgf{b}", 1)
        sim.bar(f"stge{b}", 1)
    for b in range(nslot):
        sim.bar(f"slotf{b}", 1)
        sim.bar(f"slote{b}", 1)
    for b in range(2):
        sim.bar(f"accf{b}", 1)
        sim.bar(f"acce{b}", 4)
    sim.bar("drain", 1)
    # loader: one box per row into staging buffer s % nstg (the TMA unit lands it later)
    loop = []
    for s in range(S):
        b, k = s % nstg, s // nstg
        loop += [("wait", f"stge{b}", (k & 1) ^ 1, k, "loader"), ("owns", f"stge{b}", k, "loader"),
                 ("enqueue", "tma", [("arrive", f"stgf{b}", k, 1, "tma")]), ("mark", s, nstg)]
    sim.roles.append((loop, [] if planted == "drain_only_if_aborted" else [("tma_drain", nstg, "loader")]))
    # producers: row s -> warp s % nprod
    for w in range(nprod):
        loop = []
        for s in range(w, S, nprod):
            b, k, sl, ks = s % nstg, s // nstg, s % nslot, s // nslot
            loop += [("wait", f"slote{sl}", (ks & 1) ^ 1, ks, f"prod{w}"),
                     ("wait", f"stgf{b}", k & 1, k + 1, f"prod{w}"),
                     ("owns", f"slote{sl}", ks, f"prod{w}"), ("write", f"slot{sl}", ks),
                     ("arrive", f"slotf{sl}", ks, 1, f"prod{w}"), ("arrive", f"stge{b}", k, 1, f"prod{w}")]
        sim.roles.append((loop, []))
    # MMA issuer; a commit arrives once the MMAs before it have completed
    loop = []
    shift = 1 if planted == "early_release" else 0
    released = set()

    def commit(bar, use):
        loop.append(("enqueue", "mma", [("arrive", bar, use, 1, "tcore")]))

    confirmed = -1  # the issuer waits for a row only the first time it needs it
    for i, (base, cont) in enumerate(units):
        ab, ak = i & 1, i >> 1
        if planted != "no_acc_wait":
            loop.append(("wait", f"acce{ab}", (ak & 1) ^ 1, ak, "mma"))
        loop.append(("owns", f"acce{ab}", ak, "mma"))
        for dy in range(P):
            for ky in range(3):
                q = base + dy + ky
                if q > confirmed:
                    loop.append(("wait", f"slotf{q % nslot}", (q // nslot) & 1, q // nslot + 1, "mma"))
                    confirmed = q
            # the conv row's MMAs read the three rows until they complete
            loop.append(("enqueue", "mma", [("read", f"slot{q % nslot}", q // nslot, "mma")
                                            for q in range(base + dy, base + dy + 3)]))
            r = base + dy + shift
            if r not in released:
                released.add(r)
                commit(f"slote{r % nslot}", r // nslot)
        if not cont:
            for r in (base + P, base + P + 1):
                if r not in released:
                    released.add(r)
                    commit(f"slote{r % nslot}", r // nslot)
        commit(f"accf{ab}", ak)
    sim.roles.append((loop, [("enqueue", "mma", [("arrive", "drain", 0, 1, "tcore")]),
                             ("wait", "drain", 0, 1, "mma")]))
    # epilogue: its four warps take one decision per unit (one thread waits)
    loop = []
    for i in range(len(units)):
        ab, ak = i & 1, i >> 1
        loop += [("wait", f"accf{ab}", ak & 1, ak + 1, "epilogue"), ("arrive", f"acce{ab}", ak, 4, "epilogue")]
    sim.roles.append((loop, []))
    return sim


SHIFT_UNITS = [(0, 1, 5), (0, 3, 5), (2, 9, 5), (0, 12, 4), (3, 4, 1), (0, 6, 2), (4, 11, 3)]


@pytest.mark.parametrize("P", [1, 2, 4, 8])
@pytest.mark.parametrize("units", SHIFT_UNITS, ids=lambda u: "u%d-%d_ph%d" % u)
@pytest.mark.parametrize("nslot,nstg", [(8, 4), (4, 4)])
def test_shifted_kernel_protocol(P, units, nslot, nstg):
    for seed in range(15):
        shifted_kernel(P, *units, nslot, nstg).run(seed)


@pytest.mark.parametrize("P", [2, 4])
@pytest.mark.parametrize("walk", [(0, 40, 7, 3, 2), (5, 33, 9, 2, 4), (1, 20, 5, 4, 8), (0, 12, 3, 5, 1)],
                         ids=lambda w: "u%d-%d_ph%d_ct%d_b%d" % w)
def test_shifted_kernel_blocked_walk_protocol(P, walk):
    """The walk in blocks of PHB pooled rows (every column tile of a block, then
    the next block): continuations only inside a block and column tile."""
    u0, u1, PH, CT, PHB = walk
    for seed in range(15):
        shifted_kernel(P, u0, u1, PH, 8, 4, CT=CT, PHB=PHB).run(seed)
        shifted_kernel(P, u0, u1, PH, 8, 4, CT=CT, PHB=PHB).run(seed, p_abort=0.05)


@pytest.mark.parametrize("P", [1, 4])
@pytest.mark.parametrize("units", SHIFT_UNITS, ids=lambda u: "u%d-%d_ph%d" % u)
def test_shifted_kernel_abort_leaves_nothing_in_flight(P, units):
    """Any main-loop wait may give up: afterwards every role leaves, and when the
    CTA exits no TMA box or MMA is in flight."""
    aborted = 0
    for seed in range(60):
        aborted += shifted_kernel(P, *units, 8, 4).run(seed, p_abort=0.05)
        aborted += shifted_kernel(P, *units, 4, 4).run(seed, p_abort=0.05)
    assert aborted > 0


def _planted_failures(planted, P=2, units=(0, 9, 4), p_abort=0.0, seeds=200, match="", nslot=8, nstg=4):
    failures = 0
    for seed in range(seeds):
        try:
            shifted_kernel(P, *units, nslot, nstg, planted=planted).run(seed, p_abort=p_abort)
        except AssertionError as e:
            failures += match in str(e)
    return failures


def test_shifted_model_catches_a_loader_that_drains_only_after_its_own_timeout():
    """The mistake fixed in every TMA-issuing warp: a loader whose own loop ends
    normally, while another role gave up, leaves boxes in flight at exit."""
    assert _planted_failures("drain_only_if_aborted", p_abort=0.05, match="still in flight") > 0


def test_shifted_model_catches_an_early_slot_release():
    """A slot released one conv row early is refilled while the MMAs of the
    next conv row still read it."""
    assert _planted_failures("early_release", match="overwritten") + \
        _planted_failures("early_release", match="deadlock") > 0


def test_shifted_model_catches_a_missing_accumulator_wait():
    assert _planted_failures("no_acc_wait", match="releases done") > 0


def test_shifted_model_catches_buffers_shared_between_producer_warps():
    """Four producer warps taking rows in turn over three staging buffers:
    successive uses of one buffer then belong to different warps, and a warp
    can wait on a buffer two phases ahead of it, where the parity wait passes
    on a stale phase."""
    assert _planted_failures(None, nslot=8, nstg=3, match="needs") > 0


# ------------------------------------------------------------------------------
# dwsep_conv1d_tc2_kernel's abort path (csrc/conv1d_tc2.cuh): both CTAs of the
# pair watch each other's abort flag, so one flag ends every main-loop wait of
# the pair (the model's abort is global).  Each TMA warp then waits for the
# last box it issued on every stage, the leader commits a drain barrier to both
# CTAs after its last MMA and both wait for it, and the pair leaves together
# (closing cluster barrier): no box or MMA of either CTA may be in flight.


class PairAbortSim(AbortSim):
    """AbortSim with one TMA queue and drain per CTA: ("mark2", r, s, nstg)
    records the last box CTA r issued on a stage, ("tma_drain2", r, nstg, who)
    passes once each of them has landed."""

    def __init__(self):
        super().__init__()
        self.last2 = {0: {}, 1: {}}

    def can_run(self, st):
        if st[0] == "mark2":
            return True
        if st[0] == "tma_drain2":
            _, r, nstg, _who = st
            for b, last in self.last2[r].items():
                if self.bars[f"tma{b}@{r}"].phase < last // nstg + 1:
                    return False
            return True
        return super().can_run(st)

    def step(self, st):
        if st[0] == "mark2":
            self.last2[st[1]][st[2] % st[3]] = st[2]
        elif st[0] == "tma_drain2":
            pass
        else:
            super().step(st)


def conv1d_pair_abort_kernel(T, NK, stages=3, npw=8, split=2):
    sim = PairAbortSim()
    for r in range(2):
        for s_ in range(stages):
            sim.bar(f"empty{s_}@{r}", 1)
            sim.bar(f"tma{s_}@{r}", 1)
        for b_ in range(2):
            sim.bar(f"afull{b_}@{r}", 1)
        sim.bar(f"drain@{r}", 1)
        sim.bar(f"last@{r}", 4)
    for s_ in range(stages):
        sim.bar(f"full{s_}@0", npw + split + 1)
        sim.bar(f"lfull{s_}@1", npw + split)
    for b_ in range(2):
        sim.bar(f"aempty{b_}@0", 8)
    n = T * NK
    for r in range(2):
        tma, prod, spl = [], [], []
        target = "full{}@0" if r == 0 else "lfull{}@1"
        for seq in range(n):
            st, k = seq % stages, seq // stages
            tma += [("wait", f"empty{st}@{r}", (k & 1) ^ 1, k, f"tma{r}"), ("owns", f"empty{st}@{r}", k, f"tma{r}"),
                    ("enqueue", f"box{r}", [("arrive", f"tma{st}@{r}", k, 1, f"box{r}")]), ("mark2", r, seq, stages)]
            prod += [("wait", f"tma{st}@{r}", k & 1, k + 1, f"producers{r}"),
                     ("owns", f"empty{st}@{r}", k, f"producers{r}"), ("write", f"A{st}@{r}", k)]
            if not split:  # stride 2: the producers form B_lo after their halo barrier
                prod.append(("write", f"B{st}@{r}", k))
            prod.append(("arrive", target.format(st), k, npw, f"producers{r}"))
            spl += [("wait", f"tma{st}@{r}", k & 1, k + 1, f"split{r}"),
                    ("owns", f"empty{st}@{r}", k, f"split{r}"), ("write", f"B{st}@{r}", k),
                    ("arrive", target.format(st), k, split, f"split{r}")]
        prod.append(("wait", f"last@{r}", 0, 1, f"producers{r}"))  # skipped after an abort: a loop wait
        epi = []
        for t in range(T):
            buf, bk = t & 1, t >> 1
            epi += [("wait", f"afull{buf}@{r}", bk & 1, bk + 1, f"epilogue{r}")]
            if t == T - 1:
                epi.append(("arrive", f"last@{r}", 0, 4, f"epilogue{r}"))
            epi.append(("arrive", f"aempty{buf}@0", bk, 4, f"epilogue{r}"))
        sim.roles += [(tma, [("tma_drain2", r, stages, f"tma{r}")]), (prod, [])] + ([(spl, [])] if split else []) + \
            [(epi, [])]
    rel = []
    for seq in range(n):
        st, k = seq % stages, seq // stages
        rel += [("wait", f"lfull{st}@1", k & 1, k + 1, "relay"), ("arrive", f"full{st}@0", k, 1, "relay")]
    sim.roles.append((rel, [("wait", "drain@1", 0, 1, "mma1")]))
    iss = []
    for t in range(T):
        buf, bk = t & 1, t >> 1
        iss += [("wait", f"aempty{buf}@0", (bk & 1) ^ 1, bk, "issuer"), ("owns", f"aempty{buf}@0", bk, "issuer")]
        for c in range(NK):
            seq = t * NK + c
            st, k = seq % stages, seq // stages
            iss += [("wait", f"full{st}@0", k & 1, k + 1, "issuer"),
                    ("enqueue", "mma", [("read", f"{op}{st}@{r}", k, "mma") for op in "AB" for r in range(2)]),
                    ("enqueue", "mma", [("arrive", f"empty{st}@0", k, 1, "mma"),
                                        ("arrive", f"empty{st}@1", k, 1, "mma")])]
        iss.append(("enqueue", "mma", [("arrive", f"afull{buf}@0", bk, 1, "mma"),
                                       ("arrive", f"afull{buf}@1", bk, 1, "mma")]))
    sim.roles.append((iss, [("enqueue", "mma", [("arrive", "drain@0", 0, 1, "mma"), ("arrive", "drain@1", 0, 1, "mma")]),
                            ("wait", "drain@0", 0, 1, "issuer")]))
    return sim


@pytest.mark.parametrize("T", [1, 2, 3, 5])
@pytest.mark.parametrize("NK", [1, 2, 3, 8])
def test_conv1d_pair_abort_leaves_nothing_in_flight(T, NK):
    """Any main-loop wait of either CTA may give up: afterwards every role of
    both CTAs leaves, and when the pair exits no TMA box of either CTA and no
    MMA is in flight; without an abort the protocol runs to the end."""
    aborted = 0
    for seed in range(40):
        for split in (2, 0):  # stride 1 (pw split warps) and stride 2 (the producers form B_lo)
            conv1d_pair_abort_kernel(T, NK, split=split).run(seed)
            aborted += conv1d_pair_abort_kernel(T, NK, split=split).run(seed, p_abort=0.05)
    assert aborted > 0


def test_pair_abort_model_catches_a_missing_tma_drain():
    """Plant the mistake: the peer CTA's TMA warp leaves without waiting for its
    boxes.  Some abort must then find a box still in flight at exit."""
    failures = 0
    for seed in range(200):
        sim = conv1d_pair_abort_kernel(3, 3)
        sim.roles[4] = (sim.roles[4][0], [])  # CTA 1's TMA warp: no drain
        try:
            sim.run(seed, p_abort=0.05)
        except AssertionError as e:
            failures += "still in flight" in str(e)
    assert failures > 0
