"""Host model of the mbarrier hand-offs inside one attention CTA.

The producer thread, the MMA-issuing thread and the two Q tiles' softmax
groups of attn.cuh (one shared K + V^T ring of kStages slots) and attn8.cuh
(a K ring and a V^T ring of their own, K issued kLead blocks ahead) are
replayed as coroutines, in the order the kernels issue their waits, loads,
MMAs, commits and arrivals, under random interleavings:

* a TMA load completes its full barrier at some later time;
* tcgen05.mma and tcgen05.commit go through one in-order pipe, and a commit
  completes its barrier when the pipe reaches it (all earlier MMAs done);
* softmax arrivals complete their barrier at once (the whole group of 256
  threads is one arrival here).

A wait on an mbarrier passes a parity, so it is only correct while the
barrier is at most one phase ahead of the phase the waiter means and not
behind it.  The model checks, for every wait, that no waiter starts more
than one phase early, that no barrier completes a second phase while a
waiter for the first is still blocked, and that every schedule runs to the
end (no deadlock).  It also tracks what each buffer holds: a load that
lands writes its block into its slot, an MMA checks when the pipe executes
it that its K / V^T slots, P buffer and S buffer hold what it means to read
or overwrite, and a softmax group checks that S holds its own product.
It covers tiles with no key (causal, more queries than keys), tile 1 longer
than tile 0, one KV block, and more blocks than slots.  The same machinery
checks the two halves of a row exchanging partial row maxima through slots
double-buffered by block parity, and their row sums at the end, and the
Q-on-load start (the softmax groups quantize Q before the first S product).
"""
import random

import pytest


class Deadlock(Exception):
    pass


class Sim:
    def __init__(self, rng, arrivals=None):
        self.rng = rng
        self.need = dict(arrivals or {})  # barrier -> arrivals per phase (default 1)
        self.arrived = {}
        self.count = {}          # barrier -> completed phases
        self.waiting = {}        # agent -> (barrier, phase index it waits for)
        self.pending_loads = []  # (barrier, slot, block) of TMA loads in flight
        self.pipe = []           # ('mma', reads, writes) or ('commit', barrier), in issue order
        self.content = {}        # buffer -> what it holds
        self.agents = {}

    def complete(self, bar):
        n = self.count.get(bar, 0) + 1
        for name, (b, c) in self.waiting.items():
            if b == bar:
                assert n <= c + 1, f"{bar} reached phase {n} while {name} still waits for phase index {c}"
        self.count[bar] = n

    def run(self, agents):
        self.agents = dict(agents)
        gens = {k: v() for k, v in agents.items()}
        state = {k: None for k in gens}  # None: runnable; else the yielded request
        done = set()

        def step(name):
            try:
                req = gens[name].send(None)
            except StopIteration:
                done.add(name)
                return
            state[name] = req

        for name in gens:
            step(name)
        guard = 0
        while len(done) < len(gens):
            guard += 1
            assert guard < 10 ** 6
            runnable = []
            for name, req in state.items():
                if name in done:
                    continue
                kind = req[0]
                if kind == "wait":
                    _, bar, c = req
                    if name not in self.waiting:
                        have = self.count.get(bar, 0)
                        assert have >= c, f"{name} waits for phase index {c} of {bar} at phase {have}"
                        self.waiting[name] = (bar, c)
                    if self.count.get(bar, 0) >= c + 1:
                        runnable.append(name)
                else:
                    runnable.append(name)
            events = [("agent", n) for n in runnable]
            if self.pending_loads:
                events.append(("load", None))
            if self.pipe:
                events.append(("pipe", None))
            if not events:
                raise Deadlock({n: state[n] for n in gens if n not in done})
            kind, name = self.rng.choice(events)
            if kind == "load":
                bar, slot, block = self.pending_loads.pop(self.rng.randrange(len(self.pending_loads)))
                self.content[slot] = block
                self.complete(bar)
            elif kind == "pipe":
                op = self.pipe.pop(0)
                if op[0] == "commit":
                    self.complete(op[1])
                else:
                    for buf, want in op[1]:
                        assert self.content.get(buf) == want, f"MMA reads {buf}={self.content.get(buf)}, wants {want}"
                    for buf, val in op[2]:
                        self.content[buf] = val
            else:
                req = state[name]
                if req[0] == "wait":
                    del self.waiting[name]
                elif req[0] == "load":
                    self.pending_loads.append(req[1:])
                elif req[0] == "mma":
                    self.pipe.append(req)
                elif req[0] == "check":
                    assert self.content.get(req[1]) == req[2], f"{name} reads {req[1]}={self.content.get(req[1])}"
                elif req[0] == "write":
                    self.content[req[1]] = req[2]
                elif req[0] == "commit":
                    self.pipe.append(("commit", req[1]))
                elif req[0] == "arrive":
                    bar = req[1]
                    self.arrived[bar] = self.arrived.get(bar, 0) + 1
                    if self.arrived[bar] == self.need.get(bar, 1):
                        self.arrived[bar] = 0
                        self.complete(bar)
                step(name)


def wait(bar, c):
    return ("wait", bar, c)


def softmax(i, n_i, q_on_load=False, valid=True):
    """One Q tile's softmax group: S in, S buffer released, P out once the
    previous P V is done, the last P V awaited before the epilogue.  With Q
    on load it first waits for the bf16 Q tiles, quantizes its own (when its
    tile exists) into the MMA's Q buffer and arrives on the Q-ready barrier
    (both groups arrive, whether or not tile 1 exists)."""
    def agent():
        if q_on_load:
            yield wait("Q", 0)
            if valid:
                yield ("write", ("Qcodes", i), "q")
            yield ("arrive", "QReady")
        for j in range(n_i):
            yield wait(("SFull", i), j)
            yield ("check", "S", (i, j))
            yield ("arrive", "SEmpty")
            if j > 0:
                yield wait(("PvDone", i), j - 1)
            yield ("write", ("P", i), j)
            yield ("arrive", ("PFull", i))
        if n_i > 0:
            yield wait(("PvDone", i), n_i - 1)
    return agent


def mma_common(n0, n1, k_ready, v_ready, after_qk, after_pv, k_slot, v_slot, early_k_release=False,
               q_on_load=False, q_barrier=None):
    """The MMA thread's schedule, shared by both kernels: S products of both
    tiles for block 0, then per block j: S0(j+1), PV0(j), S1(j+1), PV1(j).
    k_slot(j) / v_slot(j): the buffers holding K and V^T of block j.
    early_k_release plants a mistake: K(j+1) released before S1(j+1).
    q_on_load: the S products read the Q codes the softmax groups wrote;
    q_barrier: the barrier waited for before the first S product (default:
    Q-ready with Q on load, the Q load else)."""
    nmax = max(n0, n1)
    nqk = [0]
    last_s = [None]  # the S product the next one overwrites (read by then)

    def issue_qk(i, j):
        if nqk[0] > 0:
            yield wait("SEmpty", nqk[0] - 1)
        q_read = ((("Qcodes", i), "q"),) if q_on_load else ()
        yield ("mma", ((k_slot(j), j), ("S", last_s[0])) + q_read, (("S", (i, j)),))
        last_s[0] = (i, j)
        yield ("commit", ("SFull", i))
        nqk[0] += 1

    def issue_pv(i, j):
        yield wait(("PFull", i), j)
        yield ("mma", ((("P", i), j), (v_slot(j), j)), ())
        yield ("commit", ("PvDone", i))

    def agent():
        yield wait(q_barrier or ("QReady" if q_on_load else "Q"), 0)
        if nmax == 0:
            return
        yield from k_ready(0)
        if n0 > 0:
            yield from issue_qk(0, 0)
        if n1 > 0:
            yield from issue_qk(1, 0)
        yield from after_qk(0)
        for j in range(nmax):
            if j + 1 < nmax:
                yield from k_ready(j + 1)
            yield from v_ready(j)
            if j + 1 < n0:
                yield from issue_qk(0, j + 1)
            if j < n0:
                yield from issue_pv(0, j)
            if early_k_release and j + 1 < nmax:
                yield from after_qk(j + 1)
            if j + 1 < n1:
                yield from issue_qk(1, j + 1)
            if not early_k_release and j + 1 < nmax:
                yield from after_qk(j + 1)
            if j < n1:
                yield from issue_pv(1, j)
            yield from after_pv(j)
    return agent


def fp4_agents(n0, n1, stages, q_on_load=False, mma_waits_q_ready=True):
    """attn.cuh: one ring of K, its scales, V^T and its scales per block.
    q_on_load: the softmax groups quantize the bf16 Q tiles the producer
    loads; mma_waits_q_ready=False plants a mistake (the MMA waits only for
    the bf16 load)."""
    nmax = max(n0, n1)

    def producer():
        yield ("load", "Q", "Q", 0)
        for j in range(nmax):
            s, u = j % stages, j // stages
            if u > 0:
                yield wait(("KvEmpty", s), u - 1)
            yield ("load", ("KvFull", s), ("KV", s), j)
        # drain: the last `stages` loads
        for j in range(max(0, nmax - stages), nmax):
            yield wait(("KvFull", j % stages), j // stages)

    def k_ready(j):
        yield wait(("KvFull", j % stages), j // stages)

    def nothing(j):
        return
        yield

    def after_pv(j):
        yield ("commit", ("KvEmpty", j % stages))

    def slot(j):
        return ("KV", j % stages)

    mma = mma_common(n0, n1, k_ready, nothing, nothing, after_pv, slot, slot, q_on_load=q_on_load,
                     q_barrier=None if mma_waits_q_ready else "Q")
    return {"producer": producer, "mma": mma,
            "softmax0": softmax(0, n0, q_on_load, True), "softmax1": softmax(1, n1, q_on_load, n1 > 0)}


def i8_agents(n0, n1, k_stages, v_stages, early_k_release=False):
    """attn8.cuh: K and V^T in rings of their own, K issued kLead ahead."""
    nmax = max(n0, n1)
    lead = k_stages + 1 - v_stages

    def producer():
        yield ("load", "Q", "Q", 0)
        for t in range(nmax + lead):
            if t < nmax:
                s, r = t % k_stages, t // k_stages
                if r > 0:
                    yield wait(("KEmpty", s), r - 1)
                yield ("load", ("KFull", s), ("K", s), t)
            j = t - lead
            if 0 <= j < nmax:
                s, r = j % v_stages, j // v_stages
                if r > 0:
                    yield wait(("VEmpty", s), r - 1)
                yield ("load", ("VFull", s), ("V", s), j)
        for j in range(max(0, nmax - k_stages), nmax):
            yield wait(("KFull", j % k_stages), j // k_stages)
        for j in range(max(0, nmax - v_stages), nmax):
            yield wait(("VFull", j % v_stages), j // v_stages)

    def k_ready(j):
        yield wait(("KFull", j % k_stages), j // k_stages)

    def v_ready(j):
        yield wait(("VFull", j % v_stages), j // v_stages)

    def after_qk(j):
        yield ("commit", ("KEmpty", j % k_stages))

    def after_pv(j):
        yield ("commit", ("VEmpty", j % v_stages))

    return {"producer": producer,
            "mma": mma_common(n0, n1, k_ready, v_ready, after_qk, after_pv, lambda j: ("K", j % k_stages),
                              lambda j: ("V", j % v_stages), early_k_release),
            "softmax0": softmax(0, n0), "softmax1": softmax(1, n1)}


# (n0, n1): KV blocks seen by Q tile 0 and 1.  Causal pairs have n1 = n0 + 1
# (or n0 when the key tail ends inside tile 0's diagonal block); a pair of
# single-tile units has n1 = 0; with more queries than keys tile 0 may see
# none.
BLOCKS = [(1, 0), (1, 1), (1, 2), (2, 2), (3, 3), (5, 5), (6, 7), (7, 7), (12, 13), (13, 13), (32, 32),
          (0, 1), (0, 0), (4, 0), (20, 21)]


@pytest.mark.parametrize("stages", [3, 6])
def test_fp4_ring_has_no_deadlock_and_no_parity_alias(stages):
    for n0, n1 in BLOCKS:
        for seed in range(40):
            Sim(random.Random(seed * 7919 + n0 * 31 + n1)).run(fp4_agents(n0, n1, stages))


@pytest.mark.parametrize("k_stages,v_stages", [(3, 2), (4, 3), (2, 2)])
def test_i8_split_rings_have_no_deadlock_and_no_parity_alias(k_stages, v_stages):
    for n0, n1 in BLOCKS:
        for seed in range(40):
            Sim(random.Random(seed * 104729 + n0 * 37 + n1)).run(i8_agents(n0, n1, k_stages, v_stages))


def test_the_model_catches_a_broken_protocol():
    """Planted mistakes: the producer refills a V^T slot without waiting for
    it to be empty, K runs further ahead than its ring has slots, and a K
    slot is released before the second tile's S product has read it."""
    def producer_no_v_wait(n0, n1, k_stages, v_stages):
        agents = i8_agents(n0, n1, k_stages, v_stages)
        nmax = max(n0, n1)

        def producer():
            yield ("load", "Q", "Q", 0)
            for j in range(nmax):
                yield ("load", ("KFull", j % k_stages), ("K", j % k_stages), j)
                yield ("load", ("VFull", j % v_stages), ("V", j % v_stages), j)
        agents["producer"] = producer
        return agents

    caught = 0
    for seed in range(60):
        try:
            Sim(random.Random(seed)).run(producer_no_v_wait(8, 8, 3, 2))
        except AssertionError:
            caught += 1
    assert caught > 0

    def producer_lead_too_far(n0, n1, k_stages, v_stages):
        agents = i8_agents(n0, n1, k_stages, v_stages)
        nmax = max(n0, n1)
        lead = k_stages + 2  # more than the K ring holds

        def producer():
            yield ("load", "Q", "Q", 0)
            for t in range(nmax + lead):
                if t < nmax:
                    s, r = t % k_stages, t // k_stages
                    if r > 0:
                        yield wait(("KEmpty", s), r - 1)
                    yield ("load", ("KFull", s), ("K", s), t)
                j = t - lead
                if 0 <= j < nmax:
                    s, r = j % v_stages, j // v_stages
                    if r > 0:
                        yield wait(("VEmpty", s), r - 1)
                    yield ("load", ("VFull", s), ("V", s), j)
        agents["producer"] = producer
        return agents

    with pytest.raises(Deadlock):
        Sim(random.Random(1)).run(producer_lead_too_far(8, 8, 3, 2))

    # phases stay consistent here; only the buffer contents show the race
    caught = 0
    for seed in range(200):
        try:
            Sim(random.Random(seed)).run(i8_agents(8, 8, 3, 2, early_k_release=True))
        except AssertionError as e:
            assert "reads" in str(e), e
            caught += 1
    assert caught > 0


def exchange_agents(n_i):
    """The two halves of a row in one tile (attn.cuh and attn8.cuh softmax):
    per KV block each writes its partial row maximum into the slot of the
    block's parity, arrives on the pair's barrier (both halves per phase)
    and reads the other half's value; after the last block the row sums go
    through a slot of their own and the same barrier's next phase."""
    def half(h):
        def agent():
            for j in range(n_i):
                yield ("write", ("xch", j & 1, h), j)
                yield ("arrive", "xbar")
                yield wait("xbar", j)
                yield ("check", ("xch", j & 1, 1 - h), j)
            if n_i > 0:
                yield ("write", ("xl", h), "sum")
                yield ("arrive", "xbar")
                yield wait("xbar", n_i)
                yield ("check", ("xl", 1 - h), "sum")
        return agent
    return {"half0": half(0), "half1": half(1)}


@pytest.mark.parametrize("n_i", [1, 2, 3, 8, 33])
def test_row_max_exchange_double_buffer(n_i):
    for seed in range(200):
        Sim(random.Random(seed), arrivals={"xbar": 2}).run(exchange_agents(n_i))


def test_row_max_exchange_needs_both_slots():
    """Planted mistake: one slot for every block.  A fast half then
    overwrites the value its partner has not read yet."""
    def one_slot(n_i):
        def half(h):
            def agent():
                for j in range(n_i):
                    yield ("write", ("xch", 0, h), j)
                    yield ("arrive", "xbar")
                    yield wait("xbar", j)
                    yield ("check", ("xch", 0, 1 - h), j)
            return agent
        return {"half0": half(0), "half1": half(1)}

    caught = 0
    for seed in range(200):
        try:
            Sim(random.Random(seed), arrivals={"xbar": 2}).run(one_slot(8))
        except AssertionError:
            caught += 1
    assert caught > 0


@pytest.mark.parametrize("n0,n1", [(1, 0), (3, 3), (6, 7), (13, 13), (0, 1)])
def test_fp4_q_on_load_hand_off(n0, n1):
    for seed in range(60):
        Sim(random.Random(seed), arrivals={"QReady": 2}).run(fp4_agents(n0, n1, 6, q_on_load=True))


def test_q_on_load_without_the_ready_barrier_is_caught():
    caught = 0
    for seed in range(200):
        try:
            Sim(random.Random(seed), arrivals={"QReady": 2}).run(
                fp4_agents(6, 7, 6, q_on_load=True, mma_waits_q_ready=False))
        except AssertionError:
            caught += 1
    assert caught > 0
