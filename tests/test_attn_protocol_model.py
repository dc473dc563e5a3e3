"""A randomised model of the attention kernel's mbarrier protocol (k_attn_tc.cuh): the TMA
producer with its 3-slot K and 2-slot V rings, the two MMA issuers that alternate iterations
through turn barriers, and the two softmax groups, over random sequences of work items (full
pairs, pairs with one tile, own-block pairs whose tiles have different step counts) and random
latencies and interleavings.

Barrier model: a completion counter and pending arrivals; a parity wait is satisfied when
(completions & 1) != parity, as for mbarrier.try_wait.parity. A tcgen05.commit arrives when every
MMA its issuer issued before it has completed. The model checks that no slot is refilled while an
MMA still reads it, that every MMA reads the step (or tile) it expects, that the issuers alternate,
and that nothing deadlocks. It also follows each tile's Q buffer (gathered by the producer warp once
the previous tile of the same X has completed its last Q K^T, read by the Q K^T MMAs), the
softmax's window on S_X (no Q K^T may write S_X while the softmax reads it) and the epilogue's
window on O_X (no P V may write O_X while it is read). It is a check of the protocol's design (the kernel's waits, arrivals and
commits in their order), run on the CPU; compute-sanitizer is not available for the kernel itself.
The other tests replay the protocol bug found during development and two plausible mistakes in
the producer's Q gather, each of which must be caught.
"""
import random

KSL, VSL = 3, 2


class Bar:
    def __init__(self, count, name):
        self.count, self.pending, self.comp, self.name = count, count, 0, name

    def arrive(self):
        self.pending -= 1
        assert self.pending >= 0, self.name
        if self.pending == 0:
            self.comp += 1
            self.pending = self.count

    def ready(self, parity):
        return (self.comp & 1) != parity


class Sim:
    def __init__(self, pairs, seed, mma_lat=(5, 30)):
        self.rng = random.Random(seed)
        self.mma_lat = mma_lat
        self.t = 0
        self.events = []  # (time, seq, fn)
        self.seq = 0
        self.pairs = pairs  # list of (ns, n0, n1)
        B = Bar
        self.k_full = [B(1, f'kf{s}') for s in range(KSL)]
        self.k_empty = [B(2, f'ke{s}') for s in range(KSL)]
        self.v_full = [B(1, f'vf{s}') for s in range(VSL)]
        self.v_empty = [B(2, f've{s}') for s in range(VSL)]
        self.q_full = [B(1, f'q{x}') for x in range(2)]
        self.q_empty = [B(1, f'qe{x}') for x in range(2)]
        self.s_full = [B(1, f's{x}') for x in range(2)]
        self.p_full = [B(1, f'p{x}') for x in range(2)]
        self.o_full = [B(1, f'o{x}') for x in range(2)]
        self.o_empty = [B(1, f'oe{x}') for x in range(2)]
        self.turn = [B(1, f't{x}') for x in range(2)]
        self.turn[0].arrive()
        self.kslot = [None] * KSL  # step id held (landed) or ('loading', g)
        self.vslot = [None] * VSL
        self.kreaders = [set() for _ in range(KSL)]  # in-flight MMAs reading the slot
        self.vreaders = [set() for _ in range(VSL)]
        self.qbuf = [None, None]  # tile index of x whose rows Q_x holds, or ('loading', n)
        self.qreaders = [set(), set()]
        self.swriters = [set(), set()]  # Q K^T MMAs of x in flight (they write S_x)
        self.owriters = [set(), set()]  # P V MMAs of x in flight (they write O_x)
        self.s_reading = [False, False]  # the softmax of x reads S_x / writes P
        self.o_reading = [False, False]  # the epilogue of x reads O_x
        self.mma_tail = [0, 0]  # completion time of the last MMA per issuer
        self.pipe_free = 0
        self.order = []

    def at(self, dt, fn):
        self.seq += 1
        self.events.append((self.t + dt, self.seq, fn))

    # MMA issue: runs on the shared pipe, completes later; returns completion time
    def mma(self, x, reads, writes=()):
        start = max(self.t, self.pipe_free)
        done = start + self.rng.randint(*self.mma_lat)
        self.pipe_free = done
        self.mma_tail[x] = max(self.mma_tail[x], done)
        for (kind, s, g) in reads:
            rs = {'k': self.kreaders, 'v': self.vreaders, 'q': self.qreaders}[kind][s]
            slot = {'k': self.kslot, 'v': self.vslot, 'q': self.qbuf}[kind]
            assert slot[s] == g, f'issuer {x} reads {kind} slot {s} for step {g} but it holds {slot[s]}'
            tok = (x, g, self.seq)
            rs.add(tok)
            self.seq += 1
            self.events.append((done, self.seq, lambda rs=rs, tok=tok: rs.discard(tok)))
        for kind in writes:
            if kind == 's':
                assert not self.s_reading[x], f'Q K^T of tile {x} writes S while its softmax reads it'
            else:
                assert not self.o_reading[x], f'P V of tile {x} writes O while its epilogue reads it'
            ws = self.swriters[x] if kind == 's' else self.owriters[x]
            tok = (x, kind, self.seq)
            ws.add(tok)
            self.seq += 1
            self.events.append((done, self.seq, lambda ws=ws, tok=tok: ws.discard(tok)))

    def commit(self, x, bar):
        self.seq += 1
        self.events.append((max(self.t, self.mma_tail[x]) + self.rng.randint(1, 10), self.seq, bar.arrive))

    def run(self, procs, limit=10 ** 6):
        # procs: generators yielding ('wait', bar, parity) or ('delay', n)
        waiting = []
        for p in procs:
            waiting.append((p, None))
        active = [[p, None] for p in procs]
        steps = 0
        while True:
            progressed = False
            self.rng.shuffle(active)
            for st in active:
                p, cond = st
                if p is None:
                    continue
                while True:
                    if cond is not None:
                        kind = cond[0]
                        if kind == 'wait':
                            if not cond[1].ready(cond[2]):
                                break
                        elif kind == 'until':
                            if self.t < cond[1]:
                                break
                    try:
                        cond = next(p)
                        progressed = True
                        if cond[0] == 'delay':
                            cond = ('until', self.t + cond[1])
                    except StopIteration:
                        st[0] = None
                        cond = None
                        break
                    st[1] = cond
                    if self.rng.random() < 0.3:
                        break
                st[1] = cond
            if all(st[0] is None for st in active):
                return True
            # advance time to the next event
            if self.events:
                self.events.sort()
                tmin = self.events[0][0]
                if not progressed or self.rng.random() < 0.5:
                    self.t = max(self.t, tmin)
                    while self.events and self.events[0][0] <= self.t:
                        _, _, fn = self.events.pop(0)
                        fn()
                else:
                    self.t += 1
            else:
                if not progressed:
                    pending = [(st[1]) for st in active if st[0] is not None]
                    if all(c[0] == 'wait' for c in pending):
                        raise RuntimeError(f'deadlock at t={self.t}: {[(c[1].name, c[2]) for c in pending]}')
                self.t += 1
            steps += 1
            if steps > limit:
                raise RuntimeError('step limit')


def producer(sim, skip_q_empty=False, no_land_wait=False):
    """K/V loads (K one step ahead of V) and, after each pair's first K load, the Q rows of its
    tiles: wait for the previous tile of the same X to finish its Q K^T (q_empty), gather, wait
    for the rows to land, signal q_full. The flags plant mistakes: gathering without the q_empty
    wait, and signalling q_full without waiting for the rows."""
    gk = gv = 0
    nq = [0, 0]
    landed = {}

    def load(is_v, g):
        n = VSL if is_v else KSL
        s = g % n
        empty = sim.v_empty[s] if is_v else sim.k_empty[s]
        full = sim.v_full[s] if is_v else sim.k_full[s]
        yield ('wait', empty, ((g // n) & 1) ^ 1)
        rs = sim.vreaders[s] if is_v else sim.kreaders[s]
        assert not rs, f'producer overwrites {"v" if is_v else "k"} slot {s} (step {g}) while read by {rs}'
        slot = sim.vslot if is_v else sim.kslot
        slot[s] = ('loading', g)
        def land(slot=slot, s=s, g=g, full=full):
            slot[s] = g
            full.arrive()
        sim.at(sim.rng.randint(10, 60), land)

    def gather(x):
        n = nq[x]
        if not skip_q_empty:
            yield ('wait', sim.q_empty[x], (n & 1) ^ 1)
        assert not sim.qreaders[x], f'rows of tile {n} of {x} gathered while an MMA reads Q: {sim.qreaders[x]}'
        sim.qbuf[x] = ('loading', n)
        landed[(x, n)] = False

        def land(x=x, n=n):
            sim.qbuf[x] = n
            landed[(x, n)] = True
        sim.at(sim.rng.randint(5, 80), land)
        while not landed[(x, n)] and not no_land_wait:
            yield ('delay', 1)
        sim.q_full[x].arrive()
        nq[x] += 1

    for (ns, n0, n1) in sim.pairs:
        yield from load(False, gk); gk += 1
        for x, nx in ((0, n0), (1, n1)):
            if nx > 0:
                yield from gather(x)
        for i in range(ns):
            if i + 1 < ns:
                yield from load(False, gk); gk += 1
            yield from load(True, gv); gv += 1


def issuer(sim, x):
    gk = gv = px = tx = 0
    it = 0
    for (ns, n0, n1) in sim.pairs:
        nx = n1 if x else n0
        if nx > 0:
            yield ('wait', sim.q_full[x], tx & 1)
        for i in range(ns + 1):
            do_qk, do_pv = i < ns, i > 0
            my_qk, my_pv = do_qk and i < nx, do_pv and i - 1 < nx
            ks, vs = gk % KSL, gv % VSL
            if do_pv:
                yield ('wait', sim.v_full[vs], (gv // VSL) & 1)
            if do_qk:
                yield ('wait', sim.k_full[ks], (gk // KSL) & 1)
            if my_pv:
                yield ('wait', sim.p_full[x], px & 1)
                if i == 1:
                    yield ('wait', sim.o_empty[x], (tx & 1) ^ 1)
            yield ('wait', sim.turn[x], it & 1)
            sim.order.append((x, it))
            if my_pv:
                sim.mma(x, [('v', vs, gv)], writes=('o',))
                px += 1
                if i == nx:
                    sim.commit(x, sim.o_full[x]); tx += 1
            if my_qk:
                sim.mma(x, [('k', ks, gk), ('q', x, tx)], writes=('s',))
                sim.commit(x, sim.s_full[x])
                if i + 1 == nx:
                    sim.commit(x, sim.q_empty[x])
            sim.turn[1 - x].arrive()
            it += 1
            if do_qk:
                if my_qk: sim.commit(x, sim.k_empty[ks])
                else: sim.k_empty[ks].arrive()
                gk += 1
            if do_pv:
                if my_pv: sim.commit(x, sim.v_empty[vs])
                else: sim.v_empty[vs].arrive()
                gv += 1
            yield ('delay', sim.rng.randint(0, 3))


def softmax(sim, x):
    """The softmax group of tile x: per step wait for S, read it and write P (the S window),
    signal p_full; per tile wait for O, read it (the O window), signal o_empty."""
    g = 0
    tile = 0
    for (ns, n0, n1) in sim.pairs:
        nx = n1 if x else n0
        if nx == 0:
            continue
        for i in range(nx):
            yield ('wait', sim.s_full[x], (g + i) & 1)
            assert not sim.swriters[x], f'softmax of {x} reads S while a Q K^T writes it'
            sim.s_reading[x] = True
            yield ('delay', sim.rng.randint(5, 40))
            sim.s_reading[x] = False
            sim.p_full[x].arrive()
        yield ('wait', sim.o_full[x], tile & 1)
        assert not sim.owriters[x], f'epilogue of {x} reads O while a P V writes it'
        sim.o_reading[x] = True
        yield ('delay', sim.rng.randint(1, 30))
        sim.o_reading[x] = False
        sim.o_empty[x].arrive()
        g += nx
        tile += 1


def _run_trials(n, issuer_fn=None, mma_lat=(5, 30), **producer_kw):
    failures = []
    for seed in range(n):
        try:
            trial_with(seed, issuer_fn or issuer, mma_lat, **producer_kw)
        except (AssertionError, RuntimeError) as e:
            failures.append((seed, str(e)))
    return failures


def trial_with(seed, issuer_fn, mma_lat=(5, 30), **producer_kw):
    rng = random.Random(seed)
    pairs = []
    for _ in range(rng.randint(1, 6)):
        kind = rng.random()
        if kind < 0.4:
            ns = rng.randint(1, 6); pairs.append((ns, ns, ns))
        elif kind < 0.6:
            ns = rng.randint(1, 6); pairs.append((ns, ns, 0))
        else:
            m = rng.randint(0, 3); pairs.append((2 * m + 2, 2 * m + 1, 2 * m + 2))
    sim = Sim(pairs, seed, mma_lat)
    sim.run([producer(sim, **producer_kw), issuer_fn(sim, 0), issuer_fn(sim, 1), softmax(sim, 0),
             softmax(sim, 1)])
    if issuer_fn is issuer:
        exp = [(x, it) for it in range(len(sim.order) // 2) for x in (0, 1)]
        assert sim.order == exp, 'issue order does not alternate'


def issuer_early_release(sim, x):
    """The protocol bug found during development, in the form it had then (issuers not yet
    alternating through turns): an issuer with no work in a step released that step's K/V slot
    without waiting for the slot to be filled, so its arrival could complete the slot's previous
    phase while the other issuer still read it."""
    gk = gv = px = tx = 0
    it = 0
    for (ns, n0, n1) in sim.pairs:
        nx = n1 if x else n0
        if nx > 0:
            yield ('wait', sim.q_full[x], tx & 1)
        for i in range(ns + 1):
            do_qk, do_pv = i < ns, i > 0
            my_qk, my_pv = do_qk and i < nx, do_pv and i - 1 < nx
            ks, vs = gk % KSL, gv % VSL
            if my_pv:
                yield ('wait', sim.v_full[vs], (gv // VSL) & 1)
            if my_qk:
                yield ('wait', sim.k_full[ks], (gk // KSL) & 1)
            if my_pv:
                yield ('wait', sim.p_full[x], px & 1)
                if i == 1:
                    yield ('wait', sim.o_empty[x], (tx & 1) ^ 1)
            if my_pv:
                sim.mma(x, [('v', vs, gv)], writes=('o',))
                px += 1
                if i == nx:
                    sim.commit(x, sim.o_full[x]); tx += 1
            if my_qk:
                sim.mma(x, [('k', ks, gk), ('q', x, tx)], writes=('s',))
                sim.commit(x, sim.s_full[x])
                if i + 1 == nx:
                    sim.commit(x, sim.q_empty[x])
            if do_qk:
                if my_qk: sim.commit(x, sim.k_empty[ks])
                else: sim.k_empty[ks].arrive()
                gk += 1
            if do_pv:
                if my_pv: sim.commit(x, sim.v_empty[vs])
                else: sim.v_empty[vs].arrive()
                gv += 1
            yield ('delay', sim.rng.randint(0, 3))


def test_attention_barrier_protocol_is_race_free():
    assert _run_trials(300) == []
    assert _run_trials(300, mma_lat=(5, 400)) == []  # MMAs completing long after their issue


def test_model_catches_the_early_slot_release_bug():
    assert len(_run_trials(300, issuer_early_release)) > 30


def test_model_catches_a_gather_without_the_q_empty_wait():
    """Rows of the next tile gathered before the previous tile's last Q K^T is known complete
    overwrite Q_x under that MMA (or let it read the wrong rows)."""
    assert len(_run_trials(300, skip_q_empty=True, mma_lat=(5, 400))) > 10


def test_model_catches_q_full_before_the_rows_land():
    """q_full signalled without waiting for the requested rows (no cp.async wait) lets the
    tile's first Q K^T read a buffer still being filled."""
    assert len(_run_trials(300, no_land_wait=True)) > 10
