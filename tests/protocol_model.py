"""Discrete-event model of the barrier protocol of the persistent attention kernel.

TEST INFRASTRUCTURE.  The kernel in recurrent_depth_lm_b200/csrc/attn.cu keeps two
query-tile slots per CTA.  A producer warp writes work entries (up to 4 key blocks,
or an end marker) into a ring per slot and loads Q and K with TMA; a V producer,
the single MMA issuer and each slot's softmax warpgroup read the rings in the same
order (alternate slots, skip a slot after its end marker).  K and V stages are
rings filled in that global order.  Every hand-off is an mbarrier.

Each role here is a generator that follows the kernel's sequence of arrivals and
waits.  Waits use the hardware's parity semantics (try_wait.parity(i & 1) passes
while the barrier's current phase has the other parity), so a wait that passes a
phase early or late is an error.  TMA copies land after random delays; an MMA may
read or write its operands at any moment between its issue and its completion, but
not before an MMA issued earlier has touched its own (tcgen05 MMAs of one thread
execute in issue order; ``mma_in_order=False`` drops that), and a commit arrives
when every earlier MMA has completed.  The model flags:
a buffer (Q, K stage, V stage, S/P, O) overwritten while a reader still needs it,
an MMA or the softmax reading the wrong generation of a buffer, an early or late
phase, a deadlock, and a tile whose output misses entries.

``drop`` names barriers whose waits are skipped, to check that the model catches
the hazard each wait prevents.
"""
import random

class Bar:
    def __init__(self, name, count):
        self.name, self.count = name, count
        self.pending = count
        self.tx = 0
        self.phase = 0          # completed phases
    def arrive(self, n=1):
        self.pending -= n
        assert self.pending >= 0, f"{self.name}: too many arrivals"
        self._maybe()
    def expect_tx(self, b):
        self.tx += b
    def complete_tx(self, b):
        self.tx -= b
        assert self.tx >= 0
        self._maybe()
    def _maybe(self):
        if self.pending == 0 and self.tx == 0:
            self.phase += 1
            self.pending = self.count

class Sim:
    def __init__(self, seed, tiles_per_cta_list, mode, NK, NV, R=4, drop=(), mma_in_order=True):
        self.drop = frozenset(drop)
        self.mma_in_order = mma_in_order
        self.last_effect = 0
        self.rng = random.Random(seed)
        self.mode = mode  # 'attn' or 'mass'
        self.attn = mode == 'attn'
        self.NK, self.NV, self.R = NK, NV, R
        self.t = 0
        self.events = []   # (time, seq, fn)
        self.seq = 0
        self.tiles = tiles_per_cta_list  # list of (tile_id, n_entries, [ns per entry])
        B = {}
        def mk(n, c): B[n] = Bar(n, c)
        for x in range(2):
            mk(('q_full', x), 1); mk(('q_empty', x), 1)
            for k in range(R):
                mk(('e_full', x, k), 1); mk(('e_empty', x, k), 128 + 1 + (1 if self.attn else 0))
            mk(('s_full', x), 1); mk(('s_free', x), 128); mk(('p_full', x), 128)
            mk(('o_done', x), 1); mk(('o_free', x), 128)
        for s in range(NK):
            mk(('k_full', s), 1); mk(('k_empty', s), 1)
        for s in range(max(NV, 1)):
            mk(('v_full', s), 1); mk(('v_empty', s), 1)
        mk('final', 1)
        self.B = B
        self.ents = {}      # (x,k) -> dict
        # data state
        self.Q = [None, None]
        self.Kst = {}       # stage -> g
        self.Vst = {}
        self.S = [None, None]   # ('S', g) or ('P', g)
        self.O = [None, None]   # ('acc', tile, upto_g) ...
        self.mma_queue = []     # in-order ops: dicts
        self.mma_busy_until = 0
        self.inflight = []      # issued, not yet completed ops
        self.done_ops = set()
        self.log = []
        self.out = {}           # tile -> list of g used
        self.errors = []

    # ------------------------------------------------------------ scheduling
    def at(self, dt, fn):
        self.seq += 1
        self.events.append((self.t + dt, self.seq, fn))

    def wait(self, bar, idx):
        """yield-able wait object: intended phase index idx (0-based)"""
        return ('wait', bar, idx)

    # MMA engine: ops complete in order; an op's effects (reads/writes) are modelled
    # at random times within [issue, completion]; commits arrive at completion of all prior.
    def mma_issue(self, op):
        op['issue'] = self.t
        dur = self.rng.randint(20, 80)
        start = max(self.t, self.mma_busy_until)
        op['done'] = start + dur
        self.mma_busy_until = op['done']
        self.inflight.append(op)
        # effects at a random time in [issue, done], after the previous op's effects
        lo = max(self.t, self.last_effect) if self.mma_in_order else self.t
        te = self.rng.randint(lo, op['done'])
        self.last_effect = te
        self.seq += 1
        self.events.append((te, self.seq, lambda op=op: self.mma_effect(op)))
        self.seq += 1
        self.events.append((op['done'], self.seq, lambda op=op: self.mma_finish(op)))

    def mma_commit(self, bar):
        t_done = max(self.t, self.mma_busy_until)
        self.seq += 1
        self.events.append((t_done, self.seq, lambda: self.B[bar].arrive()))

    def mma_effect(self, op):
        k = op['kind']
        x = op['x']
        if k == 'QK':
            g = op['g']
            if self.Kst.get(g % self.NK) != g:
                self.errors.append(f"QK g={g} reads K stage holding {self.Kst.get(g % self.NK)}")
            if self.Q[x] != op['tile']:
                self.errors.append(f"QK g={g} reads Q[{x}]={self.Q[x]} want {op['tile']}")
            # S_X must not hold a P still needed
            cur = self.S[x]
            if cur is not None and cur[0] == 'P' and cur[1] not in self.pv_read:
                self.errors.append(f"QK g={g} overwrites P of g={cur[1]} before its PV read it")
            if cur is not None and cur[0] == 'S' and cur[1] not in self.s_read:
                self.errors.append(f"QK g={g} overwrites S of g={cur[1]} before it was read")
            self.S[x] = ('S', g)
        elif k == 'PV':
            g = op['g']
            if self.Vst.get(g % self.NV) != g:
                self.errors.append(f"PV g={g} reads V stage holding {self.Vst.get(g % self.NV)}")
            if self.S[x] != ('P', g):
                self.errors.append(f"PV g={g} reads S[{x}]={self.S[x]}")
            self.pv_read.add(g)
            if op['first']:
                if self.O[x] is not None and self.O[x][0] != 'read':
                    self.errors.append(f"PV g={g} (first) overwrites unread O[{x}]={self.O[x]}")
                self.O[x] = ('acc', op['tile'], [g])
            else:
                if self.O[x] is None or self.O[x][0] != 'acc' or self.O[x][1] != op['tile']:
                    self.errors.append(f"PV g={g} accumulates into O[{x}]={self.O[x]}")
                else:
                    self.O[x][2].append(g)

    def mma_finish(self, op):
        if op['kind'] == 'PV':
            self.pv_done.add(op['g'])
        if op['kind'] == 'QK':
            self.qk_done.add(op['g'])
        self.inflight.remove(op)

    def tma(self, bar, nbytes, fn):
        self.B[bar].expect_tx(nbytes)
        self.B[bar].arrive()
        dt = self.rng.randint(5, 120)
        def land():
            fn()
            self.B[bar].complete_tx(nbytes)
        self.at(dt, land)

    # ------------------------------------------------------------ roles
    def producer(self):
        R, NK = self.R, self.NK
        S = [dict(rc=0, tq=0, active=False, ended=False, first=False, ents=[], tile=None) for _ in range(2)]
        g = 0
        next_k = 0
        def step(x):
            nonlocal g, next_k
            st = S[x]
            k = st['rc'] % R
            if st['rc'] >= R:
                yield self.wait(('e_empty', x, k), st['rc'] // R - 1)
            # WAR check: all consumers read the old entry
            if not st['active']:
                if next_k >= len(self.tiles):
                    self.ents[(x, k)] = dict(kind='end')
                    self.B[('e_full', x, k)].arrive()
                    st['rc'] += 1; st['ended'] = True
                    return
                tile, ns_list = self.tiles[next_k]; next_k += 1
                if st['tq'] >= 1:
                    yield self.wait(('q_empty', x), st['tq'] - 1)
                # Q WAR: previous tile's QKs all completed
                prev = st['tile']
                if prev is not None:
                    for gg in self.tile_gs.get(prev, []):
                        if gg not in self.qk_done:
                            self.errors.append(f"Q[{x}] reload while QK g={gg} of tile {prev} pending")
                self.tma(('q_full', x), 1, lambda x=x, tile=tile: self.Q.__setitem__(x, tile))
                st['tq'] += 1; st['active'] = True; st['first'] = True; st['tile'] = tile
                st['ents'] = list(ns_list)
                self.tile_gs[tile] = []
            ns = st['ents'].pop(0)
            last = len(st['ents']) == 0
            ks = g % NK
            if g >= NK:
                yield self.wait(('k_empty', ks), g // NK - 1)
            old = self.Kst.get(ks)
            if old is not None and old not in self.qk_done:
                self.errors.append(f"K stage {ks} overwritten (g={g}) while QK g={old} pending")
            self.ents[(x, k)] = dict(kind='work', first=st['first'], last=last, ns=ns,
                                     tile=st['tile'], stage=g)
            self.tile_gs[st['tile']].append(g)
            self.B[('e_full', x, k)].arrive()
            self.tma(('k_full', ks), ns, lambda ks=ks, g=g: self.Kst.__setitem__(ks, g))
            st['rc'] += 1; g += 1; st['first'] = False
            if last: st['active'] = False
        while not (S[0]['ended'] and S[1]['ended']):
            if not S[0]['ended']:
                yield from step(0)
            if not S[1]['ended']:
                yield from step(1)

    def vproducer(self):
        if not self.attn:
            return
        R, NV = self.R, self.NV
        S = [dict(rc=0, ended=False) for _ in range(2)]
        def step(x):
            st = S[x]
            k = st['rc'] % R
            yield self.wait(('e_full', x, k), st['rc'] // R)
            e = dict(self.ents[(x, k)])
            self.B[('e_empty', x, k)].arrive()
            st['rc'] += 1
            if e['kind'] == 'end':
                st['ended'] = True; return
            g = e['stage']; vs = g % NV
            if g >= NV:
                yield self.wait(('v_empty', vs), g // NV - 1)
            old = self.Vst.get(vs)
            if old is not None and old not in self.pv_done:
                self.errors.append(f"V stage {vs} overwritten (g={g}) while PV g={old} pending")
            self.tma(('v_full', vs), e['ns'], lambda vs=vs, g=g: self.Vst.__setitem__(vs, g))
        while not (S[0]['ended'] and S[1]['ended']):
            if not S[0]['ended']:
                yield from step(0)
            if not S[1]['ended']:
                yield from step(1)

    def issuer(self):
        R, NK, NV = self.R, self.NK, self.NV
        S = [dict(rc=0, ended=False, pend=None, pvc=0, qkc=0, qtiles=0, otiles=0) for _ in range(2)]
        def issue_pv(x):
            st = S[x]
            pe = st['pend']
            yield self.wait(('p_full', x), st['pvc'])
            if pe['first']:
                if st['otiles'] >= 1:
                    yield self.wait(('o_free', x), st['otiles'] - 1)
                st['otiles'] += 1
            g = pe['stage']; vs = g % NV
            self.mma_issue(dict(kind='PV', x=x, g=g, first=pe['first'], tile=pe['tile']))
            self.mma_commit(('o_done', x))
            self.mma_commit(('v_empty', vs))
            st['pvc'] += 1
            st['pend'] = None
        def step(x):
            st = S[x]
            k = st['rc'] % R
            yield self.wait(('e_full', x, k), st['rc'] // R)
            e = dict(self.ents[(x, k)])
            self.B[('e_empty', x, k)].arrive()
            st['rc'] += 1
            if self.attn and st['pend'] is not None:
                pg = st['pend']['stage']
                yield self.wait(('v_full', pg % NV), pg // NV)
            if e['kind'] != 'end':
                g = e['stage']; ks = g % NK
                yield self.wait(('k_full', ks), g // NK)
                if e['first']:
                    yield self.wait(('q_full', x), st['qtiles'])
                    st['qtiles'] += 1
            if self.attn and st['pend'] is not None:
                yield from issue_pv(x)
            if e['kind'] == 'end':
                st['ended'] = True; return
            # attention: S_X holds the P that the PV just issued reads; in-order MMA
            # execution lets this QK follow it without a wait
            if st['qkc'] >= 1 and not self.attn:
                yield self.wait(('s_free', x), st['qkc'] - 1)
            self.mma_issue(dict(kind='QK', x=x, g=g, tile=e['tile']))
            self.mma_commit(('s_full', x))
            self.mma_commit(('k_empty', ks))
            if e['last']:
                self.mma_commit(('q_empty', x))
            st['qkc'] += 1
            if self.attn:
                st['pend'] = e
        while not (S[0]['ended'] and S[1]['ended']):
            if not S[0]['ended']:
                yield from step(0)
            if not S[1]['ended']:
                yield from step(1)
        self.mma_commit('final')
        yield self.wait('final', 0)

    def softmax(self, x):
        R = self.R
        rc = 0
        cnt = 0
        run = True
        while run:
            first = True
            tile = None
            while True:
                k = rc % R
                yield self.wait(('e_full', x, k), rc // R)
                e = dict(self.ents[(x, k)])
                self.B[('e_empty', x, k)].arrive(128)
                rc += 1
                if e['kind'] == 'end':
                    run = False; break
                if first:
                    tile = e['tile']
                yield self.wait(('s_full', x), cnt)
                g = e['stage']
                if self.S[x] != ('S', g):
                    self.errors.append(f"softmax{x} reads S={self.S[x]} want g={g}")
                cnt += 1
                if not self.attn:
                    self.s_read.add(g)
                    self.B[('s_free', x)].arrive(128)
                    self.out.setdefault(tile, []).append(g)
                    first = False
                    if e['last']: break
                    continue
                yield ('delay', self.rng.randint(1, 60))
                if not first:
                    # rescale O: previous PV must be complete, current not yet issued
                    prev = self.tile_gs[tile][self.tile_gs[tile].index(g) - 1]
                    if prev not in self.pv_done:
                        self.errors.append(f"softmax{x} rescales O while PV g={prev} pending")
                self.S[x] = ('P', g)
                self.s_read.add(g)
                self.B[('p_full', x)].arrive(128)
                first = False
                if e['last']: break
            if not run or not self.attn:
                continue
            yield self.wait(('o_done', x), cnt - 1)
            # epilogue reads O: all PVs of the tile done
            want = self.tile_gs[tile]
            if self.O[x] is None or self.O[x][0] != 'acc' or self.O[x][1] != tile or self.O[x][2] != want:
                self.errors.append(f"epilogue{x} tile {tile}: O={self.O[x]} want {want}")
            for gg in want:
                if gg not in self.pv_done:
                    self.errors.append(f"epilogue{x} reads O while PV g={gg} pending")
            self.out[tile] = list(self.O[x][2]) if self.O[x] else None
            yield ('delay', self.rng.randint(1, 30))
            self.O[x] = ('read',)
            self.B[('o_free', x)].arrive(128)

    # ------------------------------------------------------------ driver
    def run(self):
        self.pv_done, self.qk_done, self.s_read, self.pv_read = set(), set(), set(), set()
        self.tile_gs = {}
        roles = {'prod': self.producer(), 'v': self.vproducer(), 'mma': self.issuer(),
                 'sm0': self.softmax(0), 'sm1': self.softmax(1)}
        blocked = {}
        def advance(name):
            gen = roles[name]
            while True:
                try:
                    w = next(gen)
                except StopIteration:
                    del roles[name]
                    return
                if w[0] == 'delay':
                    self.at(w[1], lambda name=name: advance(name))
                    return
                _, bar, idx = w
                if (bar[0] if isinstance(bar, tuple) else bar) in self.drop:
                    continue            # mutation: this wait is skipped
                b = self.B[bar]
                # hardware semantics: try_wait.parity(idx & 1) passes iff the current
                # (incomplete) phase has the other parity
                if (b.phase & 1) != (idx & 1):
                    if b.phase != idx + 1:
                        self.errors.append(f"{name} wait {bar} phase {idx} passed at barrier phase {b.phase} ({'early' if b.phase < idx + 1 else 'late'})")
                    continue
                blocked[name] = (bar, idx)
                return
        for name in list(roles):
            self.at(self.rng.randint(0, 5), lambda name=name: advance(name))
        steps = 0
        while True:
            # wake blocked roles whose wait is now satisfied (random order)
            progressed = False
            names = list(blocked)
            self.rng.shuffle(names)
            for name in names:
                bar, idx = blocked[name]
                b = self.B[bar]
                if (b.phase & 1) != (idx & 1):
                    if b.phase != idx + 1:
                        self.errors.append(f"{name} wait {bar} phase {idx} passed at barrier phase {b.phase}")
                    del blocked[name]
                    self.at(self.rng.randint(0, 10), lambda name=name: advance(name))
                    progressed = True
            if not self.events:
                break
            self.events.sort()
            t, _, fn = self.events.pop(0)
            self.t = t
            fn()
            steps += 1
            if steps > 2_000_000:
                self.errors.append("runaway")
                break
        if roles or blocked:
            self.errors.append(f"deadlock: blocked={blocked} live={list(roles)}")
        return self.errors


def make_tiles(rng, ntiles):
    out = []
    for t in range(ntiles):
        ne = rng.choice([1, 1, 2, 3, 5, 8])
        out.append((t, [rng.randint(1, 4) for _ in range(ne)]))
    return out


def run_seeds(seeds, drop=(), mma_in_order=True):
    """Run the model over random tile mixes; returns {seed: errors} for failing runs."""
    bad = {}
    for seed in seeds:
        rng = random.Random(seed)
        ntiles = rng.choice([0, 1, 2, 3, 4, 7, 12])
        mode = rng.choice(['attn', 'attn', 'mass'])
        NK = rng.choice([3, 4, 6]) if mode == 'mass' else rng.choice([2, 3, 4])
        NV = rng.choice([2, 4]) if mode == 'attn' else 1
        tiles = make_tiles(rng, ntiles)
        sim = Sim(seed, tiles, mode, NK, NV, drop=drop, mma_in_order=mma_in_order)
        try:
            errs = sim.run()
        except (AssertionError, IndexError, KeyError, TypeError) as exc:
            errs = [f"model invariant broken: {exc!r}"]   # e.g. a barrier over-arrived
        if not errs:
            for tile, ns in tiles:
                got = sim.out.get(tile)
                if got is None or len(got) != len(ns):
                    errs.append(f"tile {tile} output {got} want {len(ns)} entries")
        if errs:
            bad[seed] = errs
    return bad
