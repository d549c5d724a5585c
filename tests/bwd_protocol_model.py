"""CPU model of the backward kernels' mbarrier protocol, for one CTA.

TEST INFRASTRUCTURE: it restates, role by role, the waits, arrivals and
tensor-core commits of the producer, the MMA thread and the compute warps of
the sm_100a backward kernels (fa_bwd_sm100.cuh: the dK/dV kernel, KV = True,
and the dQ kernel, KV = False), with the same ring slots (three for the A
stream, two for the B stream) and the same TMEM regions (one S region, one or
two dP regions).  It holds no attention arithmetic.

Barriers follow the hardware's parity semantics (a wait for parity p passes
iff completed phases & 1 != p).  TMA loads complete after random delays; the
tensor core runs one thread's MMAs in issue order, each for a random time,
reading its operands when it starts and writing its result when it ends; a
commit arrives once every MMA issued before it has ended.  Every stored
operand carries the step that wrote it, so a run reports:
  - deadlock (every role waiting, nothing in flight),
  - any wait issued while its barrier was not exactly one phase short,
  - an MMA or a compute warp reading an operand of the wrong step (a ring slot
    reloaded, or a TMEM region overwritten, before its last reader),
  - a TMA load into a slot an MMA has not finished reading."""
import random

from protocol_model import Bar

A_SLOTS, B_SLOTS = 3, 2


class BwdSim:
    def __init__(s, count, kv, dp_bufs, seed, warps=4, skip_sread=False, early_a_empty=False,
                 shared_full=False, skip_res_empty=False):
        # skip_sread / early_a_empty / shared_full: deliberately broken
        # protocols (the next S issued without waiting for this step's S to be
        # read; the A slot released before dK / dQ read it; one P_FULL and one
        # DS_FULL barrier for all steps instead of one per step parity), for
        # the model's own negative tests
        # count: blocks of the one unit, or a list of the units' block counts
        # (a persistent CTA takes several units in turn)
        s.units = list(count) if isinstance(count, (list, tuple)) else [count]
        s.kv, s.dp_bufs, s.warps = kv, dp_bufs, warps
        s.skip_res_empty = skip_res_empty
        s.skip_sread, s.early_a_empty, s.shared_full = skip_sread, early_a_empty, shared_full
        s.rng = random.Random(seed)
        s.b = {}
        for n in ['RES', 'RESE', 'SD', 'DONE']: s.b[n] = Bar(n, 1)
        # P / dS written: one barrier per step parity (a warp can run one step
        # ahead of another once the next step's S and dP are in)
        for n in ['SREAD', 'PFULL0', 'PFULL1', 'DSFULL0', 'DSFULL1']: s.b[n] = Bar(n, warps)
        for i in range(A_SLOTS): s.b[f'AF{i}'] = Bar(f'AF{i}', 1); s.b[f'AE{i}'] = Bar(f'AE{i}', 1)
        for i in range(B_SLOTS): s.b[f'BF{i}'] = Bar(f'BF{i}', 1); s.b[f'BE{i}'] = Bar(f'BE{i}', 1)
        s.events, s.now = [], 0
        s.errors = []
        # contents: ring slots ('A', i) / ('B', i) -> step; TMEM regions
        # 'S', 'DP0', 'DP1' -> (what, step); packed halves per warp
        s.mem = {}
        s.reading = {}   # ring slot -> number of MMAs still to read it
        s.pipe_end = 0   # tensor pipe: end time of the last issued MMA
        s.waits = {}

    # ------------------------------------------------------------ helpers
    def later(s, dt, fn): s.events.append((s.now + dt, fn))

    def wait(s, bar, par, who):
        B = s.b[bar]
        if (B.c & 1) != par:
            return
        s.waits[who] = bar
        while (B.c & 1) == par:
            yield ('wait', bar)

    def phase_check(s, bar, phase_idx, who):
        if s.b[bar].c < phase_idx:
            s.errors.append(('parity misread risk', who, bar, phase_idx, s.b[bar].c))

    def tma(s, slot_key, full, step):
        if s.reading.get(slot_key, 0):
            s.errors.append(('slot reloaded while an MMA reads it', slot_key, step))
        s.b[full].expect(1)

        def land():
            s.mem[slot_key] = step
            s.b[full].tx_done(1)
        s.later(s.rng.randint(1, 40), land)

    def expect(s, key, want, who):
        got = s.mem.get(key)
        if got != want:
            s.errors.append(('wrong operand', who, key, got, want))

    def mma(s, name, reads, writes):
        """One MMA group in the in-order pipe.  reads: [(key, expected)];
        writes: [(key, value)]."""
        start = max(s.now, s.pipe_end) + 1
        dur = s.rng.randint(1, 12)
        s.pipe_end = start + dur
        for key, _ in reads:
            if isinstance(key, tuple): s.reading[key] = s.reading.get(key, 0) + 1

        def begin():
            for key, want in reads: s.expect(key, want, name)

        def end():
            for key, _ in reads:
                if isinstance(key, tuple): s.reading[key] -= 1
            for key, val in writes: s.mem[key] = val
        s.events.append((start, begin))
        s.events.append((s.pipe_end, end))

    def commit(s, bar):
        s.events.append((max(s.now, s.pipe_end) + 1, lambda: s.b[bar].arrive()))

    def dp(s, it): return 'DP1' if s.dp_bufs == 2 and (it & 1) else 'DP0'

    def full(s, name, it):
        """(barrier, phase index) of P_FULL / DS_FULL for step it."""
        if s.shared_full: return name + '0', it
        return f'{name}{it & 1}', it >> 1

    # -------------------------------------------------------------- roles
    def producer(s):
        g = 0
        for k, count in enumerate(s.units):
            # the resident pair of unit k, once unit k-1's S and dP products
            # (its only readers) have ended
            if k > 0 and not s.skip_res_empty:
                s.phase_check('RESE', k - 1, 'prod')
                yield from s.wait('RESE', (k - 1) & 1, 'prod')
            s.b['RES'].expect(1)

            def land(k=k):
                s.mem['RA'] = k; s.mem['RB'] = k
                s.b['RES'].tx_done(1)
            s.later(s.rng.randint(1, 40), land)
            for it in range(count):
                gs = g + it
                for ring, slots in (('A', A_SLOTS), ('B', B_SLOTS)):
                    slot, use = gs % slots, gs // slots
                    if use > 0:
                        e = f'{ring}E{slot}'
                        s.phase_check(e, use - 1, 'prod')
                        yield from s.wait(e, (use - 1) & 1, 'prod')
                    s.tma((ring, slot), f'{ring}F{slot}', gs)
            g += count
        yield ('done',)

    def mma_thread(s):
        kv = s.kv

        def wait_ring(gs, ring):
            slots = A_SLOTS if ring == 'A' else B_SLOTS
            s.phase_check(f'{ring}F{gs % slots}', gs // slots, 'mma')
            yield from s.wait(f'{ring}F{gs % slots}', (gs // slots) & 1, 'mma')

        def issue_s(gs, k):
            s.mma(f'S({gs})', [(('A', gs % A_SLOTS), gs), ('RA', k)], [('S', ('S', gs))])

        def issue_dp(gs, k):
            s.mma(f'dP({gs})', [(('B', gs % B_SLOTS), gs), ('RB', k)], [(s.dp(gs), ('dP', gs))])
            s.commit('SD')
            if not kv: s.commit(f'BE{gs % B_SLOTS}')

        g = 0
        for k, count in enumerate(s.units):
            s.phase_check('RES', k, 'mma')
            yield from s.wait('RES', k & 1, 'mma')
            # (the previous unit's last S was read out before its last dK / dQ,
            # which waited for every warp's dS of that step)
            yield from wait_ring(g, 'A'); issue_s(g, k)
            yield from wait_ring(g, 'B'); issue_dp(g, k)
            if count == 1: s.commit('RESE')
            for it in range(count):
                gs = g + it
                more = it + 1 < count
                if more:
                    yield from wait_ring(gs + 1, 'A')
                    if not s.skip_sread:
                        s.phase_check('SREAD', gs, 'mma')
                        yield from s.wait('SREAD', gs & 1, 'mma')
                    issue_s(gs + 1, k)
                    if s.dp_bufs == 2:
                        yield from wait_ring(gs + 1, 'B'); issue_dp(gs + 1, k)
                        if it + 2 == count: s.commit('RESE')
                if kv:
                    bar, ph = s.full('PFULL', gs)
                    s.phase_check(bar, ph, 'mma')
                    yield from s.wait(bar, ph & 1, 'mma')
                    s.mma(f'dV({gs})', [(('B', gs % B_SLOTS), gs)] +
                          [((s.dp(gs), 'P', w), gs) for w in range(s.warps)], [('ACC', ('ACC', k))])
                    s.commit(f'BE{gs % B_SLOTS}')
                if s.early_a_empty: s.commit(f'AE{gs % A_SLOTS}')
                bar, ph = s.full('DSFULL', gs)
                s.phase_check(bar, ph, 'mma')
                yield from s.wait(bar, ph & 1, 'mma')
                s.mma(f'dK({gs})', [(('A', gs % A_SLOTS), gs)] +
                      [((s.dp(gs), 'dS', w), gs) for w in range(s.warps)], [('ACC', ('ACC', k))])
                if not s.early_a_empty: s.commit(f'AE{gs % A_SLOTS}')
                if more and s.dp_bufs == 1:
                    yield from wait_ring(gs + 1, 'B'); issue_dp(gs + 1, k)
                    if it + 2 == count: s.commit('RESE')
                yield ('work',)
            s.commit('DONE')
            g += count
        yield ('done',)

    def compute(s, w):
        g = 0
        for k, count in enumerate(s.units):
            for it in range(count):
                gs = g + it
                s.phase_check('SD', gs, f'c{w}')
                yield from s.wait('SD', gs & 1, f'c{w}')
                # the warps reach their loads at different times
                for _ in range(s.rng.randint(0, 20)): yield ('work',)
                # loads of S and of this step's dP region
                s.expect('S', ('S', gs), f'c{w} load S')
                r = s.dp(gs)
                s.expect(r, ('dP', gs), f'c{w} load dP')
                yield ('work',)
                s.b['SREAD'].arrive()
                for _ in range(s.rng.randint(0, 20)): yield ('work',)
                # packed tiles over this warp's own dP columns: a write of the
                # region by an MMA would clobber them, so track them per warp
                if s.kv:
                    s.mem[(r, 'P', w)] = gs
                    s.b[s.full('PFULL', gs)[0]].arrive()
                    yield ('work',)
                s.mem[(r, 'dS', w)] = gs
                s.b[s.full('DSFULL', gs)[0]].arrive()
            s.phase_check('DONE', k, f'c{w}')
            yield from s.wait('DONE', k & 1, f'c{w}')
            # epilogue: read the accumulators.  The next unit's first
            # accumulating product waits for this warp's P / dS of that unit,
            # written after this read, so no other hand-back is needed.
            for _ in range(s.rng.randint(0, 20)): yield ('work',)
            s.expect('ACC', ('ACC', k), f'c{w} epilogue')
            g += count
        yield ('done',)

    def run(s, max_steps=400000):
        # an MMA result over a dP region also overwrites the packed tiles in it
        orig = s.mma

        def mma(name, reads, writes):
            more = []
            for key, _ in writes:
                if key in ('DP0', 'DP1'):
                    for w in range(s.warps):
                        more += [((key, 'P', w), None), ((key, 'dS', w), None)]
            orig(name, reads, writes + more)
        s.mma = mma
        roles = {'prod': s.producer(), 'mma': s.mma_thread()}
        for w in range(s.warps): roles[f'c{w}'] = s.compute(w)
        done, steps = set(), 0
        state = {k: None for k in roles}
        while len(done) < len(roles):
            steps += 1
            if steps > max_steps: return 'steps'
            progressed = False
            for k in s.rng.sample(list(roles), len(roles)):
                if k in done: continue
                try:
                    st = next(roles[k])
                except StopIteration:
                    done.add(k); progressed = True; continue
                except AssertionError as e:
                    return ('overflow', str(e))
                if st[0] == 'done': done.add(k); progressed = True
                elif st[0] == 'wait':
                    key = (st[1], s.b[st[1]].c, s.b[st[1]].pending)
                    if state[k] != key: progressed = True
                    state[k] = key
                else:
                    progressed = True; state[k] = None
            s.events.sort(key=lambda e: e[0])
            fired = False
            while s.events and s.events[0][0] <= s.now:
                _, fn = s.events.pop(0)
                try:
                    fn()
                except AssertionError as e:
                    return ('overflow', str(e))
                fired = True
            s.now += 1
            if not s.events and not fired and not progressed:
                return ('deadlock', {k: state[k] for k in roles if k not in done})
        return 'ok'
