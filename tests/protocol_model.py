"""CPU model of the forward kernel's mbarrier protocol, for one CTA.

TEST INFRASTRUCTURE: it restates, role by role, the waits and arrivals of
the producer, the two MMA threads, the four softmax groups and the store
warp of the sm_100a forward kernel (fa_fwd_sm100.cuh), with the persistent
schedule, key-block ranges and ring positions computed the same way.  It
holds no attention arithmetic.

Barriers follow the hardware's parity semantics: a wait for parity p passes
iff (completed phases & 1) != p, so it misreads when the barrier is two
phases away.  TMA loads and tensor-core products complete after random
delays.  A run reports deadlock (every role waiting, nothing in flight), any
wait issued while the barrier was not exactly one phase short of it, and
these data hazards: O overwritten by a tile's first P V before both softmax
groups read it, a ring slot reloaded before its staged O was stored or while
an MMA still reads it, the Q buffer reloaded while an S product reads it, an
S or P V product reading a Q buffer or slot that does not hold its own Q, K
or V, a softmax group reading an S buffer that does not hold its
block's scores, a half of the shared P buffer overwritten while a P V
product still reads it, and a P V product reading a P half not written for
it."""
import random

class Bar:
    def __init__(s, name, count): s.name, s.count, s.pending, s.tx, s.c = name, count, count, 0, 0
    def arrive(s, n=1):
        s.pending -= n
        assert s.pending >= 0, f"{s.name}: too many arrivals"
        s._chk()
    def expect(s, b): s.pending -= 1; s.tx += b; assert s.pending >= 0, s.name
    def tx_done(s, b): s.tx -= b; s._chk()
    def _chk(s):
        if s.pending == 0 and s.tx == 0: s.c += 1; s.pending = s.count

BM = BN = 128
class P:  # params
    def __init__(s, N, causal, QS, KVS, left=-1, right=-1, B=1, H=1, lens=None, o_tma=True):
        s.N, s.causal, s.QS, s.KVS = N, causal, QS, KVS
        s.wl, s.wr = left, (0 if causal else right)
        if s.wl >= N: s.wl = -1
        if s.wr >= N: s.wr = -1
        s.lens = lens; s.B = len(lens) if lens else B; s.H = H; s.o_tma = o_tma
        rows = 128 * QS
        s.nq = (N + rows - 1) // rows; s.num_tiles = s.B * s.H * s.nq

def key_range(p, L, r0):
    if r0 >= L: return 0, 0
    nkv = (L + BN - 1) // BN; last = min(r0 + BM - 1, L - 1)
    lo = 0 if p.wl < 0 else max(0, r0 - p.wl) // BN
    hi = nkv if p.wr < 0 else min(L - 1, last + p.wr) // BN + 1
    return lo, hi

def decode(p, t):
    nbh = p.B * p.H
    if p.causal: qi = t // nbh; bh = t - qi * nbh; qb = p.nq - 1 - qi
    else: bh = t // p.nq; qb = t - bh * p.nq
    b = bh // p.H; q0 = qb * BM * p.QS
    L = p.lens[b] if p.lens else p.N
    lo = [0, 0]; hi = [0, 0]
    lo[0], hi[0] = key_range(p, L, q0)
    if p.QS == 2: lo[1], hi[1] = key_range(p, L, q0 + BM)
    n_u = 0 if hi[0] == 0 else max(hi[0], hi[1]) - lo[0]
    ti = dict(q0=q0, len=L, lo=lo, hi=hi, lo_u=lo[0], n_u=n_u)
    return ti

def inr(ti, s, j): return ti['lo'][s] <= j < ti['hi'][s]
def via_slot(p, ti, s):
    if not p.o_tma or ti['lo'][s] == ti['hi'][s]: return False
    return p.lens is None or ti['q0'] + (s + 1) * BM <= ti['len']
def nslots(p, ti): return sum(via_slot(p, ti, s) for s in range(2))
def ring_k(j): return 0 if j == 0 else 2 * j - 1
def ring_v(j, n): return 2 * j + 2 if j < n - 1 else 2 * n - 1
def next_user(ti, s, j):
    if s == 0 and inr(ti, 1, j): return 1
    if inr(ti, 0, j + 1): return 0
    if inr(ti, 1, j + 1): return 1
    return -1

class Sim:
    def __init__(s, p, G, cta, seed, shared_full=False, skip_pfree=False, skip_sfree=False,
                 skip_qempty=False):
        # shared_full: one full barrier per slot for K, V and O uses, waited
        # with the parity of position // ring depth (the first design).
        # skip_pfree: the softmax groups write their half of the shared P
        # buffer without waiting for its hand-over (a broken protocol, for the
        # model's own negative test).  skip_sfree: the S thread overwrites a
        # Q tile's S buffer without waiting for the softmax to have read it
        # (likewise broken).  skip_qempty: the producer loads the next work
        # tile's Q without waiting for the last S product of this one
        s.p, s.G, s.cta, s.rng = p, G, cta, random.Random(seed)
        s.shared = shared_full
        K = p.KVS
        s.b = {}
        def mk(n, c): s.b[n] = Bar(n, c)
        for n in ['QF', 'QE']: mk(n, 1)
        for i in range(K):
            mk(f'KS{i}', 1); mk(f'KV{i}', 1); mk(f'KO{i}', 1); mk(f'KE{i}', 1); mk(f'OS{i}', 8)
            mk(f'KF{i}', 1)
        for i in range(2):
            mk(f'SF{i}', 1); mk(f'SFR{i}', 8); mk(f'PFR{i}_0', 1); mk(f'PFR{i}_1', 1)
            mk(f'PVD{i}', 1); mk(f'OF{i}', 1); mk(f'X{i}', 8)
        mk('PF0', 8); mk('PF1', 4)
        s.events = []  # (time, fn)
        s.now = 0
        s.aliased = []
        s.where = {}; s.ctx = {}
        s.oread = {}; s.prev_tile = {0: None, 1: None}; s.hazards = []; s.slot_state = {}
        s.pend_mma = {}  # thread -> latest completion time
        s.skip_pfree = skip_pfree
        # the shared P buffer, by half: (tile, Q tile, block) of the P written
        # there, and the time the last P V K-steps reading it end
        s.p_tag = {0: None, 1: None}; s.p_busy = {0: 0, 1: 0}
        s.skip_sfree = skip_sfree
        # ring slots: the (tile, 'K' / 'V', block) last landed there and the
        # time its last reader ends; S buffers: the (tile, block) of the S in it
        s.slot_data = {}; s.slot_busy = {}; s.s_tag = {0: None, 1: None}
        s.skip_qempty = skip_qempty
        # the Q buffer: the work tile whose Q landed there, and the time its
        # last S product ends
        s.q_data = None; s.q_busy = 0
    def tiles(s):
        r = 0
        while r * s.G < s.p.num_tiles:
            t = r * s.G + ((s.G - 1 - s.cta) if r & 1 else s.cta)
            if t < s.p.num_tiles: yield t
            r += 1
    # async helpers
    def later(s, dt, fn): s.events.append((s.now + dt, fn))
    def tma_load(s, bar, nbytes=1):
        s.b[bar].expect(nbytes); s.later(s.rng.randint(1, 40), lambda: s.b[bar].tx_done(nbytes))
    def mma(s, th):
        s.pend_mma[th] = max(s.pend_mma.get(th, s.now), s.now) + s.rng.randint(1, 15)
        return s.pend_mma[th]
    def commit(s, th, bar):
        t = max(s.pend_mma.get(th, s.now), s.now) + 1
        s.events.append((t, lambda: s.b[bar].arrive()))
    def wait(s, bar, par, who):
        B = s.b[bar]
        s.where[who] = (bar, par, s.ctx.get(who))
        # aliasing: waiting for phase k = the one with parity par after c completed...
        while (B.c & 1) == par:
            yield ('wait', bar)
        return
    def check_alias(s, bar, phase_idx, who):
        # waiting for completion of phase phase_idx: require phase_idx-1 completed (c >= phase_idx)
        if s.b[bar].c < phase_idx:
            s.aliased.append((who, bar, phase_idx, s.b[bar].c))

    # ---------------- roles
    def producer(s):
        p, K = s.p, s.p.KVS
        kv = [0]; q_count = 0
        def load_kv(tag, ident):
            slot, use = kv[0] % K, kv[0] // K
            if use > 0:
                s.check_alias(f'KE{slot}', use - 1, 'prod')
                yield from s.wait(f'KE{slot}', (use - 1) & 1, 'prod')
            if s.slot_state.get(slot, ('',))[0] == 'O-staged': s.hazards.append(('slot reloaded before O store', slot))
            if s.now < s.slot_busy.get(slot, 0):
                s.hazards.append(('slot reloaded while an MMA reads it', slot, ident))
            s.slot_state[slot] = ('KV',)
            bar = ('KF' if s.shared else ('KS' if tag == 'K' else 'KV')) + str(slot)
            s.b[bar].expect(1)

            def land(slot=slot, ident=ident, bar=bar):
                s.slot_data[slot] = ident
                s.b[bar].tx_done(1)
            s.later(s.rng.randint(1, 40), land); kv[0] += 1
        def reserve():
            slot, use = kv[0] % K, kv[0] // K
            if use > 0:
                s.check_alias(f'KE{slot}', use - 1, 'prod')
                yield from s.wait(f'KE{slot}', (use - 1) & 1, 'prod')
            s.b[('KF' if s.shared else 'KO') + str(slot)].arrive(); kv[0] += 1
        for t in s.tiles():
            ti = decode(p, t)
            if ti['n_u'] == 0: continue
            yield from load_kv('K', (t, 'K', ti['lo_u']))
            if q_count > 0 and not s.skip_qempty:
                s.check_alias('QE', q_count - 1, 'prod')
                yield from s.wait('QE', (q_count - 1) & 1, 'prod')
            if s.now < s.q_busy:
                s.hazards.append(('Q reloaded while an S product reads it', t))
            s.b['QF'].expect(1)

            def land_q(t=t):
                s.q_data = t
                s.b['QF'].tx_done(1)
            s.later(s.rng.randint(1, 40), land_q); q_count += 1
            for jj in range(ti['n_u']):
                s.ctx['prod'] = ('tile', t, 'jj', jj, 'kv', kv[0])
                j = ti['lo_u'] + jj
                if jj + 1 < ti['n_u']: yield from load_kv('K', (t, 'K', j + 1))
                yield from load_kv('V', (t, 'V', j))
            for sx in range(p.QS):
                s.ctx['prod'] = ('tile', t, 'reserve', sx, 'kv', kv[0])
                if via_slot(p, ti, sx): yield from reserve()
        yield ('done',)

    def s_thread(s):
        p, K = s.p, s.p.KVS
        kv = 0; q_count = 0; sf = [0, 0]; issued = [0, 0]; waited = [0]; kuse = [0] * K
        def wait_kv(idx):
            sl = idx % K
            if s.shared:
                s.check_alias(f'KF{sl}', idx // K, 'S')
                yield from s.wait(f'KF{sl}', (idx // K) & 1, 'S'); return
            s.check_alias(f'KS{sl}', kuse[sl], 'S')
            yield from s.wait(f'KS{sl}', kuse[sl] & 1, 'S'); kuse[sl] += 1
        for t in s.tiles():
            ti = decode(p, t)
            if ti['n_u'] == 0: continue
            s.check_alias('QF', q_count, 'S')
            yield from s.wait('QF', q_count & 1, 'S'); q_count += 1
            kv0 = kv
            for jj in range(ti['n_u']):
                j = ti['lo_u'] + jj; k = kv0 + ring_k(jj)
                s.ctx['S'] = ('tile', t, 'jj', jj, 'k', k, 'waited', waited[0])
                yield from wait_kv(k)
                for sx in range(p.QS):
                    if inr(ti, sx, j):
                        if issued[sx] > 0 and not s.skip_sfree:
                            s.check_alias(f'SFR{sx}', issued[sx] - 1, 'S')
                            yield from s.wait(f'SFR{sx}', sf[sx], 'S'); sf[sx] ^= 1
                        if s.q_data != t:
                            s.hazards.append(('S read a Q buffer not holding its tile', s.q_data, t))
                        if s.slot_data.get(k % K) != (t, 'K', j):
                            s.hazards.append(('S read a slot not holding its K', k % K, s.slot_data.get(k % K), (t, 'K', j)))
                        end = s.mma('S')
                        s.slot_busy[k % K] = max(s.slot_busy.get(k % K, 0), end)
                        s.q_busy = max(s.q_busy, end)
                        s.events.append((end, lambda sx=sx, tag=(t, j): s.s_tag.__setitem__(sx, tag)))
                        s.commit('S', f'SF{sx}'); issued[sx] += 1
                s.commit('S', f'KE{k % K}')
                if jj + 1 == ti['n_u']: s.commit('S', 'QE')
            kv = kv0 + 2 * ti['n_u'] + nslots(p, ti)
        yield ('done',)

    def pv_thread(s):
        p, K = s.p, s.p.KVS
        kv = 0; waited = [0]; ppar = [0]; prod_count = 0; vuse = [0] * K
        for t in s.tiles():
            ti = decode(p, t)
            if ti['n_u'] == 0: continue
            kv0 = kv
            for jj in range(ti['n_u']):
                j = ti['lo_u'] + jj; v = kv0 + ring_v(jj, ti['n_u'])
                s.ctx['PV'] = ('tile', t, 'jj', jj, 'v', v, 'waited', waited[0])
                sl = v % K
                if s.shared:
                    s.check_alias(f'KF{sl}', v // K, 'PV')
                    yield from s.wait(f'KF{sl}', (v // K) & 1, 'PV')
                else:
                    s.check_alias(f'KV{sl}', vuse[sl], 'PV')
                    yield from s.wait(f'KV{sl}', vuse[sl] & 1, 'PV'); vuse[sl] += 1
                if s.slot_data.get(sl) != (t, 'V', j):
                    s.hazards.append(('P V read a slot not holding its V', sl, s.slot_data.get(sl), (t, 'V', j)))
                for sx in range(p.QS):
                    if not inr(ti, sx, j): continue
                    nx = next_user(ti, sx, j); nx = 0 if nx < 0 else nx
                    first = j == ti['lo'][sx]
                    for half in range(2):
                        s.check_alias(f'PF{half}', prod_count, 'PV')
                        yield from s.wait(f'PF{half}', ppar[0], 'PV')
                        if first and half == 0:
                            pt = s.prev_tile[sx]
                            if pt is not None and s.oread.get(sx, {}).get(pt, set()) != {0, 1}:
                                s.hazards.append(('O overwritten before epilogue read', sx, pt, t))
                            s.prev_tile[sx] = t
                        if s.p_tag[half] != (t, sx, j):
                            s.hazards.append(('P V read a P half not written for it', half, s.p_tag[half], (t, sx, j)))
                        end = s.mma('PV')
                        s.p_busy[half] = max(s.p_busy[half], end)
                        s.slot_busy[sl] = max(s.slot_busy.get(sl, 0), end)
                        s.commit('PV', f'PFR{nx}_{half}')
                    s.commit('PV', f'PVD{sx}'); ppar[0] ^= 1; prod_count += 1
                    if j == ti['hi'][sx] - 1: s.commit('PV', f'OF{sx}')
                s.commit('PV', f'KE{v % K}')
            kv = kv0 + 2 * ti['n_u'] + nslots(p, ti)
        yield ('done',)

    def softmax(s, sx, hf):
        # one actor per group of 4 warps: arrivals count 4 where the kernel has one per warp
        p, K = s.p, s.p.KVS
        who = f'SM{sx}{hf}'
        spar = pfpar = finpar = xpar = 0
        first_use = sx == 0
        kv = 0; pv_count = 0; s_seen = 0; pfree_seen = 0; fin_seen = 0; x_seen = 0; ouse = [0] * K
        def meet():
            nonlocal xpar, x_seen
            s.b[f'X{sx}'].arrive(4)
            s.check_alias(f'X{sx}', x_seen, who)
            yield from s.wait(f'X{sx}', xpar, who); xpar ^= 1; x_seen += 1
        for t in s.tiles():
            ti = decode(p, t)
            kv0 = kv
            if ti['n_u'] > 0: kv += 2 * ti['n_u'] + nslots(p, ti)
            myuse = None; kk = 0
            if ti['n_u'] > 0:
                for s2 in range(p.QS):
                    if via_slot(p, ti, s2):
                        sl = (kv0 + 2 * ti['n_u'] + kk) % K; kk += 1
                        if s2 == sx: myuse = (sl, ouse[sl], (kv0 + 2 * ti['n_u'] + kk - 1) // K)
                        ouse[sl] += 1
            lo, hi = ti['lo'][sx], ti['hi'][sx]
            if lo == hi: continue
            for j in range(lo, hi):
                s.ctx[who] = ('tile', t, 'j', j)
                s.check_alias(f'SF{sx}', s_seen, who)
                yield from s.wait(f'SF{sx}', spar, who); spar ^= 1; s_seen += 1
                if s.s_tag[sx] != (t, j):
                    s.hazards.append(('softmax read an S not computed for it', sx, s.s_tag[sx], (t, j)))
                yield ('work',)
                yield from meet()
                s.b[f'SFR{sx}'].arrive(4)
                rescale = j > lo and s.rng.random() < 0.2
                if not first_use and not s.skip_pfree:
                    s.check_alias(f'PFR{sx}_{hf}', pfree_seen, who)
                    yield from s.wait(f'PFR{sx}_{hf}', pfpar, who); pfpar ^= 1; pfree_seen += 1
                first_use = False
                if rescale:
                    ph = pv_count - 1
                    s.check_alias(f'PVD{sx}', ph, who)
                    yield from s.wait(f'PVD{sx}', ph & 1, who)
                    s.otouch(sx, hf, 'rescale', t)
                if hf == 1: s.b['PF0'].arrive(4)
                yield ('work',)
                # this group's half of P: the previous user's K-steps must have ended
                if s.now < s.p_busy[hf]:
                    s.hazards.append(('P half overwritten while P V reads it', hf, (t, sx, j)))
                s.p_tag[hf] = (t, sx, j)
                s.b[f'PF{hf}'].arrive(4)
                pv_count += 1
            s.check_alias(f'OF{sx}', fin_seen, who)
            yield from s.wait(f'OF{sx}', finpar, who); finpar ^= 1; fin_seen += 1
            yield from meet(); yield from meet()
            if via_slot(p, ti, sx):
                slot, u, ph = myuse
                if s.shared:
                    s.check_alias(f'KF{slot}', ph, who)
                    yield from s.wait(f'KF{slot}', ph & 1, who)
                else:
                    s.check_alias(f'KO{slot}', u, who)
                    yield from s.wait(f'KO{slot}', u & 1, who)
                s.otouch(sx, hf, 'read', t)
                s.slot_write(slot, ('O', t, sx))
                yield ('work',)
                s.b[f'OS{slot}'].arrive(4)
            else:
                s.otouch(sx, hf, 'read', t)
        yield ('done',)

    def store(s):
        p, K = s.p, s.p.KVS
        kv = 0; par = 0; seen = [0] * K
        for t in s.tiles():
            ti = decode(p, t)
            if ti['n_u'] == 0: continue
            kv0 = kv; kv += 2 * ti['n_u'] + nslots(p, ti); k = 0
            for sx in range(p.QS):
                if not via_slot(p, ti, sx): continue
                slot = (kv0 + 2 * ti['n_u'] + k) % K; k += 1
                s.check_alias(f'OS{slot}', seen[slot], 'ST')
                yield from s.wait(f'OS{slot}', (par >> slot) & 1, 'ST'); par ^= 1 << slot; seen[slot] += 1
                yield ('work',)
                s.slot_state[slot] = ('stored',)
                s.b[f'KE{slot}'].arrive()
        yield ('done',)

    def otouch(s, sx, hf, what, t):
        if what == 'read': s.oread.setdefault(sx, {}).setdefault(t, set()).add(hf)
    def slot_write(s, slot, tag):
        s.slot_state[slot] = ('O-staged', tag)

    def run(s, max_steps=2000000):
        roles = {'prod': s.producer(), 'S': s.s_thread(), 'PV': s.pv_thread(),
                 'ST': s.store()}
        for sx in range(s.p.QS):
            for hf in range(2): roles[f'SM{sx}{hf}'] = s.softmax(sx, hf)
        state = {k: None for k in roles}
        done = set(); steps = 0
        while len(done) < len(roles):
            steps += 1
            if steps > max_steps: return 'steps'
            progressed = False
            for k in s.rng.sample(list(roles), len(roles)):
                if k in done: continue
                # a waiting role retries its wait by resuming the generator
                try:
                    st = next(roles[k])
                except StopIteration:
                    done.add(k); progressed = True; continue
                except AssertionError as e:  # a barrier got more arrivals than its phase takes
                    return ('overflow', str(e))
                if st[0] == 'done': done.add(k); progressed = True
                elif st[0] == 'work': progressed = True; state[k] = None
                elif st[0] == 'wait':
                    if state[k] != (st[1], s.b[st[1]].c, s.b[st[1]].pending): progressed = True
                    state[k] = (st[1], s.b[st[1]].c, s.b[st[1]].pending)
                else: progressed = True
            # advance time: fire due events, else jump to next
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
                # everyone waiting, nothing pending
                waiting = {k: state[k] for k in roles if k not in done}
                return ('deadlock', waiting, dict(s.where))
        return 'ok'

