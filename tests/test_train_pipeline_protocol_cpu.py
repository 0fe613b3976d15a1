"""Protocol walk of the train kernels' pipeline at head_dim <= 64 (fmha_sm100.cuh: three rotating
S buffers), modelled in Python: one CTA's TMA producer, the MMA warp with its queue of owed P.V
(S(n) issued only after P.V(n-3); the queue drained at the end of each item), an in-order tensor
pipe whose commits land later, and the two softmax warpgroups, over random interleavings.  A
softmax warp waits for the previous P.V only when it rescales O (random per tile here); the P.V
completions of a query tile go round a ring of four barriers, so those waits stay unambiguous.  Every
mbarrier wait is checked for phase aliasing (a parity wait is only correct while the barrier is
at the awaited phase or one past it), every S for overwriting a P that no P.V has consumed, the
S numbering of the MMA warp against the softmax side's, and the whole for deadlock.  Item
sequences are the kernel's (pairs of query tiles, per-query-tile key-tile ranges from the masks)."""
import random

import pytest

BM = BN = 128
def cdiv(a, b): return -(-a // b)

def ranges(mode, L, S, r0, rl):
    if mode == 0:
        return 0, 0, cdiv(min(L, (rl // S + 1) * S), BN)
    a1 = ((r0 // S) * S) // BN
    e1 = cdiv(min(L, (rl // S + 1) * S), BN)
    n0 = cdiv((rl // S) * S, BN)
    return a1, e1, n0

def items(mode, L, S, B, H, grid, c):
    nq = cdiv(L, 2 * BM); BH = B * H; num = nq * BH
    k = c
    while k < num:
        qp = nq - 1 - k // BH
        q_row0 = qp * 2 * BM
        nact = 2 if q_row0 + BM < L else 1
        a1q, e1q, n0q = [0, 0], [0, 0], [0, 0]
        a1, e1, n0 = 1 << 30, 0, 0
        for q in range(2):
            r0 = q_row0 + q * BM
            if q < nact:
                a1q[q], e1q[q], n0q[q] = ranges(mode, L, S, r0, min(L, r0 + BM) - 1)
                if e1q[q] > a1q[q]:
                    a1 = min(a1, a1q[q]); e1 = max(e1, e1q[q])
                n0 = max(n0, n0q[q])
        if e1 == 0: a1 = 0
        yield dict(nact=nact, a1=a1, n1=e1 - a1, n0=n0, a1q=a1q, e1q=e1q, n0q=n0q, T=e1 - a1 + n0)
        k += grid

def needed(it, q, t):
    if t < it['n1']:
        kt = it['a1'] + t
        return it['a1q'][q] <= kt < it['e1q'][q]
    return (t - it['n1']) < it['n0q'][q]

class Bar:
    def __init__(s, name, count): s.name, s.count, s.arr, s.ph = name, count, 0, 0
    def arrive(s):
        s.arr += 1
        if s.arr == s.count: s.arr = 0; s.ph += 1

def run(mode, L, S, B, H, grid, c, NST, QBUF, NOB, rng, ring=4):
    its = list(items(mode, L, S, B, H, grid, c))
    if not its: return 0
    bars = {}
    def bar(n, cnt=1):
        if n not in bars: bars[n] = Bar(n, cnt)
        return bars[n]
    for i in range(NST): bar(('k_full', i)); bar(('v_full', i)); bar(('kv_empty', i), 2)
    for i in range(QBUF): bar(('q_full', i)); bar(('q_empty', i))
    for i in range(3): bar(('p_full', i), 1)
    for i in range(6): bar(('s_full', i))
    for i in range(2): bar(('tok', i))
    for q in range(2):
        for j in range(ring): bar(('pv_done', q, j))
    for i in range(NOB * 2): bar(('o_free', i), 1)
    tensor = []      # in-order queue of pending completions: list of bar names (commit) ; loads
    loads = []       # async TMA loads: bar names (any order)
    state = dict(pv_issued=set(), s_issued={}, soft_seq={}, p_arrived=set())
    def W(name, k):  # wait for completion of phase index k
        return ('wait', name, k)
    def producer():
        kv = 0
        for ii, it in enumerate(its):
            qb, qr = ii % QBUF, ii // QBUF
            if qr > 0: yield W(('q_empty', qb), qr - 1)
            loads.append(('q_full', qb))
            for t in range(it['T']):
                st, rd = kv % NST, kv // NST
                if rd > 0: yield W(('kv_empty', st), rd - 1)
                loads.append(('k_full', st)); loads.append(('v_full', st))
                kv += 1
    def mma():
        kv = 0; seq = 0; fifo = []; qitem = [0, 0]; qpv = [0, 0]
        def pop():
            e = fifo.pop(0)
            sb = e['seq'] % 3
            yield W(('p_full', sb), e['seq'] // 3)
            ob = e['qi'] % NOB
            if e['first'] and e['qi'] // NOB > 0: yield W(('o_free', ob * 2 + e['q']), e['qi'] // NOB - 1)
            yield W(('v_full', e['st']), e['round'])
            state['pv_issued'].add(e['seq'])
            tensor.append(('pv_done', e['q'], e['pvn'] % ring)); tensor.append(('kv_empty', e['st']))
        for ii, it in enumerate(its):
            qb = ii % QBUF
            yield W(('q_full', qb), ii // QBUF)
            seen = [False, False]
            for t in range(it['T']):
                st, rd = kv % NST, kv // NST
                while any(e['st'] == st for e in fifo):
                    yield from pop()
                yield W(('k_full', st), rd)
                for q in range(2):
                    if q >= it['nact'] or not needed(it, q, t):
                        bars[('kv_empty', st)].arrive(); continue
                    while fifo and fifo[0]['seq'] + 3 <= seq:
                        yield from pop()
                    if seq >= 3: assert seq - 3 in state['pv_issued'], ('S over unconsumed P', seq)
                    state['s_issued'][(ii, t, q)] = seq
                    tensor.append(('s_full', q * 3 + seq % 3))
                    fifo.append(dict(q=q, seq=seq, st=st, round=rd, first=not seen[q], qi=qitem[q], pvn=qpv[q]))
                    qpv[q] += 1
                    assert len(fifo) <= 3
                    seq += 1; seen[q] = True
                kv += 1
            for q in range(2):
                if q < it['nact']: qitem[q] += 1
            tensor.append(('q_empty', qb))
            while fifo: yield from pop()
    def softmax(q):
        qtile = 0; qitem = 0; seq = 0; scnt = [0, 0, 0]; ntok = 0
        for ii, it in enumerate(its):
            if q >= it['nact']:
                seq += sum(1 for t in range(it['T']) if needed(it, 0, t)); continue
            ob = qitem % NOB
            first = True
            for t in range(it['T']):
                n0 = needed(it, 0, t); n1 = it['nact'] > 1 and needed(it, 1, t)
                my = seq + (1 if (q == 1 and n0) else 0)
                seq += int(n0) + int(n1)
                if not needed(it, q, t): continue
                state['soft_seq'][(ii, t, q)] = my
                yield W(('s_full', q * 3 + my % 3), scnt[my % 3]); scnt[my % 3] += 1

                # the warp waits for the previous P.V only when it rescales O (random here)
                if not first and rng.random() < 0.3:
                    yield W(('pv_done', q, (qtile - 1) % ring), (qtile - 1) // ring)
                bars[('p_full', my % 3)].arrive()
                qtile += 1; first = False
            yield W(('pv_done', q, (qtile - 1) % ring), (qtile - 1) // ring)
            bars[('o_free', ob * 2 + q)].arrive()
            qitem += 1
    procs = {'prod': producer(), 'mma': mma(), 's0': softmax(0), 's1': softmax(1)}
    pend = {n: None for n in procs}
    done = set()
    steps = 0
    while True:
        runnable = []
        for n, g in procs.items():
            if n in done: continue
            w = pend[n]
            if w is None: runnable.append(n); continue
            b = bars[w[1]]; k = w[2]
            assert b.ph in (k, k + 1) or b.ph < k, (n, w, b.ph)
            if b.ph == k - 1 and k >= 1:
                raise AssertionError(f'parity alias: {n} waits phase {k} of {w[1]} at ph {b.ph}')
            if b.ph > k + 1: raise AssertionError(f'late wait {n} {w} ph {b.ph}')
            if b.ph > k: runnable.append(n)
        acts = runnable + (['tensor'] if tensor else []) + (['load'] if loads else [])
        if not acts:
            if len(done) == 4: break
            raise AssertionError(f'deadlock: {pend}')
        a = rng.choice(acts); steps += 1
        if a == 'tensor':
            bars[tensor.pop(0)].arrive(); continue
        if a == 'load':
            bars[loads.pop(rng.randrange(len(loads)))].arrive(); continue
        try:
            pend[a] = next(procs[a])
        except StopIteration:
            done.add(a); pend[a] = None
    assert state['s_issued'] == state['soft_seq'], 'S numbering differs'
    return steps



CASES = [(mode, L, S, nob, grid, c)
         for mode in (0, 1)
         for L in (64, 128, 130, 256, 300, 513, 1000, 1024)
         for S in (1, 4, 7, 16, 128, 256) if S <= L
         for nob in (1, 2)
         for grid in (1, 3)
         for c in range(grid)]


def test_single_pv_done_barrier_with_skipped_waits_is_caught():
    """Planted mistake: one P.V completion barrier per query tile while the softmax skips the wait
    on tiles without a rescale; the walk must report a wait that a parity check would pass early."""
    rng = random.Random(5)
    caught = 0
    for m, L, S, nob, grid, c in CASES[::7]:
        try:
            run(m, L, S, 1, 2, grid, c, 4, 2, nob, rng, ring=1)
        except AssertionError:
            caught += 1
    assert caught > 0


@pytest.mark.parametrize("mode", [0, 1])
def test_rotating_s_buffer_protocol(mode):
    rng = random.Random(11 + mode)
    n = 0
    for m, L, S, nob, grid, c in CASES:
        if m != mode:
            continue
        for _ in range(3):
            run(mode, L, S, 1, 2, grid, c, 4, 2, nob, rng)
            n += 1
    assert n > 500
