"""Protocol walk of the backward's rows-Q launch (attn_bwd_sm100.cuh, head_dim 64 and 128: one
accumulator), modelled in Python over random interleavings of its roles: the TMA producer (row
tiles, the forward's out tile, the column ring), the row-data warp (c_i and -lse log2 e per item),
the product issuer (S and dP of every sub-tile into its TMEM set), the accumulation issuer, an
in-order tensor pipe whose commits land later, and the two softmax warpgroups with the epilogue
hand-over: only the warpgroup that took an item's last sub-tile runs the epilogue, the other
writes its row sums into an exchange slot (two slots by item parity), arrives on usum_ready and
goes on; the epilogue warpgroup waits for that barrier, for the stage (stg_free, one arrival by
the thread whose store has read it) and for the accumulator, then releases the accumulator.

Every mbarrier wait is checked for phase aliasing (a parity wait is only correct while the
barrier is at the awaited phase or one past it), every buffer for reuse before its reader is done
(TMEM sets, column stages, row buffers, the out tile, the row-data slots, the exchange slots, the
stage, the accumulator), and the whole for deadlock.  Item lengths (sub-tiles per item) are
random, 1 to 9, which covers the masks' lengths and more; some runs keep the tensor pipe and the
copies slow against the warps.  Taking out the usum_ready or the acc_free wait is caught.  Taking
out the stg_free wait is not: the storing thread waits for its store's read before its warpgroup
can arrive on the next usum_ready or p_full, so the other warpgroup cannot reach the stage
earlier; the barrier stays as a guard that does not lean on that."""
import random

import pytest


class Bar:
    def __init__(s, name, count=1):
        s.name, s.count, s.arr, s.ph = name, count, 0, 0

    def arrive(s, n=1):
        s.arr += n
        assert s.arr <= s.count, f"{s.name}: too many arrivals"
        if s.arr == s.count:
            s.arr = 0
            s.ph += 1


class Walk:
    def __init__(s, nsubs, NSET, NST, RBUF, rng):
        s.nsubs, s.NSET, s.NST, s.RBUF, s.rng = nsubs, NSET, NST, RBUF, rng
        B = Bar
        s.row_full = [B(f"row_full{i}") for i in range(RBUF)]
        s.row_empty = [B(f"row_empty{i}", 2) for i in range(RBUF)]  # MMA commit + row-data warp
        s.col_full = [B(f"col_full{i}") for i in range(NST)]
        s.col_empty = [B(f"col_empty{i}") for i in range(NST)]
        s.s_full = [B(f"s_full{i}") for i in range(NSET)]
        s.p_full = [B(f"p_full{i}") for i in range(NSET)]
        s.set_free = [B(f"set_free{i}") for i in range(NSET)]
        s.acc_full, s.acc_free = B("acc_full"), B("acc_free")
        s.rowd_full = [B(f"rowd_full{i}") for i in range(2)]
        s.rowd_empty = [B(f"rowd_empty{i}", 2) for i in range(2)]  # both warpgroups
        s.out_full, s.out_empty = B("out_full"), B("out_empty")
        s.acc_issued = B("acc_issued")
        s.usum_ready = [B(f"usum_ready{i}") for i in range(2)]
        s.stg_free = B("stg_free")
        # data: what each buffer holds, to check every reader sees its own item / sub-tile
        s.rows = [None] * RBUF      # item whose Q/dO tiles are in the buffer
        s.rows_readers = [set() for _ in range(RBUF)]
        s.out = None
        s.cols = [None] * NST       # sub-tile whose K/V tile is in the stage
        s.setS = [None] * NSET      # sub-tile whose S/dP the set holds
        s.setP = [None] * NSET      # sub-tile whose p/u the set holds
        s.rowd = [None, None]
        s.rowd_read = [set(), set()]
        s.xch = [[None, None], [None, None]]
        s.acc = None                # (item, sub-tiles accumulated)
        s.stage = None
        s.tc = []                   # in-order tensor pipe: list of callables
        s.async_ops = []            # TMA loads / store reads in flight: callables
        s.item_of, s.first_of = [], []
        for iw, ns in enumerate(nsubs):
            s.first_of.append(len(s.item_of))
            s.item_of += [iw] * ns

    # a wait for the k-th completion of a barrier (k < 0: nothing to wait for)
    def ready(s, bar, k):
        if k < 0:
            return True
        assert bar.ph in (k, k + 1), f"{bar.name}: waiting for phase {k} at phase {bar.ph} (parity aliasing)"
        return bar.ph == k + 1

    def wait(s, bar, k):
        while not s.ready(bar, k):
            yield

    def producer(s):
        n = 0
        for iw, ns in enumerate(s.nsubs):
            rb = iw % s.RBUF
            yield from s.wait(s.row_empty[rb], iw // s.RBUF - 1)
            assert s.rows[rb] is None or s.rows_readers[rb] >= {"mma", "rowd"}, "row buffer reused early"

            def land_rows(rb=rb, iw=iw):
                s.rows[rb], s.rows_readers[rb] = iw, set()
                s.row_full[rb].arrive()
            s.async_ops.append(land_rows)
            yield from s.wait(s.out_empty, iw - 1)

            def land_out(iw=iw):
                s.out = iw
                s.out_full.arrive()
            s.async_ops.append(land_out)
            for t in range(ns):
                st = n % s.NST
                yield from s.wait(s.col_empty[st], n // s.NST - 1)

                def land_col(st=st, n=n):
                    s.cols[st] = n
                    s.col_full[st].arrive()
                s.async_ops.append(land_col)
                n += 1
                yield

    def rowdata(s):
        for iw in range(len(s.nsubs)):
            par, rb = iw & 1, iw % s.RBUF
            yield from s.wait(s.rowd_empty[par], (iw >> 1) - 1)
            assert s.rowd[par] is None or s.rowd_read[par] == {0, 1}, "row-data slot reused early"
            yield from s.wait(s.row_full[rb], iw // s.RBUF)
            yield from s.wait(s.out_full, iw)
            assert s.rows[rb] == iw and s.out == iw
            yield
            s.rowd[par], s.rowd_read[par] = iw, set()
            s.rows_readers[rb].add("rowd")
            s.out_empty.arrive()
            s.row_empty[rb].arrive()
            s.rowd_full[par].arrive()

    def mma(s):
        n = 0
        for iw, ns in enumerate(s.nsubs):
            rb = iw % s.RBUF
            yield from s.wait(s.row_full[rb], iw // s.RBUF)
            if iw > 0:
                yield from s.wait(s.acc_issued, iw - 1)
            for t in range(ns):
                st, st_set = n % s.NST, n % s.NSET
                yield from s.wait(s.col_full[st], n // s.NST)
                yield from s.wait(s.set_free[st_set], n // s.NSET - 1)

                def products(n=n, st=st, set_=st_set, rb=rb, iw=iw, last=(t == ns - 1)):
                    assert s.rows[rb] == iw and s.cols[st] == n, "products read a stale tile"
                    assert s.setP[set_] is None or s.setP[set_] == ("consumed", n - s.NSET) or n < s.NSET, \
                        "S/dP overwrote a p/u the accumulation has not read"
                    s.setS[set_] = n
                    s.s_full[set_].arrive()
                    if last:
                        s.rows_readers[rb].add("mma")
                        s.row_empty[rb].arrive()
                s.tc.append(products)
                n += 1
                yield

    def accum(s):
        n = 0
        for iw, ns in enumerate(s.nsubs):
            for t in range(ns):
                st, set_ = n % s.NST, n % s.NSET
                yield from s.wait(s.p_full[set_], n // s.NSET)
                if t == 0:
                    yield from s.wait(s.acc_free, iw - 1)

                def acc(n=n, st=st, set_=set_, iw=iw, t=t, last=(t == ns - 1)):
                    assert s.setP[set_] == n and s.cols[st] == n, "accumulation read a stale p/u or tile"
                    if t == 0:
                        assert s.acc is None or s.acc == ("read", iw - 1), "accumulator overwritten before read"
                        s.acc = (iw, 1)
                    else:
                        assert s.acc == (iw, t)
                        s.acc = (iw, t + 1)
                    s.setP[set_] = ("consumed", n)
                    s.col_empty[st].arrive()
                    s.set_free[set_].arrive()
                    if last:
                        s.acc_full.arrive()
                s.tc.append(acc)
                if t == ns - 1:
                    s.acc_issued.arrive()
                n += 1
                yield

    def softmax(s, w):
        n = 0
        for iw, ns in enumerate(s.nsubs):
            par = iw & 1
            yield from s.wait(s.rowd_full[par], iw >> 1)
            assert s.rowd[par] == iw
            s.rowd_read[par].add(w)
            s.rowd_empty[par].arrive()
            for t in range(ns):
                if (n & 1) == w:
                    set_ = n % s.NSET
                    yield from s.wait(s.s_full[set_], n // s.NSET)
                    assert s.setS[set_] == n, "softmax read a stale S/dP"
                    yield
                    s.setP[set_] = n
                    s.p_full[set_].arrive()
                n += 1
            w_late = (n - 1) & 1
            if w != w_late:
                slot = s.xch[par][w]
                assert slot is None or (isinstance(slot, tuple) and slot[0] == "read"), "exchange slot reused early"
                s.xch[par][w] = iw
                s.usum_ready[par].arrive()
            else:
                yield from s.wait(s.usum_ready[par], iw >> 1)
                assert s.xch[par][1 - w] == iw, "epilogue read another item's row sums"
                s.xch[par][1 - w] = ("read", iw)
                yield from s.wait(s.stg_free, iw - 1)
                yield from s.wait(s.acc_full, iw)
                assert s.acc == (iw, ns), "epilogue read an incomplete accumulator"
                yield
                assert s.stage is None or s.stage == ("read", iw - 1), "stage overwritten before the store read it"
                s.acc = ("read", iw)
                s.stage = iw
                s.acc_free.arrive()
                done = []

                def store_read(iw=iw):
                    s.stage = ("read", iw)
                    done.append(1)
                s.async_ops.append(store_read)
                while not done:  # the storing thread waits for the read, then frees the stage
                    yield
                s.stg_free.arrive()
            yield

    def run(s):
        roles = [s.producer(), s.rowdata(), s.mma(), s.accum(), s.softmax(0), s.softmax(1)]
        live = list(roles)
        idle = 0
        # how often the tensor pipe and the copies make progress against the warps: some runs
        # keep them slow, so that warps run far ahead of their data
        p_tc, p_async = s.rng.choice([0.02, 0.2]), s.rng.choice([0.01, 0.2])
        while live or s.tc or s.async_ops:
            u = s.rng.random()
            if s.tc and (u < p_tc or not live):
                kind, r = "tc", None
            elif s.async_ops and (u > 1 - p_async or not live):
                kind, r = "async", None
            elif live:
                kind, r = "role", s.rng.choice(live)
            else:
                kind, r = ("tc", None) if s.tc else ("async", None)
            if kind == "tc":
                s.tc.pop(0)()
                idle = 0
            elif kind == "async":
                s.async_ops.pop(s.rng.randrange(len(s.async_ops)))()
                idle = 0
            else:
                try:
                    next(r)
                    idle += 1
                except StopIteration:
                    live.remove(r)
                    idle = 0
            assert idle < 20000, "deadlock"
        assert s.acc == ("read", len(s.nsubs) - 1)


@pytest.mark.parametrize("cfg", [dict(NSET=3, NST=6, RBUF=2), dict(NSET=2, NST=2, RBUF=1)],
                         ids=["head_dim64", "head_dim128"])
def test_rowsq_epilogue_handover_protocol(cfg):
    rng = random.Random(20261203)
    for _ in range(300):
        nsubs = [rng.randint(1, 9) for _ in range(rng.randint(1, 9))]
        Walk(nsubs, rng=rng, **cfg).run()


def test_protocol_walk_catches_a_single_exchange_slot():
    """Planted mistake: one exchange slot and usum_ready barrier for every item instead of one
    per item parity; the walk must report it (aliasing or an overwritten slot)."""
    rng = random.Random(7)
    caught = 0
    for _ in range(300):
        nsubs = [rng.randint(1, 9) for _ in range(rng.randint(2, 9))]
        w = Walk(nsubs, NSET=3, NST=6, RBUF=2, rng=rng)
        w.usum_ready = [w.usum_ready[0]] * 2
        w.xch = [w.xch[0]] * 2
        try:
            w.run()
        except AssertionError:
            caught += 1
    assert caught > 0
