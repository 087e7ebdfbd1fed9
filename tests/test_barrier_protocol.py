"""CPU model of the kernels' mbarrier protocol (host logic; no GPU).

Every role of a CTA (Q/K producer, V producer, MMA issuer, softmax warps, the
ticket warp) is written as a generator of the waits, arrivals and asynchronous
completions its code performs, in the same order and with the same phase
arithmetic.  A random scheduler interleaves the roles; TMA loads complete in
any order, MMA commits in issue order (one thread's tcgen05 MMAs execute in
order).  Two properties are checked on many random segment layouts:

* no deadlock: some role can always move until all have finished;
* no phase aliasing: when a role waits for completion k of a barrier, the
  barrier has completed at least k - 1 and at most k + 1 phases (an mbarrier
  parity wait cannot tell phase k from k - 2 or k + 2: it would pass too early
  or hang).

Planted protocol errors (an off-by-one wait index; the wide kernel's V-tail
zeroing without its wait for the ring slot's release) must be caught.
"""
import random

import pytest


class _Bar:
    def __init__(self, count):
        self.count, self.arrived, self.done = count, 0, 0

    def arrive(self):
        self.arrived += 1
        if self.arrived == self.count:
            self.arrived = 0
            self.done += 1


class ProtocolError(RuntimeError):
    pass


def _simulate(bars, roles, rnd):
    """roles: name -> generator of ('wait', bar, k) | ('arrive', bar) | ('mma', [bars]) | ('tma', [bars])."""
    state = {r: None for r in roles}
    mma_q, tma_q = [], []
    while roles:
        runnable = []
        for r in roles:
            st = state[r]
            if st is None:
                runnable.append(r)
                continue
            b = bars[st[1]]
            if b.done > st[2] + 1:
                raise ProtocolError("aliasing: %s waits for completion %d of %s, %d done" % (r, st[2], st[1], b.done))
            if b.done > st[2]:
                runnable.append(r)
        choices = runnable + (["<mma done>"] if mma_q else []) + (["<tma done>"] if tma_q else [])
        if not choices:
            raise ProtocolError("deadlock: " + ", ".join("%s@%s" % (r, state[r][1:]) for r in roles))
        c = rnd.choice(choices)
        if c == "<mma done>":
            for b in mma_q.pop(0):
                bars[b].arrive()
            continue
        if c == "<tma done>":
            for b in tma_q.pop(rnd.randrange(len(tma_q))):
                bars[b].arrive()
            continue
        state[c] = None
        try:
            op = next(roles[c])
        except StopIteration:
            del roles[c], state[c]
            continue
        if op[0] == "wait":
            if op[2] >= 0:
                if bars[op[1]].done < op[2]:
                    # the barrier's phase op[2] - 1 is still open: a parity wait for
                    # phase op[2] would see the parity of phase op[2] - 2 and pass at once
                    raise ProtocolError("early pass: %s waits for completion %d of %s, %d done"
                                        % (c, op[2], op[1], bars[op[1]].done))
                state[c] = op
        elif op[0] == "arrive":
            bars[op[1]].arrive()
        elif op[0] == "mma":
            mma_q.append(op[1])
        elif op[0] == "tma":
            tma_q.append(op[1])


# --------------------------------------------------------------------------
# two-lane kernel (head dims 64 / 128): gqa_fwd2_kernel


def _two_lane(segs, rbq, stk, stv, rnd, mutate=False):
    """segs: list of (ntiles, kind); kind 1 = split segment (partial rows + ticket)."""
    bars = {}

    def mk(name, count):
        bars[name] = _Bar(count)

    mk("QFULL", 1)
    mk("QEMPTY", 1)
    for i in range(stk):
        mk("KF%d" % i, 1)
        mk("KE%d" % i, 1)
    for i in range(stv):
        mk("VF%d" % i, 1)
        mk("VE%d" % i, 1)
    for lane in range(2):
        mk("SF%d" % lane, 1)
        mk("PF%d" % lane, 4)
        mk("OD%d" % lane, 1)
    mk("X", 8)
    for j in range(2):
        mk("MJ%d" % j, 1)
        mk("MT%d" % j, 1)
    tail = [[rnd.random() < 0.3 for _ in range(n)] for n, _ in segs]
    merges = [rnd.random() < 0.5 for _ in segs]
    nsplit = min(2, sum(1 for _, k in segs if k == 1))

    def kprod():
        g = 0
        for si, (n, _) in enumerate(segs):
            yield ("wait", "QEMPTY", si - 1)
            yield ("tma", ["QFULL"])
            for _ in range(n):
                yield ("wait", "KE%d" % (g % stk), g // stk - 1)
                yield ("tma", ["KF%d" % (g % stk)])
                g += 1

    def vprod():
        g = 0
        for n, _ in segs:
            for _ in range(n):
                yield ("wait", "VE%d" % (g % stv), g // stv - 1)
                yield ("tma", ["VF%d" % (g % stv)])
                g += 1

    def mma():
        g = 0
        n_pv = [0, 0]

        def pv(lane, gv, wait_v):
            idx = n_pv[lane] + (1 if mutate else 0)
            yield ("wait", "PF%d" % lane, idx)
            n_pv[lane] += 1
            if wait_v:
                yield ("wait", "VF%d" % (gv % stv), gv // stv)
            yield ("mma", ["OD%d" % lane, "VE%d" % (gv % stv)] if rbq == 1 or lane == 1 else ["OD%d" % lane])

        for si, (n, _) in enumerate(segs):
            yield ("wait", "QFULL", si)
            prev = None
            pend_b = None
            for t in range(n):
                if rbq == 1 or t == 0:
                    yield ("wait", "KF%d" % (g % stk), g // stk)
                last = ["QEMPTY"] if t == n - 1 else []
                if rbq == 1:
                    lane = g & 1
                    yield ("mma", ["SF%d" % lane, "KE%d" % (g % stk)] + last)
                    if prev is not None:
                        yield from pv(prev[0], prev[1], True)
                    prev = (lane, g)
                else:
                    if t == 0:
                        yield ("mma", ["SF0"])
                    if pend_b is not None:
                        yield from pv(1, pend_b, False)
                    yield ("mma", ["SF1", "KE%d" % (g % stk)] + last)
                    # V(t) and K(t+1) awaited before P0(t); S0(t+1) right after PV0(t)
                    yield ("wait", "VF%d" % (g % stv), g // stv)
                    if t + 1 < n:
                        yield ("wait", "KF%d" % ((g + 1) % stk), (g + 1) // stk)
                    yield from pv(0, g, False)
                    if t + 1 < n:
                        yield ("mma", ["SF0"])
                    pend_b = g
                g += 1
            # the segment's last PV goes out when its tile loop ends
            if prev is not None:
                yield from pv(prev[0], prev[1], True)
            if pend_b is not None:
                yield from pv(1, pend_b, False)

    xph = [0] * 8

    def softmax(w):
        lane = w // 4
        g = 0
        cnt = 0
        njob = 0

        def xsync():
            yield ("arrive", "X")
            yield ("wait", "X", xph[w])
            xph[w] += 1

        for si, (n, kind) in enumerate(segs):
            mine = 0
            for t in range(n):
                if rbq == 1 and (g & 1) != lane:
                    g += 1
                    continue
                yield ("wait", "SF%d" % lane, cnt)
                if mine > 0 and rnd.random() < 0.3:  # lazy rescale (decided per warp)
                    yield ("wait", "OD%d" % lane, cnt - 1)
                if tail[si][t]:  # zeroing padded V rows of the tile
                    yield ("wait", "VF%d" % (g % stv), g // stv)
                yield ("arrive", "PF%d" % lane)
                cnt += 1
                mine += 1
                g += 1
            if mine > 0:
                yield ("wait", "OD%d" % lane, cnt - 1)
            if rbq == 1:
                yield from xsync()
            yield from xsync()
            if kind == 1 and njob < 2:
                if w == 0:
                    yield ("arrive", "MJ%d" % njob)
                njob += 1
        for j in range(njob):
            yield ("wait", "MT%d" % j, 0)
            if merges[j]:
                for _ in range(3):
                    yield from xsync()

    def tickets():
        for j in range(nsplit):
            yield ("wait", "MJ%d" % j, 0)
            yield ("arrive", "MT%d" % j)

    roles = {"kprod": kprod(), "vprod": vprod(), "mma": mma(), "tickets": tickets()}
    for w in range(8):
        roles["softmax%d" % w] = softmax(w)
    _simulate(bars, roles, rnd)


# --------------------------------------------------------------------------
# wide kernel (head dims 256 / 512): gqa_wide_kernel


def _wide(segs, nbox, vch, nslot, rnd, mutate=False):
    """gqa_wide_kernel (head dims 256 / 512): K and V stream through one ring of
    nslot chunks in the MMA's order (K(0); per tile g >= 1 [K(g), V(g-1)], or
    [V(g-1), K(g)] where g starts a segment; V(last)); the softmax warps zero the
    padded V rows of a segment's last tile in its ring slots."""
    bars = {}

    def mk(name, count):
        bars[name] = _Bar(count)

    mk("QFULL", 1)
    mk("QEMPTY", 1)
    for i in range(nslot):
        mk("RF%d" % i, 1)
        mk("RE%d" % i, 1)
    for b in range(2):
        mk("SF%d" % b, 1)
        mk("PF%d" % b, 4)
        mk("OD%d" % b, 1)
        mk("MJ%d" % b, 1)
    mk("OFREE", 4)
    mk("X", 4)
    ch = nbox + vch
    grow = [[rnd.random() < 0.3 for _ in range(n)] for n, _ in segs]
    tail = [rnd.random() < 0.5 for _ in segs]     # the segment ends its row-block
    nsplit = min(2, sum(1 for _, k in segs if k == 1))

    def ring():
        seq = 0
        prev = False
        for n, _ in segs:
            for t in range(n):
                order = (["V"] * vch + ["K"] * nbox) if (prev and t == 0) else \
                    (["K"] * nbox + (["V"] * vch if prev else []))
                for _ in order:
                    yield ("wait", "RE%d" % (seq % nslot), seq // nslot - 1)
                    yield ("tma", ["RF%d" % (seq % nslot)])
                    seq += 1
                prev = True
        if prev:
            for _ in range(vch):
                yield ("wait", "RE%d" % (seq % nslot), seq // nslot - 1)
                yield ("tma", ["RF%d" % (seq % nslot)])
                seq += 1

    def qprod():
        for si in range(len(segs)):
            yield ("wait", "QEMPTY", si - 1)
            yield ("tma", ["QFULL"])

    def mma():
        st = {"seq": 0}

        def take():
            sq = st["seq"]
            yield ("wait", "RF%d" % (sq % nslot), sq // nslot)
            st["seq"] += 1
            return sq % nslot

        def s_mma(gg, last):
            for _ in range(nbox):
                sl = yield from take()
                yield ("mma", ["RE%d" % sl])
            yield ("mma", ["SF%d" % (gg % 2)] + (["QEMPTY"] if last else []))

        def pv(gg, first, seg):
            yield ("wait", "PF%d" % (gg % 2), gg // 2)
            if first and seg > 0:
                yield ("wait", "OFREE", seg - 1)
            for _ in range(vch):
                sl = yield from take()
                yield ("mma", ["RE%d" % sl])
            yield ("mma", ["OD%d" % (gg % 2)])

        g = 0
        prev = None
        for si, (n, _) in enumerate(segs):
            if prev is not None:
                yield from pv(*prev)
                prev = None
            yield ("wait", "QFULL", si)
            for t in range(n):
                yield from s_mma(g, t == n - 1)
                if prev is not None:
                    yield from pv(*prev)
                prev = (g, t == 0, si)
                g += 1
        if prev is not None:
            yield from pv(*prev)

    xph = [0] * 4

    def softmax(w):
        def xsync():
            yield ("arrive", "X")
            yield ("wait", "X", xph[w])
            xph[w] += 1

        g = 0
        njob = 0
        for si, (n, kind) in enumerate(segs):
            for t in range(n):
                yield ("wait", "SF%d" % (g % 2), g // 2)
                if grow[si][t] and t > 0:
                    yield ("wait", "OD%d" % ((g - 1) % 2), (g - 1) // 2)
                if tail[si] and t == n - 1:
                    vs = nbox + g * ch  # V(g)'s first ring chunk
                    for v in range(vch):
                        sq = vs + v
                        if not mutate:
                            yield ("wait", "RE%d" % (sq % nslot), sq // nslot - 1)
                        yield ("wait", "RF%d" % (sq % nslot), sq // nslot)
                yield ("arrive", "PF%d" % (g % 2))
                g += 1
            yield ("wait", "OD%d" % ((g - 1) % 2), (g - 1) // 2)
            yield ("arrive", "OFREE")
            if kind == 1 and njob < 2:
                yield from xsync()
                if w == 0:
                    yield ("arrive", "MJ%d" % njob)
                njob += 1
        for j in range(njob):
            for _ in range(3):
                yield from xsync()

    def publisher():
        for j in range(nsplit):
            yield ("wait", "MJ%d" % j, 0)

    roles = {"ring": ring(), "qprod": qprod(), "mma": mma(), "publisher": publisher()}
    for w in range(4):
        roles["softmax%d" % w] = softmax(w)
    _simulate(bars, roles, rnd)


# --------------------------------------------------------------------------
# swap-AB decode kernel (head dim 128, at most 16 packed rows): gqa_dec_kernel


def _decode(segs, stk, stv, rnd, epiw=True, mutate=False):
    """epiw: the segment epilogues run on their own warpgroup (bf16 K/V);
    otherwise the softmax warps run each one right after the segment (FP8 K/V,
    whose warps 8-11 convert tiles)."""
    bars = {}

    def mk(name, count):
        bars[name] = _Bar(count)

    for i in range(2):
        mk("QF%d" % i, 1)
        mk("QE%d" % i, 1)
        mk("SF%d" % i, 1)
        mk("PF%d" % i, 4)
        mk("PD%d" % i, 1)
        mk("OF%d" % i, 4)   # epilogue has read O' buffer i and its row statistics
        mk("ST%d" % i, 4)   # softmax has written the row statistics of buffer i
        mk("SP%d" % i, 1)   # a segment's last PV' into buffer i completed
    for i in range(stk):
        mk("KF%d" % i, 1)
        mk("KE%d" % i, 1)
    for i in range(stv):
        mk("VF%d" % i, 1)
        mk("VE%d" % i, 1)
    mk("RED", 4)
    mk("X", 4)
    mk("E", 4)
    mk("BOUNDS", 1)
    # decisions every softmax warp takes alike (they follow the CTA-wide row maxima)
    grow = [[rnd.random() < 0.3 for _ in range(n)] for n, _ in segs]
    tail = [[rnd.random() < 0.3 for _ in range(n)] for n, _ in segs]
    merges = [rnd.random() < 0.5 for _ in segs]

    def kprod():
        g = 0
        for si, (n, _) in enumerate(segs):
            yield ("wait", "QE%d" % (si % 2), si // 2 - 1)
            yield ("tma", ["QF%d" % (si % 2)])
            for _ in range(n):
                yield ("wait", "KE%d" % (g % stk), g // stk - 1)
                yield ("tma", ["KF%d" % (g % stk)])
                g += 1

    def vprod():
        g = 0
        for n, _ in segs:
            for _ in range(n):
                yield ("wait", "VE%d" % (g % stv), g // stv - 1)
                yield ("tma", ["VF%d" % (g % stv)])
                g += 1

    def bounds():
        yield ("arrive", "BOUNDS")

    def mma():
        def pv(gg, first, seg, last):
            yield ("wait", "PF%d" % (gg % 2), gg // 2)
            yield ("wait", "VF%d" % (gg % stv), gg // stv)
            if first and seg >= 2:
                yield ("wait", "OF%d" % (seg % 2), (seg - 2) // 2)
            yield ("mma", ["PD%d" % (gg % 2), "VE%d" % (gg % stv)] + (["SP%d" % (seg % 2)] if last else []))

        g = 0
        prev = None
        for si, (n, _) in enumerate(segs):
            if prev is not None:
                yield from pv(*prev, True)
                prev = None
            yield ("wait", "QF%d" % (si % 2), si // 2)
            for t in range(n):
                yield ("wait", "KF%d" % (g % stk), g // stk)
                yield ("mma", ["SF%d" % (g % 2), "KE%d" % (g % stk)] + (["QE%d" % (si % 2)] if t == n - 1 else []))
                if prev is not None:
                    yield from pv(*prev, False)
                prev = (g, t == 0, si)
                g += 1
        if prev is not None:
            yield from pv(*prev, True)

    ph = {}
    # the statistics slots: the segment each epilogue warp last read from slot b
    read = [[-2] * 4 for _ in range(2)]

    def epilogue(w, si, kind, sync):
        yield ("wait", "ST%d" % (si % 2), si // 2)
        yield ("wait", "SP%d" % (si % 2), si // 2)
        read[si % 2][w] = si  # O' buffer and statistics read, then released
        yield ("arrive", "OF%d" % (si % 2))
        if kind == 1:
            yield from sync()
            if w == 0:
                yield ("wait", "BOUNDS", 0)
            yield from sync()
            if merges[si]:
                for _ in range(3):
                    yield from sync()

    def softmax(w):
        ph[w] = {"RED": 0, "X": 0}

        def sync(name):
            yield ("arrive", name)
            yield ("wait", name, ph[w][name])
            ph[w][name] += 1

        g = 0
        for si, (n, kind) in enumerate(segs):
            for t in range(n):
                yield ("wait", "SF%d" % (g % 2), g // 2)
                yield from sync("RED")
                if grow[si][t] and t > 0:
                    yield ("wait", "PD%d" % ((g - 1) % 2), (g - 1) // 2)
                if g >= 2:
                    yield ("wait", "PD%d" % (g % 2), (g - 2) // 2)
                if tail[si][t]:
                    yield ("wait", "VF%d" % (g % stv), g // stv)
                yield ("arrive", "PF%d" % (g % 2))
                g += 1
            yield from sync("RED")
            if si >= 2 and not mutate:
                yield ("wait", "OF%d" % (si % 2), (si - 2) // 2)
            # writing slot si % 2 while an epilogue warp has not read segment si - 2 from it
            if si >= 2 and min(read[si % 2]) < si - 2:
                raise ProtocolError("statistics slot %d overwritten before segment %d was read" % (si % 2, si - 2))
            yield ("arrive", "ST%d" % (si % 2))
            if not epiw:
                yield from epilogue(w, si, kind, lambda: sync("X"))

    def epi_warp(w):
        ph[("e", w)] = 0

        def sync():
            yield ("arrive", "E")
            yield ("wait", "E", ph[("e", w)])
            ph[("e", w)] += 1

        for si, (n, kind) in enumerate(segs):
            yield from epilogue(w, si, kind, sync)

    roles = {"kprod": kprod(), "vprod": vprod(), "mma": mma(), "bounds": bounds()}
    for w in range(4):
        roles["softmax%d" % w] = softmax(w)
        if epiw:
            roles["epilogue%d" % w] = epi_warp(w)
    _simulate(bars, roles, rnd)


def _layouts(seed, count):
    rnd = random.Random(seed)
    for trial in range(count):
        segs = [(rnd.randint(1, 6), rnd.choice([0, 1])) for _ in range(rnd.randint(1, 5))]
        yield trial, segs, rnd.randint(2, 4), rnd.randint(2, 4)


@pytest.mark.parametrize("rbq", [1, 2])
def test_two_lane_protocol_has_no_deadlock_or_aliasing(rbq):
    for trial, segs, stk, stv in _layouts(11 + rbq, 400):
        _two_lane(segs, rbq, stk, stv, random.Random(trial))


@pytest.mark.parametrize("nbox,vch,nslot", [(8, 4, 6), (4, 4, 10), (8, 4, 5), (4, 4, 4)])
def test_wide_protocol_has_no_deadlock_or_aliasing(nbox, vch, nslot):
    """The shapes of the two instantiations (d = 512: 8 K and 4 V chunks per tile,
    6 slots; d = 256: 4 + 4, 10 slots) and two tighter rings."""
    for trial, segs, _, _ in _layouts(17 + nslot, 300):
        _wide(segs, nbox, vch, nslot, random.Random(trial))


def test_model_catches_the_wide_tail_wait_without_the_release_wait():
    """The hazard needs the ring producer to lag behind the softmax warps, which
    few random interleavings produce: the seeded trials include some."""
    caught = 0
    for trial, segs, _, _ in _layouts(23, 1000):
        try:
            _wide(segs, 8, 4, 6, random.Random(trial), mutate=True)
        except ProtocolError:
            caught += 1
    assert caught > 0


@pytest.mark.parametrize("epiw", [True, False])
def test_decode_protocol_has_no_deadlock_or_aliasing(epiw):
    for trial, segs, stk, stv in _layouts(5, 400):
        _decode(segs, stk, stv, random.Random(trial), epiw=epiw)


def test_model_catches_the_decode_statistics_written_before_their_slot_is_free():
    """Without the softmax's wait for the epilogue two segments back, the
    statistics barrier can run two phases ahead of the epilogue warps."""
    caught = 0
    rnd = random.Random(29)
    for trial in range(1000):
        # short split segments: the softmax runs ahead of the epilogue warps
        segs = [(rnd.randint(1, 2), 1) for _ in range(6)]
        try:
            _decode(segs, 3, 3, random.Random(trial), epiw=True, mutate=True)
        except ProtocolError:
            caught += 1
    assert caught > 0


def test_model_catches_a_wrong_wait_index():
    caught = 0
    for trial, segs, stk, stv in _layouts(3, 60):
        try:
            _two_lane(segs, 1, stk, stv, random.Random(trial), mutate=True)
        except ProtocolError:
            caught += 1
    assert caught == 60
