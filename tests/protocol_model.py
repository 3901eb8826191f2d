"""Randomised models of the attention kernels' mbarrier protocols (test infrastructure).

Each kernel's roles (TMA producers, the MMA issuer, compute warpgroups) are
written as Python generators that follow the kernel's wait / arrive / issue
sequence, with the same barrier counts (a role played by several warps counts
once per warp group here) and the same phase arithmetic.  A scheduler runs one
runnable role at a time in random order; the tensor pipe executes issued MMAs
and commits in order; TMA copies land in any order.

Checked on every schedule:
  * no deadlock (every role finishes);
  * every parity wait is evaluated with its barrier at the awaited phase or one
    past it -- the hardware sees only the parity, so a barrier two phases ahead
    (or one behind) would block forever (or pass early);
  * every buffer (K/V/Q/dO stages, the S/P and dP/dS regions of TMEM, the
    accumulators, staged row statistics) holds the expected tile whenever an
    MMA or a compute role reads or overwrites it.

The sequences restate the kernels in csrc/ (fwd_sm100.cu, bwd_dq_sm100.cu,
bwd_dkdv_sm100.cu, bwd_fused_sm100.cu); a change to a kernel's protocol needs
the same change here.
"""
from __future__ import annotations

import random


class Hazard(Exception):
    pass


class Bar:
    def __init__(self, name, count):
        self.name, self.count, self.pending, self.done = name, count, 0, 0

    def arrive(self):
        self.pending += 1
        if self.pending == self.count:
            self.pending = 0
            self.done += 1

    def ready(self, k):
        """Wait for phase k (k = -1: the phase before the first, complete on a fresh barrier)."""
        c = self.done
        if c == k + 2:
            raise Hazard(f"{self.name}: wait for phase {k} with the barrier two phases ahead")
        if c >= k + 3 or (c <= k - 1 and not (k == -1 and c == 0)):
            raise Hazard(f"{self.name}: wait for phase {k} evaluated with {c} phases done")
        return c >= k + 1


def wait(name, k):
    return ("wait", name, k)


STEP = ("step",)


class Sim:
    def __init__(self, seed):
        self.rng = random.Random(seed)
        self.bars = {}
        self.pipe = []  # in order: ("mma", fn) | ("commit", barrier)
        self.tma = []   # in flight: (barrier, fn)

    def bar(self, name, count=1):
        self.bars[name] = Bar(name, count)

    def arrive(self, name):
        self.bars[name].arrive()

    def run(self, roles, max_steps=400000):
        pending, finished = {}, set()

        def advance(name):
            try:
                pending[name] = next(roles[name])
            except StopIteration:
                finished.add(name)

        for name in roles:
            advance(name)
        for _ in range(max_steps):
            cands = [n for n in roles if n not in finished and
                     (pending[n][0] != "wait" or self.bars[pending[n][1]].ready(pending[n][2]))]
            if self.pipe:
                cands.append("#pipe")
            if self.tma:
                cands.append("#tma")
            if not cands:
                if len(finished) == len(roles):
                    return
                raise Hazard(f"deadlock: { {n: pending[n] for n in roles if n not in finished} }")
            c = self.rng.choice(cands)
            if c == "#pipe":
                kind, x = self.pipe.pop(0)
                if kind == "mma":
                    x()
                else:
                    self.arrive(x)
            elif c == "#tma":
                b, f = self.tma.pop(self.rng.randrange(len(self.tma)))
                f()
                self.arrive(b)
            else:
                advance(c)
        raise Hazard("step bound exceeded")


def ring_reader(sim, ring, k, R):
    """Waits for ring entry k, reads it and releases it (one arrival)."""
    yield wait(f"ring_full{k % R}", k // R)
    it = ring[k % R]
    sim.arrive(f"ring_empty{k % R}")
    return it


# ----------------------------------------------------------------------------
# forward (fm_fwd_kernel): producer, MMA, two softmax groups that also write O
# ----------------------------------------------------------------------------
def fwd_model(items, seed, R=4, SLOTS=5):
    sim = Sim(seed)
    for i in range(R):
        sim.bar(f"ring_full{i}")
        sim.bar(f"ring_empty{i}", 1 + 2)  # MMA + the two softmax groups
    for nm in ("q_full", "q_empty"):
        sim.bar(nm)
    for i in range(SLOTS):
        sim.bar(f"slot_full{i}")
        sim.bar(f"slot_empty{i}")
    for g in range(2):
        for nm in ("s_full", "o_full", "p_full", "o_free"):
            sim.bar(f"{nm}{g}")
    ring = [None] * R
    st = {"slot": [None] * SLOTS, "q": None, "S": [None, None], "O": ["free", "free"]}
    seq = list(items) + [None]

    def producer():
        k, nxt_i, pos, act = 0, 0, 0, 0

        def take():
            nonlocal k, nxt_i
            yield wait(f"ring_empty{k % R}", k // R - 1)
            it = seq[nxt_i] if nxt_i < len(seq) else None
            nxt_i += 1
            ring[k % R] = it
            sim.arrive(f"ring_full{k % R}")
            k += 1
            return it

        nxt = yield from take()  # items are taken one ahead
        while nxt is not None:
            it = nxt
            nxt = yield from take()
            j, n = it
            if n == 0:
                continue
            yield wait("q_empty", act - 1)
            sim.tma.append(("q_full", lambda j=j: st.__setitem__("q", j)))
            act += 1
            for t in range(n):
                for kv in range(2):
                    sl = pos % SLOTS
                    yield wait(f"slot_empty{sl}", pos // SLOTS - 1)
                    sim.tma.append((f"slot_full{sl}", lambda sl=sl, c=(j, t, kv): st["slot"].__setitem__(sl, c)))
                    pos += 1

    def op_s(g, j, t, sl):
        def f():
            if st["q"] != j or st["slot"][sl] != (j, t, 0):
                raise Hazard(f"S{g}({j},{t}): Q {st['q']} slot {st['slot'][sl]}")
            if st["S"][g] is not None and st["S"][g][0] != "used":
                raise Hazard(f"S{g}({j},{t}) overwrites {st['S'][g]}")
            st["S"][g] = ("S", j, t)
        return f

    def op_pv(g, j, t, sl):
        def f():
            if st["slot"][sl] != (j, t, 1) or st["S"][g] != ("P", j, t):
                raise Hazard(f"PV{g}({j},{t}): slot {st['slot'][sl]} S/P {st['S'][g]}")
            o = st["O"][g]
            if (t == 0 and o != "free") or (t > 0 and o != (j, t - 1)):
                raise Hazard(f"PV{g}({j},{t}): O holds {o}")
            st["S"][g] = ("used", j, t)
            st["O"][g] = (j, t)
        return f

    def mma():
        pos = tile = act = k = 0
        while True:
            it = yield from ring_reader(sim, ring, k, R)
            k += 1
            if it is None:
                return
            j, n = it
            if n == 0:
                continue
            yield wait("q_full", act)
            for t in range(n):
                sv, sk2 = (pos + 1) % SLOTS, (pos + 2) % SLOTS
                if t == 0:
                    sk = pos % SLOTS
                    yield wait(f"slot_full{sk}", pos // SLOTS)
                    for g in range(2):
                        sim.pipe += [("mma", op_s(g, j, 0, sk)), ("commit", f"s_full{g}")]
                    sim.pipe.append(("commit", f"slot_empty{sk}"))
                    if n == 1:
                        sim.pipe.append(("commit", "q_empty"))
                yield wait(f"slot_full{sv}", (pos + 1) // SLOTS)
                yield wait("p_full0", tile)
                if t == 0:
                    yield wait("o_free0", act - 1)
                sim.pipe.append(("mma", op_pv(0, j, t, sv)))
                if t == n - 1:
                    sim.pipe.append(("commit", "o_full0"))
                if t + 1 < n:
                    yield wait(f"slot_full{sk2}", (pos + 2) // SLOTS)
                    sim.pipe += [("mma", op_s(0, j, t + 1, sk2)), ("commit", "s_full0")]
                yield wait("p_full1", tile)
                if t == 0:
                    yield wait("o_free1", act - 1)
                sim.pipe.append(("mma", op_pv(1, j, t, sv)))
                if t == n - 1:
                    sim.pipe.append(("commit", "o_full1"))
                sim.pipe.append(("commit", f"slot_empty{sv}"))
                if t + 1 < n:
                    sim.pipe += [("mma", op_s(1, j, t + 1, sk2)), ("commit", "s_full1"),
                                 ("commit", f"slot_empty{sk2}")]
                    if t + 2 == n:
                        sim.pipe.append(("commit", "q_empty"))
                tile += 1
                pos += 2
            act += 1

    def softmax(g):
        tile = act = 0
        it = yield from ring_reader(sim, ring, 0, R)
        k = 1
        while it is not None:
            j, n = it
            for t in range(n):
                yield wait(f"s_full{g}", tile)
                if st["S"][g] != ("S", j, t):
                    raise Hazard(f"softmax{g}({j},{t}): S holds {st['S'][g]}")
                if t > 0 and sim.rng.random() < 0.3 and st["O"][g] != (j, t - 1):  # lazy O rescale
                    raise Hazard(f"softmax{g}({j},{t}) rescale: O holds {st['O'][g]}")
                yield STEP
                st["S"][g] = ("P", j, t)
                sim.arrive(f"p_full{g}")
                tile += 1
            it_next = yield from ring_reader(sim, ring, k, R)  # next item taken before the epilogue
            k += 1
            if n > 0:
                yield wait(f"o_full{g}", act)
                if st["O"][g] != (j, n - 1):
                    raise Hazard(f"softmax{g} epilogue({j}): O holds {st['O'][g]}")
                yield STEP
                st["O"][g] = "free"
                sim.arrive(f"o_free{g}")
                act += 1
            it = it_next

    sim.run({"producer": producer(), "mma": mma(), "softmax0": softmax(0), "softmax1": softmax(1)})


# ----------------------------------------------------------------------------
# backward, query side (fm_bwd_dq_kernel)
# ----------------------------------------------------------------------------
def dq_model(items, seed, R=4, KST=3, VST=2):
    sim = Sim(seed)
    for i in range(R):
        sim.bar(f"ring_full{i}")
        sim.bar(f"ring_empty{i}", 1 + 1 + 2)  # MMA + second producer + the two compute warpgroups
    for nm in ("q_full", "q_empty", "dp_full", "dq_full"):
        sim.bar(nm)
    for i in range(KST):
        sim.bar(f"k_full{i}")
        sim.bar(f"k_empty{i}")
    for i in range(VST):
        sim.bar(f"v_full{i}")
        sim.bar(f"v_empty{i}")
    for b in range(2):
        sim.bar(f"s_full{b}")
        sim.bar(f"ds_full{b}", 2)
    sim.bar("dp_read", 2)
    sim.bar("dq_free", 2)
    ring = [None] * R
    st = {"k": [None] * KST, "v": [None] * VST, "q": None, "S": [[None, None], [None, None]],
          "dP": None, "dP_read": [None, None], "dQ": "free", "dQ_read": [False, False]}
    seq = list(items) + [None]

    def producer():
        k = nxt_i = kv = act = 0

        def take():
            nonlocal k, nxt_i
            yield wait(f"ring_empty{k % R}", k // R - 1)
            it = seq[nxt_i] if nxt_i < len(seq) else None
            nxt_i += 1
            ring[k % R] = it
            sim.arrive(f"ring_full{k % R}")
            k += 1
            return it

        nxt = yield from take()
        while nxt is not None:
            it = nxt
            nxt = yield from take()
            j, n = it
            if n == 0:
                continue
            yield wait("q_empty", act - 1)
            sim.tma.append(("q_full", lambda j=j: st.__setitem__("q", j)))
            act += 1
            for t in range(n):
                s = kv % KST
                yield wait(f"k_empty{s}", kv // KST - 1)
                sim.tma.append((f"k_full{s}", lambda s=s, c=(j, t): st["k"].__setitem__(s, c)))
                kv += 1

    def producer2():
        kv = k = 0
        while True:
            it = yield from ring_reader(sim, ring, k, R)
            k += 1
            if it is None:
                return
            j, n = it
            for t in range(n):
                s = kv % VST
                yield wait(f"v_empty{s}", kv // VST - 1)
                sim.tma.append((f"v_full{s}", lambda s=s, c=(j, t): st["v"].__setitem__(s, c)))
                kv += 1

    def op_s(j, t, tj, ks):
        def f():
            if st["q"] != j or st["k"][ks] != (j, t):
                raise Hazard(f"S({j},{t}): Q {st['q']} K {st['k'][ks]}")
            b = tj & 1
            if any(h is not None and h[0] != "used" for h in st["S"][b]):
                raise Hazard(f"S({j},{t}) overwrites buffer {b}: {st['S'][b]}")
            st["S"][b] = [("S", tj), ("S", tj)]
        return f

    def op_dp(j, t, tj, vs):
        def f():
            if st["q"] != j or st["v"][vs] != (j, t):
                raise Hazard(f"dP({j},{t}): dO {st['q']} V {st['v'][vs]}")
            if st["dP"] is not None and st["dP_read"] != [st["dP"], st["dP"]]:
                raise Hazard(f"dP({j},{t}) overwrites dP {st['dP']} read by {st['dP_read']}")
            st["dP"] = tj
        return f

    def op_dq(j, t, tj, ks):
        def f():
            b = tj & 1
            if st["S"][b] != [("dS", tj), ("dS", tj)] or st["k"][ks] != (j, t):
                raise Hazard(f"dQ({j},{t}): dS {st['S'][b]} K {st['k'][ks]}")
            d = st["dQ"]
            if (t == 0 and d != "free") or (t > 0 and d != (j, t - 1)):
                raise Hazard(f"dQ({j},{t}): accumulator holds {d}")
            st["S"][b] = [("used", tj), ("used", tj)]
            st["dQ"] = (j, t)
        return f

    def mma():
        kv = tc = act = k = 0
        while True:
            it = yield from ring_reader(sim, ring, k, R)
            k += 1
            if it is None:
                return
            j, n = it
            if n == 0:
                continue
            yield wait("q_full", act)
            sk, sv = kv % KST, kv % VST
            yield wait(f"k_full{sk}", kv // KST)
            sim.pipe += [("mma", op_s(j, 0, tc, sk)), ("commit", f"s_full{tc & 1}")]
            yield wait(f"v_full{sv}", kv // VST)
            sim.pipe += [("mma", op_dp(j, 0, tc, sv)), ("commit", "dp_full"), ("commit", f"v_empty{sv}")]
            if n == 1:
                sim.pipe.append(("commit", "q_empty"))
            for t in range(n):
                kj, tj = kv + t, tc + t
                ks, ks2, vs2 = kj % KST, (kj + 1) % KST, (kj + 1) % VST
                if t + 1 < n:
                    yield wait(f"k_full{ks2}", (kj + 1) // KST)
                    sim.pipe += [("mma", op_s(j, t + 1, tj + 1, ks2)), ("commit", f"s_full{(tj + 1) & 1}")]
                    yield wait("dp_read", tj)
                    yield wait(f"v_full{vs2}", (kj + 1) // VST)
                    sim.pipe += [("mma", op_dp(j, t + 1, tj + 1, vs2)), ("commit", "dp_full"),
                                 ("commit", f"v_empty{vs2}")]
                    if t + 2 == n:
                        sim.pipe.append(("commit", "q_empty"))
                if t == 0:
                    yield wait("dq_free", act - 1)
                yield wait(f"ds_full{tj & 1}", tj >> 1)
                sim.pipe += [("mma", op_dq(j, t, tj, ks)), ("commit", f"k_empty{ks}")]
            kv += n
            tc += n
            act += 1
            sim.pipe.append(("commit", "dq_full"))

    def compute(h):
        tc = act = k = 0
        while True:
            it = yield from ring_reader(sim, ring, k, R)
            k += 1
            if it is None:
                return
            j, n = it
            if n == 0:  # dQ = 0 written directly
                continue
            for t in range(n):
                b = tc & 1
                yield wait(f"s_full{b}", tc >> 1)
                yield wait("dp_full", tc)
                if st["S"][b][h] != ("S", tc) or st["dP"] != tc:
                    raise Hazard(f"compute{h}({j},{t}): S {st['S'][b][h]} dP {st['dP']}")
                st["dP_read"][h] = tc
                sim.arrive("dp_read")
                yield STEP
                st["S"][b][h] = ("dS", tc)
                sim.arrive(f"ds_full{b}")
                tc += 1
            yield wait("dq_full", act)  # epilogue: this warpgroup's half of the dQ columns
            if st["dQ"] != (j, n - 1):
                raise Hazard(f"compute{h} epilogue({j}): accumulator holds {st['dQ']}")
            yield STEP
            st["dQ_read"][h] = True
            if all(st["dQ_read"]):
                st["dQ"], st["dQ_read"] = "free", [False, False]
            sim.arrive("dq_free")
            act += 1

    sim.run({"producer": producer(), "producer2": producer2(), "mma": mma(), "compute0": compute(0),
             "compute1": compute(1)})


# ----------------------------------------------------------------------------
# backward, key side (fm_bwd_dkdv_kernel)
# ----------------------------------------------------------------------------
def dkdv_model(items, seed, R=4, QST=3, DOST=2, LST=2):
    sim = Sim(seed)
    for i in range(R):
        sim.bar(f"ring_full{i}")
        sim.bar(f"ring_empty{i}", 1 + 1 + 2)  # MMA + second producer + the two compute warpgroups
    for nm in ("k_full", "k_empty", "v_full", "v_empty", "s_full", "dp_full", "dkdv_full"):
        sim.bar(nm)
    for nm in ("p_full", "ds_full", "dkdv_free"):
        sim.bar(nm, 2)
    for i in range(QST):
        sim.bar(f"q_full{i}")
        sim.bar(f"q_empty{i}")
    for i in range(DOST):
        sim.bar(f"do_full{i}")
        sim.bar(f"do_empty{i}")
    for i in range(LST):
        sim.bar(f"l_full{i}")
        sim.bar(f"l_empty{i}", 2)
    ring = [None] * R
    st = {"k": None, "v": None, "q": [None] * QST, "do": [None] * DOST, "l": [None] * LST,
          "S": [None, None], "dP": [None, None], "dV": "free", "dK": "free"}
    seq = list(items) + [None]

    def producer():  # publishes items (not one ahead), loads K and every q-tile's Q
        sq = act = k = 0
        for it in seq:
            yield wait(f"ring_empty{k % R}", k // R - 1)
            ring[k % R] = it
            sim.arrive(f"ring_full{k % R}")
            k += 1
            if it is None:
                return
            j, n = it
            if n == 0:
                continue
            yield wait("k_empty", act - 1)
            sim.tma.append(("k_full", lambda j=j: st.__setitem__("k", j)))
            act += 1
            for t in range(n):
                s = sq % QST
                yield wait(f"q_empty{s}", sq // QST - 1)
                sim.tma.append((f"q_full{s}", lambda s=s, c=(j, t): st["q"].__setitem__(s, c)))
                sq += 1

    def producer2():  # V, every q-tile's dO and LSE2 / D rows
        sq = act = k = 0
        while True:
            it = yield from ring_reader(sim, ring, k, R)
            k += 1
            if it is None:
                return
            j, n = it
            if n == 0:
                continue
            yield wait("v_empty", act - 1)
            sim.tma.append(("v_full", lambda j=j: st.__setitem__("v", j)))
            act += 1
            for t in range(n):
                s, l = sq % DOST, sq % LST
                yield wait(f"do_empty{s}", sq // DOST - 1)
                sim.tma.append((f"do_full{s}", lambda s=s, c=(j, t): st["do"].__setitem__(s, c)))
                yield wait(f"l_empty{l}", sq // LST - 1)
                sim.tma.append((f"l_full{l}", lambda l=l, c=(j, t): st["l"].__setitem__(l, c)))
                sq += 1

    def op_s(j, t, tj, qs):
        def f():
            if st["k"] != j or st["q"][qs] != (j, t):
                raise Hazard(f"S({j},{t}): K {st['k']} Q {st['q'][qs]}")
            if any(h is not None and h[0] != "used" for h in st["S"]):
                raise Hazard(f"S({j},{t}) overwrites {st['S']}")
            st["S"] = [("S", tj), ("S", tj)]
        return f

    def op_dp(j, t, tj, ds):
        def f():
            if st["v"] != j or st["do"][ds] != (j, t):
                raise Hazard(f"dP({j},{t}): V {st['v']} dO {st['do'][ds]}")
            if any(h is not None and h[0] != "used" for h in st["dP"]):
                raise Hazard(f"dP({j},{t}) overwrites {st['dP']}")
            st["dP"] = [("dP", tj), ("dP", tj)]
        return f

    def op_dv(j, t, tj, ds):
        def f():
            if st["S"] != [("P", tj), ("P", tj)] or st["do"][ds] != (j, t):
                raise Hazard(f"dV({j},{t}): P {st['S']} dO {st['do'][ds]}")
            a = st["dV"]
            if (t == 0 and a != "free") or (t > 0 and a != (j, t - 1)):
                raise Hazard(f"dV({j},{t}): accumulator holds {a}")
            st["S"] = [("used", tj), ("used", tj)]
            st["dV"] = (j, t)
        return f

    def op_dk(j, t, tj, qs):
        def f():
            if st["dP"] != [("dS", tj), ("dS", tj)] or st["q"][qs] != (j, t):
                raise Hazard(f"dK({j},{t}): dS {st['dP']} Q {st['q'][qs]}")
            a = st["dK"]
            if (t == 0 and a != "free") or (t > 0 and a != (j, t - 1)):
                raise Hazard(f"dK({j},{t}): accumulator holds {a}")
            st["dP"] = [("used", tj), ("used", tj)]
            st["dK"] = (j, t)
        return f

    def mma():
        sq = tc = act = k = 0
        while True:
            it = yield from ring_reader(sim, ring, k, R)
            k += 1
            if it is None:
                return
            j, n = it
            if n == 0:
                continue
            qs, ds = sq % QST, sq % DOST
            yield wait("k_full", act)
            yield wait(f"q_full{qs}", sq // QST)
            sim.pipe += [("mma", op_s(j, 0, tc, qs)), ("commit", "s_full")]
            if n == 1:
                sim.pipe.append(("commit", "k_empty"))
            yield wait("v_full", act)
            yield wait(f"do_full{ds}", sq // DOST)
            sim.pipe += [("mma", op_dp(j, 0, tc, ds)), ("commit", "dp_full")]
            if n == 1:
                sim.pipe.append(("commit", "v_empty"))
            for t in range(n):
                sj, tj = sq + t, tc + t
                qs, ds = sj % QST, sj % DOST
                qs2, ds2 = (sj + 1) % QST, (sj + 1) % DOST
                if t == 0:
                    yield wait("dkdv_free", act - 1)
                yield wait("p_full", tj)
                sim.pipe += [("mma", op_dv(j, t, tj, ds)), ("commit", f"do_empty{ds}")]
                if t + 1 < n:
                    yield wait(f"q_full{qs2}", (sj + 1) // QST)
                    sim.pipe += [("mma", op_s(j, t + 1, tj + 1, qs2)), ("commit", "s_full")]
                    if t + 2 == n:
                        sim.pipe.append(("commit", "k_empty"))
                yield wait("ds_full", tj)
                sim.pipe += [("mma", op_dk(j, t, tj, qs)), ("commit", f"q_empty{qs}")]
                if t + 1 < n:
                    yield wait(f"do_full{ds2}", (sj + 1) // DOST)
                    sim.pipe += [("mma", op_dp(j, t + 1, tj + 1, ds2)), ("commit", "dp_full")]
                    if t + 2 == n:
                        sim.pipe.append(("commit", "v_empty"))
            sq += n
            tc += n
            act += 1
            sim.pipe.append(("commit", "dkdv_full"))

    def compute(h):
        sq = tc = act = k = 0
        while True:
            it = yield from ring_reader(sim, ring, k, R)
            k += 1
            if it is None:
                return
            j, n = it
            if n == 0:  # dK = dV = 0 written directly
                continue
            for t in range(n):
                l = sq % LST
                yield wait("s_full", tc)
                yield wait(f"l_full{l}", sq // LST)
                if st["S"][h] != ("S", tc) or st["l"][l] != (j, t):
                    raise Hazard(f"compute{h}({j},{t}): S {st['S'][h]} rows {st['l'][l]}")
                yield STEP
                st["S"][h] = ("P", tc)
                sim.arrive("p_full")
                yield wait("dp_full", tc)
                if st["dP"][h] != ("dP", tc):
                    raise Hazard(f"compute{h}({j},{t}): dP {st['dP'][h]}")
                yield STEP
                st["dP"][h] = ("dS", tc)
                sim.arrive("ds_full")
                sim.arrive(f"l_empty{l}")
                sq += 1
                tc += 1
            yield wait("dkdv_full", act)  # warpgroup 0 writes dV, warpgroup 1 dK
            acc = "dV" if h == 0 else "dK"
            if st[acc] != (j, n - 1):
                raise Hazard(f"compute{h} epilogue({j}): {acc} holds {st[acc]}")
            yield STEP
            st[acc] = "free"
            sim.arrive("dkdv_free")
            act += 1

    sim.run({"producer": producer(), "producer2": producer2(), "mma": mma(), "compute0": compute(0),
             "compute1": compute(1)})


# ----------------------------------------------------------------------------
# fused backward (fm_bwd_fused_kernel): dkdv's roles plus dQ(t) = dS K into the
# dP^T region, read out by the compute warpgroups between the halves of P^T(t+1)
# ----------------------------------------------------------------------------
def fused_model(items, seed, R=4, QST=2, DOST=1, LST=2):
    sim = Sim(seed)
    for i in range(R):
        sim.bar(f"ring_full{i}")
        sim.bar(f"ring_empty{i}", 1 + 1 + 2 + 1)  # MMA + second producer + two compute warpgroups + drain
    for nm in ("k_full", "k_empty", "v_full", "v_empty", "s_full", "dp_full", "dq_full", "dkdv_full"):
        sim.bar(nm)
    for nm in ("p_full", "ds_full", "dkdv_free"):  # the two compute warpgroups
        sim.bar(nm, 2)
    sim.bar("dq_free", 1)  # the drain warpgroup
    for nm in ("staged", "dsbuf_free", "buf_free"):
        sim.bar(nm)
    for i in range(QST):
        sim.bar(f"q_full{i}")
        sim.bar(f"q_empty{i}")
    for i in range(DOST):
        sim.bar(f"do_full{i}")
        sim.bar(f"do_empty{i}")
    for i in range(LST):
        sim.bar(f"l_full{i}")
        sim.bar(f"l_empty{i}", 2)
    ring = [None] * R
    st = {"k": None, "v": None, "q": [None] * QST, "do": [None] * DOST, "l": [None] * LST,
          "S": [None, None], "dP": [None, None], "dsm": [None, None], "stage": None, "dV": "free", "dK": "free"}
    seq = list(items) + [None]

    def producer():  # K and every q-tile's Q; K is freed after the item's last dQ
        sq = act = k = 0
        for it in seq:
            yield wait(f"ring_empty{k % R}", k // R - 1)
            ring[k % R] = it
            sim.arrive(f"ring_full{k % R}")
            k += 1
            if it is None:
                return
            j, n = it
            if n == 0:
                continue
            yield wait("k_empty", act - 1)
            sim.tma.append(("k_full", lambda j=j: st.__setitem__("k", j)))
            act += 1
            for t in range(n):
                s = sq % QST
                yield wait(f"q_empty{s}", sq // QST - 1)
                sim.tma.append((f"q_full{s}", lambda s=s, c=(j, t): st["q"].__setitem__(s, c)))
                sq += 1

    def producer2():  # V, every q-tile's dO and LSE2 / D rows
        sq = act = k = 0
        while True:
            it = yield from ring_reader(sim, ring, k, R)
            k += 1
            if it is None:
                return
            j, n = it
            if n == 0:
                continue
            yield wait("v_empty", act - 1)
            sim.tma.append(("v_full", lambda j=j: st.__setitem__("v", j)))
            act += 1
            for t in range(n):
                s, l = sq % DOST, sq % LST
                yield wait(f"do_empty{s}", sq // DOST - 1)
                sim.tma.append((f"do_full{s}", lambda s=s, c=(j, t): st["do"].__setitem__(s, c)))
                yield wait(f"l_empty{l}", sq // LST - 1)
                sim.tma.append((f"l_full{l}", lambda l=l, c=(j, t): st["l"].__setitem__(l, c)))
                sq += 1

    def op_s(j, t, tj, qs):
        def f():
            if st["k"] != j or st["q"][qs] != (j, t):
                raise Hazard(f"S({j},{t}): K {st['k']} Q {st['q'][qs]}")
            if any(h is not None and h[0] != "used" for h in st["S"]):
                raise Hazard(f"S({j},{t}) overwrites {st['S']}")
            st["S"] = [("S", tj), ("S", tj)]
        return f

    def op_dp(j, t, tj, ds):
        def f():
            if st["v"] != j or st["do"][ds] != (j, t):
                raise Hazard(f"dP({j},{t}): V {st['v']} dO {st['do'][ds]}")
            if any(h is not None and h[0] != "used" for h in st["dP"]):
                raise Hazard(f"dP({j},{t}) overwrites {st['dP']}")
            st["dP"] = [("dP", tj), ("dP", tj)]
        return f

    def op_dv(j, t, tj, ds):
        def f():
            if st["S"] != [("P", tj), ("P", tj)] or st["do"][ds] != (j, t):
                raise Hazard(f"dV({j},{t}): P {st['S']} dO {st['do'][ds]}")
            a = st["dV"]
            if (t == 0 and a != "free") or (t > 0 and a != (j, t - 1)):
                raise Hazard(f"dV({j},{t}): accumulator holds {a}")
            st["S"] = [("used", tj), ("used", tj)]
            st["dV"] = (j, t)
        return f

    def op_dk(j, t, tj, qs):
        def f():
            if st["dP"] != [("dS", tj), ("dS", tj)] or st["q"][qs] != (j, t):
                raise Hazard(f"dK({j},{t}): dS {st['dP']} Q {st['q'][qs]}")
            a = st["dK"]
            if (t == 0 and a != "free") or (t > 0 and a != (j, t - 1)):
                raise Hazard(f"dK({j},{t}): accumulator holds {a}")
            st["dP"] = [("read", tj), ("read", tj)]
            st["dK"] = (j, t)
        return f

    def op_dq(j, t, tj):
        def f():
            if st["k"] != j or st["dsm"] != [("dS", tj), ("dS", tj)]:
                raise Hazard(f"dQ({j},{t}): K {st['k']} dS {st['dsm']}")
            if st["dP"] != [("read", tj), ("read", tj)]:
                raise Hazard(f"dQ({j},{t}) overwrites {st['dP']}")
            st["dsm"] = [("used", tj), ("used", tj)]
            st["dP"] = [("dQ", tj), ("dQ", tj)]
        return f

    def mma():
        sq = tc = act = k = 0
        while True:
            it = yield from ring_reader(sim, ring, k, R)
            k += 1
            if it is None:
                return
            j, n = it
            if n == 0:
                continue
            qs, ds = sq % QST, sq % DOST
            yield wait("k_full", act)
            yield wait(f"q_full{qs}", sq // QST)
            sim.pipe += [("mma", op_s(j, 0, tc, qs)), ("commit", "s_full")]
            yield wait("v_full", act)
            yield wait(f"do_full{ds}", sq // DOST)
            if tc > 0:
                yield wait("dq_free", tc - 1)
            sim.pipe += [("mma", op_dp(j, 0, tc, ds)), ("commit", "dp_full")]
            if n == 1:
                sim.pipe.append(("commit", "v_empty"))
            for t in range(n):
                sj, tj = sq + t, tc + t
                qs, ds = sj % QST, sj % DOST
                qs2, ds2 = (sj + 1) % QST, (sj + 1) % DOST
                if t == 0:
                    yield wait("dkdv_free", act - 1)
                yield wait("p_full", tj)
                sim.pipe += [("mma", op_dv(j, t, tj, ds)), ("commit", f"do_empty{ds}")]
                if t + 1 < n:
                    yield wait(f"q_full{qs2}", (sj + 1) // QST)
                    sim.pipe += [("mma", op_s(j, t + 1, tj + 1, qs2)), ("commit", "s_full")]
                yield wait("ds_full", tj)
                sim.pipe += [("mma", op_dk(j, t, tj, qs)), ("commit", f"q_empty{qs}")]
                sim.pipe += [("mma", op_dq(j, t, tj)), ("commit", "dq_full")]
                if t + 1 == n:
                    sim.pipe.append(("commit", "k_empty"))
                if t + 1 < n:
                    yield wait("dq_free", tj)
                    yield wait(f"do_full{ds2}", (sj + 1) // DOST)
                    sim.pipe += [("mma", op_dp(j, t + 1, tj + 1, ds2)), ("commit", "dp_full")]
                    if t + 2 == n:
                        sim.pipe.append(("commit", "v_empty"))
            sq += n
            tc += n
            act += 1
            sim.pipe.append(("commit", "dkdv_full"))  # after the item's last dK and dQ

    def compute(h):
        sq = tc = act = k = 0
        while True:
            it = yield from ring_reader(sim, ring, k, R)
            k += 1
            if it is None:
                return
            j, n = it
            if n == 0:  # dK = dV = 0 written directly
                continue
            for t in range(n):
                l = sq % LST
                yield wait("s_full", tc)
                yield wait(f"l_full{l}", sq // LST)
                if st["S"][h] != ("S", tc) or st["l"][l] != (j, t):
                    raise Hazard(f"compute{h}({j},{t}): S {st['S'][h]} rows {st['l'][l]}")
                yield STEP  # P^T
                st["S"][h] = ("P", tc)
                sim.arrive("p_full")
                yield wait("dp_full", tc)
                if st["dP"][h] != ("dP", tc):
                    raise Hazard(f"compute{h}({j},{t}): dP {st['dP'][h]}")
                if tc > 0:
                    yield wait("dsbuf_free", tc - 1)  # the reduction has read dQ(tc-1) staged there
                if st["dsm"][h] is not None and st["dsm"][h][0] != "free":
                    raise Hazard(f"compute{h}({j},{t}): dS buffer still holds {st['dsm'][h]}")
                yield STEP
                st["dP"][h] = ("dS", tc)
                st["dsm"][h] = ("dS", tc)
                sim.arrive("ds_full")
                sim.arrive(f"l_empty{l}")
                sq += 1
                tc += 1
            yield wait("dkdv_full", act)  # warpgroup 0 writes dV, warpgroup 1 dK
            acc = "dV" if h == 0 else "dK"
            if st[acc] != (j, n - 1):
                raise Hazard(f"compute{h} epilogue({j}): {acc} holds {st[acc]}")
            yield STEP
            st[acc] = "free"
            sim.arrive("dkdv_free")
            act += 1

    def drain():  # dQ(t): TMEM -> the dS buffer (cols 0-63) and the staging buffer
        tc = k = 0
        while True:
            it = yield from ring_reader(sim, ring, k, R)
            k += 1
            if it is None:
                return
            j, n = it
            for t in range(n):
                if tc > 0:
                    yield wait("buf_free", tc - 1)
                yield wait("dq_full", tc)
                if st["dP"] != [("dQ", tc), ("dQ", tc)]:
                    raise Hazard(f"drain({j},{t}): dP region holds {st['dP']}")
                if st["dsm"] != [("used", tc), ("used", tc)]:
                    raise Hazard(f"drain({j},{t}): dS buffer holds {st['dsm']}")
                if st["stage"] is not None and st["stage"][0] != "free":
                    raise Hazard(f"drain({j},{t}): staging buffer holds {st['stage']}")
                yield STEP
                st["dP"] = [("used", tc), ("used", tc)]
                sim.arrive("dq_free")
                st["dsm"] = [("dQ", tc), ("dQ", tc)]
                st["stage"] = ("dQ", tc)
                sim.arrive("staged")
                tc += 1

    def reducer():  # the drain warpgroup's elected thread: the bulk reductions read both buffers
        tc = 0
        total = sum(n for _, n in items)
        while tc < total:
            yield wait("staged", tc)
            if st["dsm"] != [("dQ", tc), ("dQ", tc)] or st["stage"] != ("dQ", tc):
                raise Hazard(f"reducer({tc}): buffers hold {st['dsm']} / {st['stage']}")
            yield STEP
            st["dsm"] = [("free", tc), ("free", tc)]
            sim.arrive("dsbuf_free")
            yield STEP
            st["stage"] = ("free", tc)
            sim.arrive("buf_free")
            tc += 1

    sim.run({"producer": producer(), "producer2": producer2(), "mma": mma(), "compute0": compute(0),
             "compute1": compute(1), "drain": drain(), "reducer": reducer()})


MODELS = {"fwd": fwd_model, "dq": dq_model, "dkdv": dkdv_model, "fused": fused_model}


def random_items(rng):
    """A work sequence: item j with n non-skipped tiles (0 = an item whose tiles are all skipped)."""
    return [(j, rng.choice([0, 1, 1, 2, 2, 3, 5])) for j in range(rng.randrange(0, 9))]
