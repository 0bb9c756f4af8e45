"""Discrete-event model of the mbarrier protocol of the tensor-core attention kernel
(prefix_shared_attention_b200/csrc/bat_attn_tc.cu), for the deadlock test.

Each role of one CTA is a generator that yields ("wait", barrier, parity) whenever the kernel
waits on an mbarrier phase, and performs the kernel's arrivals, expect-tx and commits as
plain calls.  Asynchronous completions are modelled as queues: every MMA issuer's tcgen05
operations complete in issue order (a commit arrives once everything issued before it by that
issuer has completed), TMA loads complete in any order.  The scheduler runs every runnable
role, then completes one random pending operation; if no role can run and nothing is in
flight, the protocol has deadlocked.  The roles follow the kernel:

  producer     pops work items from the global list into the item queue; with two rings it
               loads the Q tiles, then the K tiles into the K ring; with one ring it loads the
               K and V tiles into the shared ring in consumption order K0, K1, V0, K2, V1, ...
  vproducer    (two rings) pops the items and loads the V tiles into the V ring
  qproducer    (one ring) pops the items and loads the Q tiles
  mma X        walks the tiles in consumption order: S of key tile j+1 (K slot landed,
               Q landed for the first S, the softmax has read the previous S), then PV of
               tile j (V slot landed, P written, per P half); frees each slot by a commit or,
               for a tile query tile X does not read, a plain arrive.  A V tile whose valid
               keys end inside a 16-key step has its tail rows zeroed by its lower-numbered
               consumer, which arrives on the slot's v_zeroed barrier when both tiles read it;
               the other consumer waits for that barrier
  softmax X    per tile: S landed -> s_free; optionally (data dependent) waits for the last
               PV before rescaling O; per P half: waits for the previous tile's PV of that
               half, writes P, p_full; after the item: waits for the last PV (epilogue)
"""

from __future__ import annotations

import random

TILE = 128
ITEM_QUEUE = 4


class Bar:
    def __init__(self, name, count):
        self.name, self.count, self.pending, self.tx, self.phase = name, count, count, 0, 0

    def arrive(self, n=1):
        self.pending -= n
        assert self.pending >= 0, f"{self.name}: more arrivals than its count"
        self._advance()

    def expect_tx(self, nbytes):
        self.tx += nbytes
        self.arrive()

    def complete_tx(self, nbytes):
        self.tx -= nbytes
        assert self.tx >= 0, f"{self.name}: transaction count below zero"
        self._advance()

    def _advance(self):
        if self.pending == 0 and self.tx == 0:
            self.phase += 1
            self.pending = self.count

    def done(self, parity):
        """mbarrier.try_wait.parity: true once the phase with this parity has completed."""
        return (self.phase & 1) != parity


class Stream:
    """The key tiles of one work item: prefix tiles, then suffix tiles (shared, or A and B
    interleaved then the longer one's rest), with the mask of query tiles that read each."""

    def __init__(self, w):
        cd = lambda a: (int(a) + TILE - 1) // TILE
        self.nq = int(w["n_q"])
        self.shared = bool(w["shared"]) or self.nq == 1
        self.npre = cd(w["pre_len"])
        self.nsA = cd(w["sA_len"])
        self.nsB = 0 if self.shared else cd(w["sB_len"])
        self.n = self.npre + self.nsA + self.nsB
        self.w = w

    def valid(self, j):
        """Valid keys of global tile j."""
        w = self.w
        if j < self.npre:
            return min(TILE, int(w["pre_len"]) - j * TILE)
        k = j - self.npre
        if self.shared:
            return min(TILE, int(w["sA_len"]) - k * TILE)
        mm = min(self.nsA, self.nsB)
        x = (k & 1) if k < 2 * mm else (0 if self.nsA > self.nsB else 1)
        idx = (k >> 1) if k < 2 * mm else mm + (k - 2 * mm)
        return min(TILE, int(w["sB_len" if x else "sA_len"]) - idx * TILE)

    def count(self, x):
        return self.npre + (self.nsA if (self.shared or x == 0) else self.nsB)

    def mask(self, j):
        if j < self.npre or self.shared:
            return 3 if self.nq == 2 else 1
        k = j - self.npre
        mm = min(self.nsA, self.nsB)
        x = (k & 1) if k < 2 * mm else (0 if self.nsA > self.nsB else 1)
        return 1 << x

    def order(self):
        """Consumption order of the item's loads: (tile, is_v)."""
        out = [(0, False)]
        for j in range(self.n):
            if j + 1 < self.n:
                out.append((j + 1, False))
            out.append((j, True))
        return out


def simulate(items, two_rings: bool, k_stages: int, v_stages: int, shared_stages: int, pv_halves: int,
             seed: int = 0, max_steps: int = 5_000_000) -> str:
    """Runs one CTA over `items` (records with n_q, shared, pre_len, sA_len, sB_len).
    Returns "ok" or a description of the deadlock."""
    rng = random.Random(seed)
    mma_q = [[], []]    # per issuer: ("mma",) or ("commit", bar), completed in order
    tma_q = []          # (bar, bytes), completed in any order

    def ring(name, n, empty_count):
        return [Bar(f"{name}_full{i}", 1) for i in range(n)], [Bar(f"{name}_empty{i}", empty_count) for i in range(n)]

    if two_rings:
        k_full, k_empty = ring("k", k_stages, 2)
        v_full, v_empty = ring("v", v_stages, 2)
        v_zeroed = [Bar(f"v_zeroed{i}", 1) for i in range(v_stages)]
    else:
        kv_full, kv_empty = ring("kv", shared_stages, 2)
        v_zeroed = [Bar(f"v_zeroed{i}", 1) for i in range(shared_stages)]
    bars = {n: [Bar(f"{n}{x}", c) for x in range(k)] for n, c, k in (
        ("q_full", 1, 2), ("q_empty", 1, 2), ("s_full", 1, 2), ("s_free", 128, 2), ("p_full", 128, 4),
        ("pv_done", 1, 4))}
    consumers = 2 + 8 + 1                                 # MMA issuers, softmax warps, V or Q producer
    itq_full = [Bar(f"itq_full{i}", 1) for i in range(ITEM_QUEUE)]
    itq_empty = [Bar(f"itq_empty{i}", consumers) for i in range(ITEM_QUEUE)]
    itq = [None] * ITEM_QUEUE

    def slot(r, full, empty):
        n = len(full)
        return full[r % n], empty[r % n], (r // n) & 1

    def pop(arrivals):
        k = 0
        while True:
            s = k % ITEM_QUEUE
            yield ("wait", itq_full[s], (k // ITEM_QUEUE) & 1)
            w = itq[s]
            itq_empty[s].arrive(arrivals)
            k += 1
            yield ("item", w)
            if w is None:
                return

    def load(full, empty, r):
        f, e, ph = slot(r, full, empty)
        yield ("wait", e, ph ^ 1)
        f.expect_tx(1)
        tma_q.append((f, 1))

    def producer():
        k, qcnt, r = 0, [0, 0], 0
        for w in list(items) + [None]:
            s = k % ITEM_QUEUE
            yield ("wait", itq_empty[s], ((k // ITEM_QUEUE) & 1) ^ 1)
            itq[s] = w
            itq_full[s].arrive()
            k += 1
            if w is None:
                return
            for x in range(int(w["n_q"]) if two_rings else 0):
                yield ("wait", bars["q_empty"][x], (qcnt[x] & 1) ^ 1)
                bars["q_full"][x].expect_tx(1)
                tma_q.append((bars["q_full"][x], 1))
                qcnt[x] += 1
            st = Stream(w)
            if two_rings:
                for _ in range(st.n):
                    yield from load(k_full, k_empty, r)
                    r += 1
            else:
                for _ in st.order():
                    yield from load(kv_full, kv_empty, r)
                    r += 1

    def vproducer():
        r = 0
        for ev in pop(1):
            if ev[0] != "item":
                yield ev
                continue
            if ev[1] is None:
                return
            for _ in range(Stream(ev[1]).n):
                yield from load(v_full, v_empty, r)
                r += 1

    def qproducer():
        qcnt = [0, 0]
        for ev in pop(1):
            if ev[0] != "item":
                yield ev
                continue
            if ev[1] is None:
                return
            for x in range(int(ev[1]["n_q"])):
                yield ("wait", bars["q_empty"][x], (qcnt[x] & 1) ^ 1)
                bars["q_full"][x].expect_tx(1)
                tma_q.append((bars["q_full"][x], 1))
                qcnt[x] += 1

    def mma(X):
        q = mma_q[X]
        kr = vr = r = 0
        qcnt = s_issued = p_seen = 0
        vz_par = [0] * len(v_zeroed)
        for ev in pop(1):
            if ev[0] != "item":
                yield ev
                continue
            w = ev[1]
            if w is None:
                return
            st = Stream(w)
            mine = X < st.nq
            s_left = st.count(X) if mine else 0
            first_s = True
            for j, is_v in st.order():
                if two_rings:
                    if is_v:
                        f, e, ph = slot(vr, v_full, v_empty)
                        zs = vr % len(v_full)
                        vr += 1
                    else:
                        f, e, ph = slot(kr, k_full, k_empty)
                        kr += 1
                else:
                    f, e, ph = slot(r, kv_full, kv_empty)
                    zs = r % len(kv_full)
                    r += 1
                yield ("wait", f, ph)
                if not mine or not ((st.mask(j) >> X) & 1):
                    e.arrive()
                    continue
                if not is_v:
                    if first_s:
                        yield ("wait", bars["q_full"][X], qcnt & 1)
                        qcnt += 1
                        first_s = False
                    if s_issued > 0:
                        yield ("wait", bars["s_free"][X], (s_issued - 1) & 1)
                    q += [("mma",), ("commit", bars["s_full"][X])]
                    if s_left == 1:
                        q.append(("commit", bars["q_empty"][X]))
                    q.append(("commit", e))
                    s_left -= 1
                    s_issued += 1
                else:
                    mask = st.mask(j)
                    if st.valid(j) % 16:
                        if X == (0 if mask & 1 else 1):
                            if mask == 3:
                                v_zeroed[zs].arrive()
                        else:
                            yield ("wait", v_zeroed[zs], vz_par[zs])
                        if mask == 3:
                            vz_par[zs] ^= 1
                    for h in range(2 - pv_halves, 2):
                        yield ("wait", bars["p_full"][2 * X + h], p_seen & 1)
                        q += [("mma",), ("commit", bars["pv_done"][2 * X + h])]
                    p_seen += 1
                    q.append(("commit", e))

    def softmax(X):
        s_seen = pv_base = 0
        for ev in pop(4):                                  # four warps per query tile
            if ev[0] != "item":
                yield ev
                continue
            w = ev[1]
            if w is None:
                return
            st = Stream(w)
            if X >= st.nq:
                continue
            n = st.count(X)
            for t in range(n):
                yield ("wait", bars["s_full"][X], s_seen & 1)
                s_seen += 1
                bars["s_free"][X].arrive(128)
                if t > 0 and rng.random() < 0.3:           # a row's maximum grew: rescale O
                    yield ("wait", bars["pv_done"][2 * X + 1], (pv_base + t - 1) & 1)
                for h in range(2):
                    if t > 0 and (pv_halves == 2 or h == 0):
                        yield ("wait", bars["pv_done"][2 * X + (h if pv_halves == 2 else 1)], (pv_base + t - 1) & 1)
                    if pv_halves == 2 or h == 1:
                        bars["p_full"][2 * X + h].arrive(128)
            yield ("wait", bars["pv_done"][2 * X + 1], (pv_base + n - 1) & 1)
            pv_base += n

    roles = {"producer": producer(), "mma0": mma(0), "mma1": mma(1), "softmax0": softmax(0), "softmax1": softmax(1)}
    roles["vproducer" if two_rings else "qproducer"] = vproducer() if two_rings else qproducer()
    waiting = {k: None for k in roles}
    done = set()
    for _ in range(max_steps):
        if len(done) == len(roles):
            return "ok"
        progressed = False
        for name, gen in roles.items():
            if name in done:
                continue
            cond = waiting[name]
            if cond is not None and not cond[1].done(cond[2]):
                continue
            while True:
                try:
                    ev = next(gen)
                except StopIteration:
                    done.add(name)
                    break
                if ev[0] == "wait":
                    waiting[name] = ev
                    break
            progressed = True
        live = [q for q in mma_q if q]
        if live or tma_q:
            if live and (not tma_q or rng.random() < 0.5):
                op = rng.choice(live).pop(0)
                if op[0] == "commit":
                    op[1].arrive()
            else:
                b, n = tma_q.pop(rng.randrange(len(tma_q)))
                b.complete_tx(n)
            progressed = True
        if not progressed:
            stuck = {k: f"{v[1].name} parity {v[2]}" for k, v in waiting.items() if k not in done and v}
            return f"deadlock: {stuck}"
    return "step limit reached"
