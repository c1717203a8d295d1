"""Host-side model of the persistent prefill kernel's synchronisation protocol.

fa_prefill_persist_kernel runs four kinds of roles in one CTA (TMA producer,
MMA thread, eight softmax warps, two E4M3 converter warps) that hand tiles to
each other through mbarriers waited on by phase parity.  With paged K/V the
producer also hands over the V tile of a request's last, partly filled page
only after zeroing its rows past the cache end (`tails`).  A mistake in that
protocol shows up on the GPU as a hang (bounded by the kernels' wait limits),
a stale tile or a wrong output; this model finds such mistakes on the host.

Each role is a Python generator that issues the same waits, arrivals,
commits, copies and MMAs as the kernel, in the same order and with the same
phase counters.  The simulator gives them random durations and checks:

  * every role finishes (no deadlock);
  * a parity wait never targets a phase other than the next one to complete
    (parity aliasing would let it pass early or late on the hardware);
  * every read finds the content it expects, already landed; no write (TMA,
    MMA or shared-memory store) lands on content that is still being read;
  * a queue entry is released (its item_empty phase completes) only after
    every consumer has read it;
  * an O accumulator is overwritten (first P V of an item) only after the
    epilogue of the previous item has read it.

`mutation` plants one protocol mistake, so tests can check the model
catches it.
"""
from __future__ import annotations

import heapq
import random


class ProtocolError(RuntimeError):
    pass


class _Bar:
    def __init__(self, count):
        self.count = count
        self.pending = count
        self.tx = 0
        self.completed = 0

    def try_complete(self):
        if self.pending == 0 and self.tx == 0:
            self.completed += 1
            self.pending = self.count
            return True
        return False


class _Sim:
    def __init__(self, seed):
        self.rng = random.Random(seed)
        self.t = 0.0
        self.events = []
        self.seq = 0
        self.bars = {}
        self.content = {}      # resource -> (tag, time it landed)
        self.readers = {}      # resource -> [(tag, end of read)]
        self.mma_end = 0.0
        self.blocked = {}      # role -> (barrier, phase)
        self.roles = {}
        self.finished = set()
        self.on_complete = {}  # barrier -> check run when one of its phases completes

    def err(self, msg):
        raise ProtocolError(f"t={self.t:.2f}: {msg}")

    def bar(self, name, count=1):
        self.bars[name] = _Bar(count)

    def at(self, t, fn):
        self.seq += 1
        heapq.heappush(self.events, (t, self.seq, fn))

    def arrive(self, name):
        b = self.bars[name]
        b.pending -= 1
        if b.pending < 0:
            self.err(f"more arrivals than expected on {name}")
        if b.try_complete():
            if name in self.on_complete:
                self.on_complete[name]()
            self._wake(name)

    def complete_tx(self, name, nbytes):
        b = self.bars[name]
        b.tx -= nbytes
        if b.try_complete():
            self._wake(name)

    def _passes(self, name, phase):
        """Parity wait for `phase`; checks that no other phase can alias it."""
        b = self.bars[name]
        passes = (b.completed & 1) != (phase & 1)
        if passes and b.completed != phase + 1:
            self.err(f"parity wait on {name} for phase {phase} passes with {b.completed} phases done")
        return passes

    def _wake(self, name):
        for role, (bn, phase) in list(self.blocked.items()):
            if bn == name and self._passes(bn, phase):
                del self.blocked[role]
                self.at(self.t, lambda r=role: self._step(r))

    def write(self, res, tag, landed):
        for rtag, rend in self.readers.get(res, []):
            if rend > self.t + 1e-9:
                self.err(f"{tag} written to {res} while {rtag} is read until {rend:.2f}")
        self.content[res] = (tag, landed)

    def read(self, res, tag, end):
        cur = self.content.get(res)
        if cur is None or cur[0] != tag:
            self.err(f"{res}: expected {tag}, found {cur and cur[0]}")
        if cur[1] > self.t + 1e-9:
            self.err(f"{res}: {tag} read before it landed")
        self.readers.setdefault(res, []).append((tag, end))

    def add_role(self, name, gen):
        self.roles[name] = gen
        self.at(0.0, lambda: self._step(name))

    def _step(self, role):
        gen = self.roles[role]
        while True:
            try:
                op = next(gen)
            except StopIteration:
                self.finished.add(role)
                return
            kind = op[0]
            if kind == "wait":
                if self._passes(op[1], op[2]):
                    continue
                self.blocked[role] = (op[1], op[2])
                return
            if kind == "delay":
                self.at(self.t + op[1], lambda: self._step(role))
                return
            if kind == "arrive":
                self.arrive(op[1])
            elif kind == "expect_tx":          # mbarrier.arrive.expect_tx
                self.bars[op[1]].tx += op[2]
                self.arrive(op[1])
            elif kind == "tma":                # async copy into res, completes tx on bar
                _, bn, nb, res, tag = op
                landed = self.t + self.rng.uniform(0.5, 4.0)
                for rtag, rend in self.readers.get(res, []):
                    if rend > self.t + 1e-9:
                        self.err(f"copy of {tag} into {res} starts while {rtag} is read until {rend:.2f}")

                def land(bn=bn, nb=nb, res=res, tag=tag, landed=landed):
                    self.write(res, tag, landed)
                    self.complete_tx(bn, nb)
                self.at(landed, land)
            elif kind == "mma":                # in-order tensor pipe
                _, reads, writes = op
                start = max(self.t, self.mma_end)
                end = start + self.rng.uniform(0.3, 1.2)
                self.mma_end = end

                def run(reads=reads, writes=writes, end=end):
                    for res, tag in reads:
                        self.read(res, tag, end)
                    for res, tag, check in writes:
                        if check is not None:
                            check()
                        self.write(res, tag, end)
                self.at(start, run)
            elif kind == "commit":             # arrives once every MMA issued so far is done
                self.at(max(self.t, self.mma_end), lambda bn=op[1]: self.arrive(bn))
            elif kind == "read":
                self.read(op[1], op[2], self.t)
            elif kind == "write":
                self.write(op[1], op[2], self.t)
            else:
                raise ValueError(kind)

    def run(self):
        while self.events:
            t, _, fn = heapq.heappop(self.events)
            self.t = t
            fn()
        unfinished = set(self.roles) - self.finished
        if unfinished:
            self.err(f"deadlock: {sorted(unfinished)} blocked on {self.blocked}")


def prefill_items(lens, num_q_heads, num_kv_heads, causal, BM=128, BN=128):
    """Work items in launch order, numbered as the kernels number them:
    sequences heaviest first, one group per (sequence, kv head), q tiles
    heaviest first inside a group.  Each item: key tiles per slot."""
    G = num_q_heads // num_kv_heads
    order = sorted(range(len(lens)), key=lambda b: -(lens[b] * (lens[b] + 1) / 2 if causal else lens[b] ** 2))
    items = []
    for b in order:
        nq = -(-lens[b] // BM)
        nk = -(-lens[b] // BN)
        for _ in range(num_kv_heads):
            ctas = nq * (G // 2) if G % 2 == 0 else ((nq + 1) // 2) * G
            for rank in range(ctas):
                if G % 2 == 0:
                    t = nq - 1 - rank // (G // 2)
                    qt = (t, t)
                else:
                    pr = (nq + 1) // 2 - 1 - rank // G
                    qt = (2 * pr, 2 * pr + 1)
                nkv = tuple(0 if not 0 <= q < nq else
                            (min(nk, (q * BM + BM - 1) // BN + 1) if causal else nk) for q in qt)
                items.append(nkv)
    return items


MUTATIONS = ("no_q_empty_wait", "late_q_empty", "no_epilogue_wait", "consumers_short",
             "no_vh_empty_wait", "v_release_before_pv", "rescale_after_half")
# planted mistakes of the paged producer's tail hand-off
PAGED_MUTATIONS = ("tail_full_before_zero", "tail_no_land_wait")


def simulate(items, claimed, NS, F8, seed=0, QD=4, mutation=None, tails=frozenset()):
    """One CTA taking the items `claimed` (indices into `items`, in claim
    order).  Raises ProtocolError on any violation.  tails (paged K/V, bf16
    only): items whose last V tile holds the cache's last, partly filled page;
    that tile lands on the vtail barrier, the producer zeroes its rows past the
    end and only then arrives on its kv_full barrier."""
    assert not (tails and F8)
    sim = _Sim(seed)
    rng = sim.rng
    sim.bar("q0")
    sim.bar("q1")
    for i in range(NS):
        sim.bar(f"kv_full{i}")
        sim.bar(f"kv_empty{i}", 2 if (F8 and i % 2 == 1) else 1)
    for k in range(2):
        sim.bar(f"s_full{k}")
        sim.bar(f"p_full{k}", 4)
        sim.bar(f"p_half{k}", 4)
        sim.bar(f"o_done{k}")
        sim.bar(f"q_empty{k}")
        if F8:
            sim.bar(f"vh_full{k}", 2)
            sim.bar(f"vh_empty{k}")
    consumers = 1 + 8 + (2 if F8 else 0)
    for i in range(QD):
        sim.bar(f"item_full{i}")
        sim.bar(f"item_empty{i}", 1 + 8 if mutation == "consumers_short" else consumers)

        def all_read(i=i):
            if queue_reads.get(i, 0) != consumers:
                sim.err(f"queue entry {i} released after {queue_reads.get(i, 0)} of {consumers} reads")
        sim.on_complete[f"item_empty{i}"] = all_read
    sim.bar("final")
    sim.bar("vtail")
    queue, queue_reads = {}, {}
    o_state = [None, None]      # per slot: (item, tiles accumulated) or "read out"
    epilogue_reads = {}
    half_done = {}
    rescale = {}

    def producer():
        issued, qc, tails_done = 0, [0, 0], 0
        for n, it in enumerate(list(claimed) + [-1]):
            qi = n % QD
            if n >= QD:
                yield ("wait", f"item_empty{qi}", n // QD - 1)
                if queue_reads.get(qi, 0) != consumers:
                    sim.err(f"queue entry {qi} overwritten after {queue_reads.get(qi, 0)} of {consumers} reads")
            queue[qi], queue_reads[qi] = it, 0
            yield ("write", f"queue{qi}", ("item", n))
            yield ("arrive", f"item_full{qi}")
            if it < 0:
                return
            nkv = items[it]
            tail_R = None
            for e in range(2 * max(nkv)):
                R = issued
                if R >= NS:
                    yield ("wait", f"kv_empty{R % NS}", R // NS - 1)
                if it in tails and e == 2 * max(nkv) - 1:
                    # the tail V tile lands on vtail; it is marked full below
                    yield ("expect_tx", "vtail", 1)
                    yield ("tma", "vtail", 1, f"ring{R % NS}", ("KV raw", it, e))
                    tail_R = (R, e)
                else:
                    yield ("expect_tx", f"kv_full{R % NS}", 1)
                    yield ("tma", f"kv_full{R % NS}", 1, f"ring{R % NS}", ("KV", it, e))
                issued += 1
                if e == 0:
                    for k in range(2):
                        if nkv[k] > 0:
                            if qc[k] >= 1 and mutation != "no_q_empty_wait":
                                yield ("wait", f"q_empty{k}", qc[k] - 1)
                            yield ("expect_tx", f"q{k}", 1)
                            yield ("tma", f"q{k}", 1, f"qtile{k}", ("Q", it, k))
                            qc[k] += 1
            if tail_R is not None:
                R, e = tail_R
                if mutation == "tail_full_before_zero":
                    yield ("arrive", f"kv_full{R % NS}")
                if mutation != "tail_no_land_wait":
                    yield ("wait", "vtail", tails_done)
                    yield ("read", f"ring{R % NS}", ("KV raw", it, e))
                yield ("delay", rng.uniform(0.1, 0.6))          # the warp zeroes the rows past the end
                yield ("write", f"ring{R % NS}", ("KV", it, e))
                if mutation != "tail_full_before_zero":
                    yield ("arrive", f"kv_full{R % NS}")
                tails_done += 1
            yield ("delay", rng.uniform(0.0, 0.2))

    def take(n):
        qi = n % QD
        yield ("wait", f"item_full{qi}", n // QD)
        yield ("read", f"queue{qi}", ("item", n))
        it = queue[qi]
        queue_reads[qi] += 1
        yield ("arrive", f"item_empty{qi}")
        return it

    def mma():
        ring, qc, tiles, vcount, n = 0, [0, 0], [0, 0], 0, 0
        while True:
            it = yield from take(n)
            n += 1
            if it < 0:
                break
            nk = items[it]
            n_max = max(nk)
            yield ("wait", f"kv_full{ring % NS}", ring // NS)
            for k in range(2):
                if nk[k] > 0:
                    yield ("wait", f"q{k}", qc[k])
                    yield ("mma", [(f"qtile{k}", ("Q", it, k)), (f"ring{ring % NS}", ("KV", it, 0))],
                           [(f"sp{k}a", ("S", it, k, 0), None), (f"sp{k}b", ("S", it, k, 0), None)])
                    yield ("commit", f"s_full{k}")
                    if nk[k] == 1:
                        yield ("commit", f"q_empty{k}")
                    qc[k] += 1
            yield ("commit", f"kv_empty{ring % NS}")

            def slot_step(k, j, v_R, vslot, k_R, it=it, nk=nk):
                if j >= nk[k]:
                    return
                yield ("wait", f"p_half{k}", tiles[k] + j)
                v = (f"vh{vslot}", ("VH", it, j)) if F8 else (f"ring{v_R % NS}", ("KV", it, 2 * j + 1))

                def check_o(k=k, j=j, it=it):
                    if j == 0 and o_state[k] not in (None, "read out"):
                        sim.err(f"first P V of item {it} overwrites O {o_state[k]} before its epilogue")
                    if j > 0 and o_state[k] != (it, j):
                        sim.err(f"P V ({it}, {j}) accumulates onto {o_state[k]}")
                    o_state[k] = (it, j + 1)
                # P V over the first 64 keys, then (p_full) the last 64
                yield ("mma", [(f"sp{k}a", ("P", it, k, j)), v], [(f"o{k}", ("O half", it, k, j + 1), check_o)])
                yield ("wait", f"p_full{k}", tiles[k] + j)
                def check_half(k=k, j=j, it=it):
                    cur = sim.content.get(f"o{k}")
                    if cur is None or cur[0] != ("O half", it, k, j + 1):
                        sim.err(f"second half of P V ({it}, {j}) accumulates onto {cur and cur[0]}")
                yield ("mma", [(f"sp{k}b", ("P", it, k, j)), v], [(f"o{k}", ("O", it, k, j + 1), check_half)])
                yield ("commit", f"o_done{k}")
                if j + 1 < nk[k]:
                    yield ("mma", [(f"qtile{k}", ("Q", it, k)), (f"ring{k_R % NS}", ("KV", it, 2 * j + 2))],
                           [(f"sp{k}a", ("S", it, k, j + 1), None), (f"sp{k}b", ("S", it, k, j + 1), None)])
                    yield ("commit", f"s_full{k}")
                    if j + (3 if mutation == "late_q_empty" else 2) == nk[k]:
                        yield ("commit", f"q_empty{k}")

            for j in range(n_max):
                v_R, k_R = ring + 2 * j + 1, ring + 2 * j + 2
                vslot = vcount & 1
                need_k = j + 1 < nk[0] or j + 1 < nk[1]
                if F8:
                    yield ("wait", f"vh_full{vslot}", vcount >> 1)
                else:
                    yield ("wait", f"kv_full{v_R % NS}", v_R // NS)
                if need_k:
                    yield ("wait", f"kv_full{k_R % NS}", k_R // NS)
                release = ("commit", f"vh_empty{vslot}") if F8 else ("commit", f"kv_empty{v_R % NS}")
                if mutation == "v_release_before_pv":
                    yield release
                yield from slot_step(0, j, v_R, vslot, k_R)
                yield from slot_step(1, j, v_R, vslot, k_R)
                if mutation != "v_release_before_pv":
                    yield release
                if need_k:
                    yield ("commit", f"kv_empty{k_R % NS}")
                vcount += 1
            ring += 2 * n_max
            tiles[0] += nk[0]
            tiles[1] += nk[1]
        yield ("commit", "final")
        yield ("wait", "final", 0)

    def converter(half):
        ring, vcount, n = 0, 0, 0
        while True:
            it = yield from take(n)
            n += 1
            if it < 0:
                return
            n_max = max(items[it])
            for j in range(n_max):
                v_R = ring + 2 * j + 1
                vslot = vcount & 1
                yield ("wait", f"kv_full{v_R % NS}", v_R // NS)
                if vcount >= 2 and mutation != "no_vh_empty_wait":
                    yield ("wait", f"vh_empty{vslot}", (vcount >> 1) - 1)
                yield ("read", f"ring{v_R % NS}", ("KV", it, 2 * j + 1))
                yield ("delay", rng.uniform(0.2, 1.0))
                # each half stores its 64 keys; the tile is whole after both
                yield ("write", f"vh{vslot}", ("VH half", it, j, half))
                half_done[(it, j)] = half_done.get((it, j), 0) + 1
                if half_done[(it, j)] == 2:
                    yield ("write", f"vh{vslot}", ("VH", it, j))
                yield ("arrive", f"vh_full{vslot}")
                yield ("arrive", f"kv_empty{v_R % NS}")
                vcount += 1
            ring += 2 * n_max

    def softmax(k, wq):
        tiles, n = 0, 0
        while True:
            it = yield from take(n)
            n += 1
            if it < 0:
                return
            nk = items[it][k]
            for j in range(nk):
                g = tiles + j
                yield ("wait", f"s_full{k}", g)
                if wq == 0:          # the warpgroup's S read and P stores, modelled once
                    yield ("read", f"sp{k}a", ("S", it, k, j))
                    yield ("read", f"sp{k}b", ("S", it, k, j))
                yield ("delay", rng.uniform(0.3, 1.0))
                if wq == 0:
                    yield ("write", f"sp{k}a", ("P", it, k, j))
                if j > 0 and rescale[(it, k, j)]:
                    # before any of this tile's P V: the previous P V has landed
                    if mutation != "rescale_after_half":
                        yield ("wait", f"o_done{k}", g - 1)
                        yield ("delay", rng.uniform(0.1, 0.5))   # the O loads take time
                        if wq == 0:
                            yield ("read", f"o{k}", ("O", it, k, j))
                            yield ("write", f"o{k}", ("O", it, k, j))
                yield ("arrive", f"p_half{k}")
                if j > 0 and rescale[(it, k, j)] and mutation == "rescale_after_half":
                    yield ("wait", f"o_done{k}", g - 1)
                    yield ("delay", rng.uniform(0.1, 0.5))
                    if wq == 0:
                        yield ("read", f"o{k}", ("O", it, k, j))
                        yield ("write", f"o{k}", ("O", it, k, j))
                yield ("delay", rng.uniform(0.3, 1.0))
                if wq == 0:
                    yield ("write", f"sp{k}b", ("P", it, k, j))
                yield ("arrive", f"p_full{k}")
            if nk == 0:
                continue
            if mutation != "no_epilogue_wait":
                yield ("wait", f"o_done{k}", tiles + nk - 1)
            if wq == 0:
                yield ("read", f"o{k}", ("O", it, k, nk))
            yield ("delay", rng.uniform(0.3, 1.5))
            epilogue_reads[(it, k)] = epilogue_reads.get((it, k), 0) + 1
            if epilogue_reads[(it, k)] == 4:
                o_state[k] = "read out"
            tiles += nk

    for it in claimed:
        for k in range(2):
            for j in range(items[it][k]):
                rescale[(it, k, j)] = rng.random() < 0.2
    sim.add_role("producer", producer())
    sim.add_role("mma", mma())
    for k in range(2):
        for wq in range(4):
            sim.add_role(f"softmax{k}.{wq}", softmax(k, wq))
    if F8:
        for h in range(2):
            sim.add_role(f"converter{h}", converter(h))
    sim.run()


def random_case(seed):
    """A random item list and one CTA's claimed subset, bf16 or E4M3."""
    rng = random.Random(seed)
    lens = [rng.choice([1, 5, 127, 128, 129, 200, 256, 300, 513, 700]) for _ in range(rng.randint(1, 4))]
    hkv = rng.choice([1, 2])
    G = rng.choice([1, 2, 3, 4])
    F8 = rng.random() < 0.5
    NS = 8 if F8 else rng.choice([5, 8])
    items = prefill_items(lens, hkv * G, hkv, rng.random() < 0.7)
    claimed = sorted(rng.sample(range(len(items)), min(len(items), rng.randint(1, 12))))
    return items, claimed, NS, F8


def random_paged_case(seed):
    """random_case restricted to bf16, with a random set of items whose last
    V tile is a partly filled page (paged K/V)."""
    rng = random.Random(seed + 30011)
    items, claimed, _, _ = random_case(seed)
    tails = frozenset(i for i in claimed if rng.random() < 0.5)
    return items, claimed, rng.choice([5, 8]), tails
