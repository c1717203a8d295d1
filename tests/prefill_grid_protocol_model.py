"""Host-side model of the grid-form prefill kernel's synchronisation protocol
(fa_prefill_pp_kernel: one CTA = one work item of two 128-row query tiles, the
slots, that read the same K/V tiles).  The grid form runs when the schedule is
"grid", while a stream is being captured into a graph, and for the cascade
decode's prefix pass.

Roles, as in the kernel: a TMA producer (Q of slot 0, K_0, Q of slot 1, then
the K/V ring; paged K/V: the V tile of the cache's last, partly filled page
lands on its own barrier, is zeroed past the end and only then marked full),
one MMA thread, four softmax warps per slot (one per TMEM lane quadrant) and,
with E4M3 inputs, two converter warps that widen each V tile into one of two
f16 tiles.  The MMA thread issues both slots' first S from K_0 and then frees
it; per key tile j and slot k it issues the first half of P_k V_j once the
slot's softmax has handed over keys 0-63 (p_half), the second half after
p_full, commits o_done, and then S_k(j+1) into the TMEM columns P_k(j)
occupies.  A softmax warp reads S, writes P over S's first 64 columns in two
halves, rescales its quadrant of O when its maximum grew (after waiting for
the previous P V), and arrives on p_half and p_full.

The simulator is the one of the persistent prefill's model; it checks deadlock
freedom, parity aliasing, reads of content that has landed and is the
expected one, and writes that never land on content still being read.
`mutation` plants one protocol mistake so tests can check the model sees it.
"""
from __future__ import annotations

import random

from tests.persist_protocol_model import ProtocolError, _Sim  # noqa: F401  (re-exported)

MUTATIONS = (
    "k0_released_before_s",    # K_0 freed before the slots' first S MMAs
    "v_released_before_pv",    # a V ring slot freed before its P V MMAs
    "pv_without_p_half",       # first half of P V issued before P's first half is written
    "next_s_before_pv",        # S_k(j+1) issued over P_k(j) before the P V that reads it
    "p_half_before_rescale",   # p_half arrived before the rescale of O
    "epilogue_without_wait",   # O read out before the last P V has landed
    "s_parity",                # softmax waits on S with the wrong parity
    "converter_without_empty",  # E4M3: f16 V tile rewritten while P V may read it
    "tail_full_before_zero",   # paged: tail V tile marked full before its rows are zeroed
)

# Waits the kernel keeps although the protocol already implies them.  Before
# rescaling O at tile j a softmax warp waits for slot k's P V of tile j - 1;
# but it has just waited on s_full for S_k(j), which the MMA thread issued
# after that P V, and a tcgen05 commit completes only after every earlier MMA
# of the thread.
REDUNDANT = ("rescale_without_wait",)


def simulate(nk, NS, f8, tail, rescale, seed=0, mutation=None):
    """One CTA: slot k has nk[k] key tiles (nk[0] >= 1); a ring of NS K/V
    slots; f8: E4M3 inputs (converters); tail: paged K/V whose last V tile
    ends inside a page (bf16 only); rescale[k][w][j]: quadrant w of slot k
    rescales O at tile j (j >= 1).  Raises ProtocolError on any violation."""
    assert nk[0] >= 1 and not (f8 and tail)
    n_max = max(nk)
    sim = _Sim(seed)
    rng = sim.rng
    sim.bar("q0")
    sim.bar("q1")
    for i in range(NS):
        sim.bar(f"kv_full{i}")
        sim.bar(f"kv_empty{i}", 2 if (f8 and i % 2 == 1) else 1)
    for k in range(2):
        sim.bar(f"s_full{k}")
        sim.bar(f"p_full{k}", 4)
        sim.bar(f"p_half{k}", 4)
        sim.bar(f"o_done{k}")
        if f8:
            sim.bar(f"vh_full{k}", 2)
            sim.bar(f"vh_empty{k}")
    sim.bar("final")
    sim.bar("vtail")
    tail_item = 2 * n_max - 1 if tail else -1

    def ring(item, h):           # half h (keys 64h..64h+63) of the item's ring slot
        return f"ring{item % NS}_{h}"

    def producer():
        if nk[0] > 0:
            yield ("expect_tx", "q0", 1)
            yield ("tma", "q0", 1, "q0", ("Q", 0))
        for item in range(2 * n_max):
            yield ("wait", f"kv_empty{item % NS}", item // NS - 1)
            name = ("V" if item & 1 else "K", item >> 1)
            if item == tail_item:
                yield ("expect_tx", "vtail", 2)
                for h in range(2):
                    yield ("tma", "vtail", 1, ring(item, h), ("V raw", item >> 1))
            else:
                yield ("expect_tx", f"kv_full{item % NS}", 2)
                for h in range(2):
                    yield ("tma", f"kv_full{item % NS}", 1, ring(item, h), name)
            if item == 0 and nk[1] > 0:
                yield ("expect_tx", "q1", 1)
                yield ("tma", "q1", 1, "q1", ("Q", 1))
            yield ("delay", rng.uniform(0.0, 0.2))
        if tail:
            if mutation == "tail_full_before_zero":
                yield ("arrive", f"kv_full{tail_item % NS}")
            yield ("wait", "vtail", 0)
            for h in range(2):
                yield ("read", ring(tail_item, h), ("V raw", n_max - 1))
            yield ("delay", rng.uniform(0.1, 0.6) + (rng.expovariate(0.3) if rng.random() < 0.3 else 0.0))
            for h in range(2):
                yield ("write", ring(tail_item, h), ("V", n_max - 1))
            if mutation != "tail_full_before_zero":
                yield ("arrive", f"kv_full{tail_item % NS}")

    def s_mma(k, j, item):
        # S_k(j) = Q_k K_j^T into slot k's TMEM columns, P's columns included
        writes = []
        for w in range(4):
            writes.append((f"S{k}_{w}", ("S", k, j), None))
            for h in range(2):
                writes.append((f"P{k}_{w}_{h}", ("S", k, j), None))
        return ("mma", [(f"q{k}", ("Q", k)), (ring(item, 0), ("K", j)), (ring(item, 1), ("K", j))], writes)

    def o_check(k, w, j, h):
        def check():
            if j == 0 and h == 0:
                return
            want = ("O", k, j, 0, False) if h == 1 else ("O", k, j - 1, 1, bool(rescale[k][w][j]))
            cur = sim.content.get(f"O{k}_{w}")
            if cur is None or cur[0] != want:
                sim.err(f"P V half {h} of slot {k} tile {j} accumulates onto {cur and cur[0]}, expected {want}")
            if cur[1] > sim.t + 1e-9:
                sim.err(f"P V half {h} of slot {k} tile {j} starts before {want} has landed")
        return check

    def pv_mma(k, j, h):
        v_src = (f"vh{j & 1}_{h}", ("VH", j)) if f8 else (ring(2 * j + 1, h), ("V", j))
        reads = [v_src] + [(f"P{k}_{w}_{h}", ("P", k, j)) for w in range(4)]
        return ("mma", reads, [(f"O{k}_{w}", ("O", k, j, h, False), o_check(k, w, j, h)) for w in range(4)])

    def mma():
        yield ("wait", "q0", 0)
        yield ("wait", "kv_full0", 0)
        if mutation == "k0_released_before_s":
            yield ("commit", "kv_empty0")
        if nk[0] > 0:
            yield s_mma(0, 0, 0)
            yield ("commit", "s_full0")
        if nk[1] > 0:
            yield ("wait", "q1", 0)
            yield s_mma(1, 0, 0)
            yield ("commit", "s_full1")
        if mutation != "k0_released_before_s":
            yield ("commit", "kv_empty0")

        def slot_step(k, j, k_item):
            if j >= nk[k]:
                return
            if mutation == "next_s_before_pv" and j + 1 < nk[k]:
                yield s_mma(k, j + 1, k_item)
            if mutation != "pv_without_p_half":
                yield ("wait", f"p_half{k}", j)
            yield pv_mma(k, j, 0)
            yield ("wait", f"p_full{k}", j)
            yield pv_mma(k, j, 1)
            yield ("commit", f"o_done{k}")
            if mutation != "next_s_before_pv" and j + 1 < nk[k]:
                yield s_mma(k, j + 1, k_item)
                yield ("commit", f"s_full{k}")
            elif j + 1 < nk[k]:
                yield ("commit", f"s_full{k}")

        for j in range(n_max):
            v_item, k_item = 2 * j + 1, 2 * j + 2
            need_k = j + 1 < nk[0] or j + 1 < nk[1]
            if f8:
                yield ("wait", f"vh_full{j & 1}", j >> 1)
            else:
                yield ("wait", f"kv_full{v_item % NS}", v_item // NS)
            if need_k:
                yield ("wait", f"kv_full{k_item % NS}", k_item // NS)
            if mutation == "v_released_before_pv" and not f8:
                yield ("commit", f"kv_empty{v_item % NS}")
            yield from slot_step(0, j, k_item)
            yield from slot_step(1, j, k_item)
            if f8:
                yield ("commit", f"vh_empty{j & 1}")
            elif mutation != "v_released_before_pv":
                yield ("commit", f"kv_empty{v_item % NS}")
            if need_k:
                yield ("commit", f"kv_empty{k_item % NS}")
        yield ("commit", "final")
        yield ("wait", "final", 0)

    def converter(h):
        for j in range(n_max):
            v_item = 2 * j + 1
            yield ("wait", f"kv_full{v_item % NS}", v_item // NS)
            if mutation != "converter_without_empty":
                yield ("wait", f"vh_empty{j & 1}", (j >> 1) - 1)
            yield ("read", ring(v_item, h), ("V", j))
            yield ("delay", rng.uniform(0.2, 1.0))
            yield ("read", ring(v_item, h), ("V", j))
            yield ("write", f"vh{j & 1}_{h}", ("VH", j))
            yield ("arrive", f"vh_full{j & 1}")
            yield ("arrive", f"kv_empty{v_item % NS}")

    def softmax(k, w):
        for j in range(nk[k]):
            yield ("wait", f"s_full{k}", j + 1 if mutation == "s_parity" and j % 2 == 1 else j)
            yield ("read", f"S{k}_{w}", ("S", k, j))
            yield ("delay", rng.uniform(0.2, 1.0))           # row maximum, first half of P
            yield ("write", f"P{k}_{w}_0", ("P", k, j))
            resc = j > 0 and rescale[k][w][j]
            if resc and mutation == "p_half_before_rescale":
                yield ("arrive", f"p_half{k}")
            if resc:
                if mutation != "rescale_without_wait":
                    yield ("wait", f"o_done{k}", j - 1)
                yield ("read", f"O{k}_{w}", ("O", k, j - 1, 1, False))
                yield ("delay", rng.uniform(0.05, 0.4))
                yield ("write", f"O{k}_{w}", ("O", k, j - 1, 1, True))
            if not (resc and mutation == "p_half_before_rescale"):
                yield ("arrive", f"p_half{k}")
            yield ("delay", rng.uniform(0.2, 1.0))           # second half of P
            yield ("write", f"P{k}_{w}_1", ("P", k, j))
            yield ("arrive", f"p_full{k}")
        if nk[k] > 0:
            if mutation != "epilogue_without_wait":
                yield ("wait", f"o_done{k}", nk[k] - 1)
            yield ("read", f"O{k}_{w}", ("O", k, nk[k] - 1, 1, False))

    sim.add_role("producer", producer())
    sim.add_role("mma", mma())
    if f8:
        for h in range(2):
            sim.add_role(f"converter{h}", converter(h))
    for k in range(2):
        for w in range(4):
            sim.add_role(f"softmax{k}_{w}", softmax(k, w))
    sim.run()


def random_case(seed):
    """(nk, NS, f8, tail, rescale) over the kernel's configurations: a ring of
    5 K/V tiles for bf16 with d = 128, 8 for d = 64 and for E4M3; any pair of
    key-tile counts."""
    r = random.Random(3000 + seed)
    f8 = r.random() < 0.3
    tail = (not f8) and r.random() < 0.4
    NS = 8 if f8 else r.choice([5, 8])
    n0 = r.choice([1, 2, 3, 4, 5, 8, 11])
    n1 = r.choice([0, 1, max(1, n0 - 1), n0, n0 + 1])
    nk = (n0, n1)
    rescale = [[[r.random() < 0.3 for _ in range(max(nk) + 1)] for _ in range(4)] for _ in range(2)]
    return nk, NS, f8, tail, rescale
