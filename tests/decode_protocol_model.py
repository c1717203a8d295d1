"""Host-side models of the split-decode kernels' synchronisation protocols:
the tensor-core kernel (fa_decode_tc_kernel, `simulate`) and, at the end of
this file, the CUDA-core kernel (fa_decode_split_kernel, `simulate_cc`); one
CTA = one (request, kv head, split).

The kernel runs a TMA producer (warp 0), an MMA thread (warp 1) and four
softmax warps, one per TMEM lane quadrant.  They hand data to each other
through mbarriers waited on by phase parity:

  * the producer fills a ring of ITEMS shared-memory slots with the split's
    K and V tiles as separate items (K_0, V_0, K_1, ...); the slot of item
    `it` is it % ITEMS and the MMA thread frees it by a commit after the MMAs
    that read it (S for a K item, P V for a V item);
  * the MMA thread issues S_0 and S_1 into two TMEM score buffers, then per
    tile j: P V_j into the one O accumulator, then S_{j+2} into S_j's buffer;
  * the softmax warps read S_j, agree the tile maxima through a double-buffered
    shared array and the named barrier, write P_j into one of two
    shared-memory P buffers (after P V_{j-2} has read it), rescale O when a
    maximum grew (after P V_{j-1} has landed), and arrive on p_full;
  * the epilogue reads O once the last P V has landed;
  * the V tile holding the cache's last, partly filled page lands on its own
    barrier (vtail); the producer zeroes the rows past the cache end and only
    then arrives on the slot's kv_full barrier;
  * with an E4M3 cache the softmax warps build the Q operand themselves
    (a four-arrival q barrier); with bf16 the producer copies it by TMA.

Each role is a generator issuing the kernel's waits, arrivals, commits, copies,
MMAs and shared/TMEM accesses in the kernel's order with its phase counters;
the simulator (shared with the prefill model) gives them random durations and
checks deadlock freedom, parity aliasing, reads of content that has landed and
is the expected one, and writes that never land on content still being read.
`mutation` plants one protocol mistake so tests can check the model sees it.
"""
from __future__ import annotations

from tests.persist_protocol_model import ProtocolError, _Sim  # noqa: F401  (re-exported)

MUTATIONS = (
    "k_release_before_s",      # K slot freed before its S MMA is issued
    "v_release_before_pv",     # V slot freed before its P V MMA is issued
    "s_before_p_wait",         # S_{j+2} issued before P_j is handed over
    "rescale_no_wait",         # O rescaled before P V_{j-1} has landed
    "epilogue_no_wait",        # O read out before the last P V has landed
    "p_full_before_p",         # p_full arrived before P_j is written
    "red_single_buffer",       # one tile-maxima buffer for every tile
    "s_parity",                # S wait with the tile index as parity
    "ring_parity",             # producer waits on the slot's current phase
    "tail_full_before_zero",   # tail V slot marked full before its rows are zeroed
    "tail_no_land_wait",       # tail V rows zeroed before the copy has landed
)

# Waits the kernel keeps although the protocol already implies them.  Before
# writing P_j (j >= 2) the softmax waits for P V_{j-2} to finish reading the P
# buffer; but it has just waited on s_full for S_j, which the MMA thread issued
# after P V_{j-2}, and a tcgen05 commit completes only after every earlier MMA
# of the thread.  Dropping that wait can therefore never expose the buffer.
REDUNDANT = ("p_no_o_done_wait",)


def simulate(n_tiles, items, kv8, tail, grew, seed=0, mutation=None):
    """One CTA over `n_tiles` key tiles with a ring of `items` slots.  `tail`:
    the last V tile is the cache's partly filled last page.  `grew[j]` (j >= 1):
    some head's running maximum grew at tile j, so the softmax rescales O.
    Raises ProtocolError on any violation."""
    assert n_tiles >= 1 and items >= 3 and len(grew) == n_tiles
    sim = _Sim(seed)
    rng = sim.rng
    sim.bar("q", 4 if kv8 else 1)
    for s in range(items):
        sim.bar(f"kv_full{s}")
        sim.bar(f"kv_empty{s}")
    for k in range(2):
        sim.bar(f"s_full{k}")
        sim.bar(f"p_full{k}", 4)
        sim.bar(f"o_done{k}")
    sim.bar("vtail")
    sim.bar("final")
    sim.bar("named", 4)          # bar.sync 1, 128 over the four softmax warps
    tail_item = 2 * n_tiles - 1 if tail else -1

    def slot(it):
        return it % items

    def producer():
        if not kv8:
            yield ("expect_tx", "q", 1)
            yield ("tma", "q", 1, "q", ("Q",))
        for it in range(2 * n_tiles):
            phase = it // items if mutation == "ring_parity" else it // items - 1
            yield ("wait", f"kv_empty{slot(it)}", phase)
            i, is_v = it >> 1, it & 1
            if it == tail_item:
                yield ("expect_tx", "vtail", 1)
                yield ("tma", "vtail", 1, f"ring{slot(it)}", ("V raw", i))
            else:
                yield ("expect_tx", f"kv_full{slot(it)}", 1)
                yield ("tma", f"kv_full{slot(it)}", 1, f"ring{slot(it)}", ("V" if is_v else "K", i))
            yield ("delay", rng.uniform(0.0, 0.2))
        if tail:
            s = slot(tail_item)
            if mutation == "tail_full_before_zero":
                yield ("arrive", f"kv_full{s}")
            if mutation != "tail_no_land_wait":
                yield ("wait", "vtail", 0)
                yield ("read", f"ring{s}", ("V raw", n_tiles - 1))
            # the warp zeroes rows past the end (a warp can also stall for a while)
            yield ("delay", rng.uniform(0.1, 0.6) + (rng.expovariate(0.3) if rng.random() < 0.3 else 0.0))
            yield ("write", f"ring{s}", ("V", n_tiles - 1))
            if mutation != "tail_full_before_zero":
                yield ("arrive", f"kv_full{s}")

    q_reads = [("q", ("Q",))] if not kv8 else [(f"q{w}", ("Q",)) for w in range(4)]

    def issue_s(i):
        it = 2 * i
        if mutation == "k_release_before_s":
            yield ("commit", f"kv_empty{slot(it)}")
        yield ("mma", [(f"ring{slot(it)}", ("K", i))] + q_reads, [(f"S{i & 1}", ("S", i), None)])
        yield ("commit", f"s_full{i & 1}")
        if mutation != "k_release_before_s":
            yield ("commit", f"kv_empty{slot(it)}")

    def o_check(j, w):
        def check():
            if j == 0:
                return
            want = ("O", j - 1, bool(grew[j]))
            cur = sim.content.get(f"O{w}")
            if cur is None or cur[0] != want:
                sim.err(f"P V_{j} accumulates onto {cur and cur[0]} in O quadrant {w}, expected {want}")
            if cur[1] > sim.t + 1e-9:
                sim.err(f"P V_{j} starts before {want} has landed in O quadrant {w}")
        return check

    def issue_pv(j):
        it = 2 * j + 1
        if mutation == "v_release_before_pv":
            yield ("commit", f"kv_empty{slot(it)}")
        reads = [(f"ring{slot(it)}", ("V", j))] + [(f"P{j & 1}_{w}", ("P", j)) for w in range(4)]
        yield ("mma", reads, [(f"O{w}", ("O", j, False), o_check(j, w)) for w in range(4)])
        yield ("commit", f"o_done{j & 1}")
        if mutation != "v_release_before_pv":
            yield ("commit", f"kv_empty{slot(it)}")

    def mma():
        yield ("wait", "q", 0)
        for i in range(min(2, n_tiles)):
            yield ("wait", f"kv_full{slot(2 * i)}", (2 * i) // items)
            yield from issue_s(i)
        for j in range(n_tiles):
            n = j + 2
            if mutation == "s_before_p_wait" and n < n_tiles:
                yield ("wait", f"kv_full{slot(2 * n)}", (2 * n) // items)
                yield from issue_s(n)
            yield ("wait", f"p_full{j & 1}", j >> 1)
            yield ("wait", f"kv_full{slot(2 * j + 1)}", (2 * j + 1) // items)
            yield from issue_pv(j)
            if mutation != "s_before_p_wait" and n < n_tiles:
                yield ("wait", f"kv_full{slot(2 * n)}", (2 * n) // items)
                yield from issue_s(n)
        yield ("commit", "final")
        yield ("wait", "final", 0)

    def softmax(w):
        syncs = 0

        def named_sync():
            nonlocal syncs
            yield ("arrive", "named")
            yield ("wait", "named", syncs)
            syncs += 1

        if kv8:
            yield ("delay", rng.uniform(0.1, 0.5))
            yield ("write", f"q{w}", ("Q",))
            yield ("arrive", "q")
        yield from named_sync()
        for j in range(n_tiles):
            yield ("wait", f"s_full{j & 1}", j if mutation == "s_parity" else j >> 1)
            yield ("read", f"S{j & 1}", ("S", j))
            yield ("delay", rng.uniform(0.1, 0.8))
            red = 0 if mutation == "red_single_buffer" else j & 1
            yield ("write", f"red{red}_{w}", ("max", j))
            yield from named_sync()
            yield ("delay", rng.uniform(0.0, 1.5))         # a warp may lag before reading the maxima
            for v in range(4):
                yield ("read", f"red{red}_{v}", ("max", j))
            if j >= 2 and mutation != "p_no_o_done_wait":
                yield ("wait", f"o_done{j & 1}", (j - 2) >> 1)
            if mutation == "p_full_before_p":
                yield ("arrive", f"p_full{j & 1}")
            yield ("delay", rng.uniform(0.2, 1.5))         # exponentials
            yield ("write", f"P{j & 1}_{w}", ("P", j))
            if j > 0 and grew[j]:
                if mutation != "rescale_no_wait":
                    yield ("wait", f"o_done{(j - 1) & 1}", (j - 1) >> 1)
                # each warp scales its own TMEM lane quadrant of O
                yield ("read", f"O{w}", ("O", j - 1, False))
                yield ("delay", rng.uniform(0.05, 0.3))
                yield ("write", f"O{w}", ("O", j - 1, True))
            if mutation != "p_full_before_p":
                yield ("arrive", f"p_full{j & 1}")
        # epilogue: normaliser partials, then O once the last P V has landed
        yield ("write", f"lred_{w}", ("l",))
        yield from named_sync()
        for v in range(4):
            yield ("read", f"lred_{v}", ("l",))
        jl = n_tiles - 1
        if mutation != "epilogue_no_wait":
            yield ("wait", f"o_done{jl & 1}", jl >> 1)
        yield ("read", f"O{w}", ("O", jl, False))

    sim.add_role("producer", producer())
    sim.add_role("mma", mma())
    for w in range(4):
        sim.add_role(f"softmax{w}", softmax(w))
    sim.run()


def random_case(seed):
    """(n_tiles, items, kv8, tail, grew): ring depths of the kernel's
    configurations (bf16: 3 slots with 8 padded rows, 6 with 16; E4M3: 6, 12)."""
    import random
    r = random.Random(1000 + seed)
    kv8 = r.random() < 0.5
    items = r.choice([6, 12] if kv8 else [3, 6])
    n_tiles = r.choice([1, 2, 3, 4, 5, 7, 9, 12])
    tail = r.random() < 0.5
    grew = [False] + [r.random() < 0.4 for _ in range(n_tiles - 1)]
    return n_tiles, items, kv8, tail, grew


# --------------------------------------------------------------------------
# The CUDA-core split kernel (fa_decode_split_kernel): one TMA lane fills a
# ring of STAGES page slots (K and V of one 64-token page each; full barrier
# with a byte count, empty barrier with four arrivals); four consumer warps
# each read their own 16 token rows of a page (scores from K, then P V from V)
# and arrive on the page's empty barrier; after the last page the warps pass
# the named barrier, write their (O, m, l) states into a combine scratch that
# aliases the start of the K ring, pass the named barrier again and read every
# warp's state.  Shared memory of the K ring is tracked in 256-byte chunks so
# the aliasing is exact for every head size, group size and cache type.

CC_MUTATIONS = (
    "empty_three_arrivals",    # a page slot freed after three of the four warps
    "release_before_pv",       # a warp frees the slot after its scores, before P V
    "no_barrier_before_combine",
    "no_barrier_after_combine",
    "full_parity",             # consumers wait with the page index as parity
    "ring_parity",             # producer waits on the slot's current phase
)

_CHUNK = 256


def simulate_cc(num_pages, d, gc, kv8, seed=0, mutation=None):
    """One CTA over `num_pages` cached pages (head size d, gc query heads per
    CTA, E4M3 cache if kv8).  Raises ProtocolError on any violation."""
    assert num_pages >= 1 and d in (64, 128) and gc in (1, 2, 4, 8)
    stages = 6 if kv8 else 3
    row_bytes = d * (1 if kv8 else 2)
    tile_bytes = 64 * row_bytes
    cmb_m = 4 * gc * d * 4
    cmb_l = cmb_m + 4 * gc * 4
    assert cmb_l + 4 * gc * 4 <= 2 * stages * tile_bytes
    sim = _Sim(seed)
    rng = sim.rng
    for s in range(stages):
        sim.bar(f"full{s}")
        sim.bar(f"empty{s}", 3 if mutation == "empty_three_arrivals" else 4)
    sim.bar("named", 4)

    def chunks(lo, hi):          # K-ring chunks covering bytes [lo, hi)
        return [f"k{c}" for c in range(lo // _CHUNK, (hi + _CHUNK - 1) // _CHUNK)]

    def rows(st, w):             # warp w's 16 token rows of slot st
        lo = st * tile_bytes + w * 16 * row_bytes
        return chunks(lo, lo + 16 * row_bytes)

    def producer():
        for i in range(num_pages):
            st = i % stages
            phase = i // stages if mutation == "ring_parity" else i // stages - 1
            yield ("wait", f"empty{st}", phase)
            # one byte count for both copies; each piece of the page lands on its own
            parts = [(c, ("K", i)) for w in range(4) for c in rows(st, w)] + \
                    [(f"v{st}_{w}", ("V", i)) for w in range(4)]
            yield ("expect_tx", f"full{st}", len(parts))
            for res, tag in parts:
                yield ("tma", f"full{st}", 1, res, tag)
            yield ("delay", rng.uniform(0.0, 0.2))

    def cmb_parts(w):
        o = chunks(w * gc * d * 4, (w + 1) * gc * d * 4)
        m = chunks(cmb_m + w * gc * 4, cmb_m + (w + 1) * gc * 4)
        l = chunks(cmb_l + w * gc * 4, cmb_l + (w + 1) * gc * 4)
        return sorted(set(o + m + l))

    def consumer(w):
        syncs = 0

        def named_sync():
            nonlocal syncs
            yield ("arrive", "named")
            yield ("wait", "named", syncs)
            syncs += 1

        for i in range(num_pages):
            st = i % stages
            yield ("wait", f"full{st}", i if mutation == "full_parity" else i // stages)
            for c in rows(st, w):
                yield ("read", c, ("K", i))
            yield ("delay", rng.uniform(0.2, 1.5))              # q . k for the warp's rows
            for c in rows(st, w):
                yield ("read", c, ("K", i))
            if mutation == "release_before_pv":
                yield ("arrive", f"empty{st}")
            yield ("read", f"v{st}_{w}", ("V", i))
            yield ("delay", rng.uniform(0.2, 1.5))              # softmax and P V
            yield ("read", f"v{st}_{w}", ("V", i))
            if mutation != "release_before_pv":
                yield ("arrive", f"empty{st}")
        if mutation != "no_barrier_before_combine":
            yield from named_sync()
        yield ("delay", rng.uniform(0.0, 0.5))
        for c in cmb_parts(w):
            yield ("write", c, ("combine",))
        if mutation != "no_barrier_after_combine":
            yield from named_sync()
        yield ("delay", rng.uniform(0.0, 0.3))
        for v in range(4):
            for c in cmb_parts(v):
                yield ("read", c, ("combine",))

    sim.add_role("producer", producer())
    for w in range(4):
        sim.add_role(f"consumer{w}", consumer(w))
    sim.run()


def random_cc_case(seed):
    """(num_pages, d, gc, kv8) over the kernel's configurations."""
    import random
    r = random.Random(2000 + seed)
    return r.choice([1, 2, 3, 4, 5, 6, 7, 9, 13, 20]), r.choice([64, 128]), r.choice([1, 2, 4, 8]), \
        r.random() < 0.5
