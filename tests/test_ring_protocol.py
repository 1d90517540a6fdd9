"""A model of the tensor-core prefill's package-ring protocol, run under random
interleavings (no GPU needed).

The kernel's chain CTAs run the sequence-heads ("chains") in rounds of P at a
time; position q of a round numbers the packages of its chain s = base_r + c,
base_r being the sum of the longest chain of every earlier round, and ring slot
s mod R of position q holds package s. A preparing CTA claims items in the
order (round, chunk, position), skips the numbers a chain shorter than its
round's longest does not have, waits until consumed[q][s mod R] >= slices *
(s div R) (every slice has read the slot's previous occupant), writes the
package and sets ready[q][s mod R] = s div R + 1. Each slice of a chain waits
for that value, reads the package and adds 1 to consumed; at the end of its
chain it also adds 1 for every number its chain leaves unused in the round.

The model checks, over many random problems and interleavings, that a slice
always reads the package it expects (never one written before or after it),
that every package is read by every slice exactly once and that the run never
deadlocks. It restates the protocol; it does not run the CUDA code.
"""
import random

import pytest


def ring_run(nch, P, S, R, n_prep, rng, wait_slices=None, bump_holes=True):
    """Simulate one launch; nch[j] = chunks of chain j. Returns the reads made.
    `wait_slices` (default S) is how many slices' reads a slot's reuse waits for;
    `bump_holes` whether a chain counts the numbers it leaves unused."""
    wait_slices = S if wait_slices is None else wait_slices
    chains = len(nch)
    n_rounds = (chains + P - 1) // P
    rounds = []   # (first chain, chains in round, longest chain, base)
    base = 0
    for r in range(n_rounds):
        j0, cpr = r * P, min(P, chains - r * P)
        maxc = max(nch[j0:j0 + cpr])
        rounds.append((j0, cpr, maxc, base))
        base += maxc
    items = [(r, c, q) for r, (j0, cpr, maxc, b) in enumerate(rounds) for c in range(maxc) for q in range(cpr)]

    slot = {}                     # (q, s mod R) -> package number held
    ready = {}                    # (q, s mod R) -> flag
    consumed = {}                 # (q, s mod R) -> count
    reads = []
    next_item = [0]

    def prep_agent():
        while True:
            while True:           # claim the next item that has a package
                if next_item[0] >= len(items):
                    return
                r, c, q = items[next_item[0]]
                next_item[0] += 1
                j0, cpr, maxc, b = rounds[r]
                if c < nch[j0 + q]:
                    break
            s = b + c
            key = (q, s % R)
            while consumed.get(key, 0) < wait_slices * (s // R):
                yield "wait"
            # (a number left unused by a short chain publishes nothing, so the flag may
            # lag behind s div R; it must never be ahead of it)
            assert ready.get(key, 0) <= s // R, "a slot was written for a later number first"
            slot[key] = s
            ready[key] = s // R + 1
            yield "step"

    def slice_agent(q, i):
        for r, (j0, cpr, maxc, b) in enumerate(rounds):
            if q >= cpr:
                return            # no chain at this position in this round (the last one)
            j = j0 + q
            for c in range(nch[j]):
                s = b + c
                key = (q, s % R)
                while ready.get(key, 0) < s // R + 1:
                    yield "wait"
                assert slot[key] == s, f"slice ({q}, {i}) expected package {s}, found {slot[key]}"
                reads.append((j, i, c))
                consumed[key] = consumed.get(key, 0) + 1
                yield "step"
            for c in range(nch[j], maxc if bump_holes else nch[j]):   # numbers left unused
                key = (q, (b + c) % R)
                consumed[key] = consumed.get(key, 0) + 1
            yield "step"

    agents = [prep_agent() for _ in range(n_prep)]
    agents += [slice_agent(q, i) for q in range(P) for i in range(S)]
    live = list(agents)
    stalled = 0
    while live:
        a = rng.choice(live)
        try:
            what = next(a)
        except StopIteration:
            live.remove(a)
            stalled = 0
            continue
        stalled = stalled + 1 if what == "wait" else 0
        if stalled > 50 * len(live) + 1000:
            raise AssertionError("deadlock: every live agent is waiting")
    return reads


def _check(nch, P, S, R, n_prep, seed):
    reads = ring_run(nch, P, S, R, n_prep, random.Random(seed))
    expected = sorted((j, i, c) for j, n in enumerate(nch) for i in range(S) for c in range(n))
    assert sorted(reads) == expected


@pytest.mark.parametrize("P,S,R,n_prep", [(1, 1, 2, 1), (2, 4, 3, 3), (4, 2, 12, 8), (3, 1, 5, 2), (16, 4, 12, 84)])
def test_equal_chains_in_rounds(P, S, R, n_prep):
    for seed in range(5):
        _check([40] * 7, P, S, R, n_prep, seed)


def test_random_lengths_holes_and_rounds():
    rng = random.Random(2024)
    for trial in range(150):
        chains = rng.randint(1, 12)
        nch = [rng.choice([0, 1, 2, 3, 5, 13, 26]) for _ in range(chains)]
        if max(nch) == 0:
            nch[0] = 1
        P = rng.randint(1, chains)
        S = rng.choice([1, 2, 4])
        R = rng.choice([1, 2, 3, 12])
        n_prep = rng.randint(1, 10)
        _check(nch, P, S, R, n_prep, seed=trial)


def test_the_model_catches_a_slot_reused_too_early():
    """The checks are sharp: if a slot's reuse waited for one slice fewer, some
    interleaving overwrites a package before its last reader gets to it."""
    caught = 0
    for seed in range(40):
        try:
            ring_run([30, 30, 30], 3, 4, 2, 4, random.Random(seed), wait_slices=3)
        except AssertionError:
            caught += 1
    assert caught > 0
    for seed in range(10):    # the real threshold never trips
        ring_run([30, 30, 30], 3, 4, 2, 4, random.Random(seed))


def test_the_model_reports_the_deadlock_of_uncounted_holes():
    """Without the end-of-chain count of unused numbers, a later round waits for
    ever on a slot whose previous number was a hole: the model must say so."""
    with pytest.raises(AssertionError, match="deadlock"):
        ring_run([3, 20, 20, 20], 2, 2, 4, 3, random.Random(1), bump_holes=False)
    ring_run([3, 20, 20, 20], 2, 2, 4, 3, random.Random(1))


# ------------------------------------------------ one chain CTA's mbarriers ---

class MBarrier:
    """An mbarrier as the kernel uses it: a phase completes when `count` arrivals
    have been made; a wait on parity P returns once the phase of that parity has
    completed, which it reads off the parity of the current phase -- so a waiter
    two phases behind sees its phase as not completed."""

    def __init__(self, count):
        self.count, self.pending, self.phase = count, count, 0

    def arrive(self):
        self.pending -= 1
        if self.pending == 0:
            self.phase += 1
            self.pending = self.count

    def test_wait(self, parity):
        return (self.phase & 1) != parity


def chain_cta_run(n_chunks, rng, releasing_warp_arrives=True, max_idle=5000, nb=2):
    """The issuing, releasing and compute warps of one chain CTA over nb input
    buffers (chunk gc in buffer gc % nb, its use number gc // nb giving the
    parity). A copy lands some time after it is issued (completing bar_full);
    the releasing warp counts each landed copy once; compute reads each chunk in
    order. Returns the chunks the releasing warp counted."""
    full = [MBarrier(1) for _ in range(nb)]
    free = [MBarrier(2 if releasing_warp_arrives else 1) for _ in range(nb)]
    in_flight = []            # buffers whose copy has been issued but has not landed
    counted = []

    def issuer():
        for gc in range(n_chunks):
            b = gc % nb
            if gc >= nb:
                while not free[b].test_wait(((gc - nb) // nb) & 1):
                    yield "wait"
            in_flight.append(b)
            yield "step"

    def lander():             # the asynchronous copies
        landed = 0
        while landed < n_chunks:
            if in_flight and rng.random() < 0.5:
                full[in_flight.pop(0)].arrive()
                landed += 1
                yield "step"
            else:
                yield "wait"

    def releaser():
        for gc in range(n_chunks):
            b = gc % nb
            while not full[b].test_wait((gc // nb) & 1):
                yield "wait"
            if releasing_warp_arrives:
                free[b].arrive()
            counted.append(gc)
            yield "step"

    def compute():
        for gc in range(n_chunks):
            b = gc % nb
            while not full[b].test_wait((gc // nb) & 1):
                yield "wait"
            for _ in range(rng.randint(0, 3)):   # the chunk's work
                yield "step"
            free[b].arrive()
            yield "step"

    live = [issuer(), lander(), releaser(), compute()]
    weights = [1, 1, 1 if releasing_warp_arrives else 0.02, 1]   # a releasing warp that may lag
    idle = 0
    while live:
        k = rng.choices(range(len(live)), weights=weights[:len(live)])[0]
        try:
            what = next(live[k])
        except StopIteration:
            live.pop(k)
            weights.pop(k)
            idle = 0
            continue
        idle = idle + 1 if what == "wait" else 0
        if idle > max_idle:
            raise AssertionError(f"hang: the releasing warp counted {len(counted)} of {n_chunks} chunks")
    return counted


@pytest.mark.parametrize("nb", [2, 3])
def test_chain_cta_releasing_warp_never_loses_a_phase(nb):
    for seed in range(200):
        assert chain_cta_run(24, random.Random(seed), nb=nb) == list(range(24))


def test_a_releasing_warp_that_does_not_gate_the_buffer_can_lose_a_phase():
    """Without its arrival on the free barrier, a releasing warp that lags a copy
    behind waits on a parity that has come round again: it misses that chunk's
    phase and ends up waiting for a copy that never comes."""
    hangs = 0
    for seed in range(60):
        try:
            chain_cta_run(24, random.Random(seed), releasing_warp_arrives=False)
        except AssertionError:
            hangs += 1
    assert hangs > 0


# --------------------------------- a prep CTA's queue and its publication ---

def prep_cta_run(n_chunks, P, R, K, rng, writer=True, max_idle=20000):
    """K preparing CTAs and P one-slice chains of n_chunks over a ring of R slots
    per chain. Each CTA's hand-over warp claims items into a two-entry queue
    (entry k & 1 is reused once item k - 2 is published) and waits for the
    item's slot; its compute warps stage item `it`'s package once the images of
    item it - 1 have been read, and its writing warp copies each staged package
    out and publishes it in order, on its own (writer). With writer=False the
    package is held until the compute warps start item it + 1 (publication in
    the next item's first stage), which can wait on the package's own slot.
    Returns the chains' reads."""
    items = [(c, q) for c in range(n_chunks) for q in range(P)]
    nxt = [0]
    ready, consumed, slot, reads = {}, {}, {}, []
    END = object()

    def make_cta():
        handed, staged, read, published = {}, set(), set(), set()

        def publish(k):
            c, q = handed[k]
            key = (q, c % R)
            slot[key] = c
            ready[key] = c // R + 1
            published.add(k)

        def hand_over():
            k = 0
            while True:
                while k >= 2 and (k - 2) not in published:
                    yield "wait"
                if nxt[0] >= len(items):
                    handed[k] = END
                    return
                c, q = items[nxt[0]]
                nxt[0] += 1
                while consumed.get((q, c % R), 0) < c // R:
                    yield "wait"
                handed[k] = (c, q)
                k += 1
                yield "step"

        def compute():
            it = 0
            while True:
                while it not in handed:
                    yield "wait"
                if not writer and it >= 1:
                    read.add(it - 1)
                    publish(it - 1)
                if handed[it] is END:
                    return
                while it >= 1 and (it - 1) not in read:
                    yield "wait"
                staged.add(it)
                it += 1
                yield "step"

        def write():
            it = 0
            while True:
                while it not in handed:
                    yield "wait"
                if handed[it] is END:
                    return
                while it not in staged:
                    yield "wait"
                read.add(it)
                yield "step"
                publish(it)
                it += 1
                yield "step"

        return [hand_over(), compute()] + ([write()] if writer else [])

    def chain(q):
        for c in range(n_chunks):
            key = (q, c % R)
            while ready.get(key, 0) < c // R + 1:
                yield "wait"
            assert slot[key] == c
            reads.append((q, c))
            consumed[key] = consumed.get(key, 0) + 1
            yield "step"

    live = [a for _ in range(K) for a in make_cta()] + [chain(q) for q in range(P)]
    idle = 0
    while live:
        a = rng.choice(live)
        try:
            what = next(a)
        except StopIteration:
            live.remove(a)
            idle = 0
            continue
        idle = idle + 1 if what == "wait" else 0
        if idle > max_idle:
            raise AssertionError("deadlock: a package waits to be published behind its own slot")
    return reads


@pytest.mark.parametrize("P,R,K", [(1, 1, 1), (1, 2, 1), (2, 1, 3), (3, 2, 2), (4, 12, 6)])
def test_prep_writer_publishes_every_package(P, R, K):
    for seed in range(20):
        reads = prep_cta_run(15, P, R, K, random.Random(seed))
        assert sorted(reads) == [(q, c) for q in range(P) for c in range(15)]


def test_publication_held_until_the_next_item_deadlocks_on_a_small_ring():
    with pytest.raises(AssertionError, match="deadlock"):
        prep_cta_run(15, 1, 1, 1, random.Random(0), writer=False)


# ------------------------------ a chain CTA's MMA warp and compute warps ---

def chain_mma_run(n_chunks, rng, max_idle=5000, separate_barriers=True):
    """The MMA warp and the eight compute warps of one chain CTA, each warp an
    agent of its own (no barrier across them). Per chunk the MMA warp waits for
    the 16-bit state copy of all eight warps (bar_s), issues Y and commits it,
    waits for U_s from the four U warps (bar_u), issues dS and commits it. With
    separate_barriers, Y commits to bar_y and dS to bar_ds; otherwise both to one
    barrier (the planted mistake for per-warp waits). A commit completes when its
    product finishes, some time later, in issue order. Each compute warp waits
    for Y, then (U warps) arrives on bar_u or (O warps) on bar_o, where the first
    O warp waits for all four before its store; then it waits for dS and arrives
    on bar_s. Every wait is by parity. Returns each warp's reads as (chunk,
    product, the latest completed product of that kind when it read)."""
    bar_y, bar_ds = MBarrier(1), MBarrier(1)
    if not separate_barriers:
        bar_ds = bar_y
    bar_u, bar_s, bar_o = MBarrier(4), MBarrier(8), MBarrier(4)
    issued = []               # products whose commit has not completed yet
    last = {}                 # kind -> the latest completed product
    seen = {w: [] for w in range(8)}

    def mma_warp():
        ph_s = ph_u = 0
        for gc in range(n_chunks):
            while not bar_s.test_wait(ph_s):
                yield "wait"
            ph_s ^= 1
            issued.append((gc, "Y"))
            yield "step"
            while not bar_u.test_wait(ph_u):
                yield "wait"
            ph_u ^= 1
            issued.append((gc, "dS"))
            yield "step"

    def tensor_core():
        n = 0
        while n < 2 * n_chunks:
            if issued and rng.random() < 0.4:
                gc, kind = issued.pop(0)
                last[kind] = gc
                (bar_y if kind == "Y" else bar_ds).arrive()
                n += 1
                yield "step"
            else:
                yield "wait"

    def compute(w):
        u_warp = w in (0, 1, 4, 5)
        ph_y = ph_ds = ph_o = 0
        bar_s.arrive()        # the first state copy
        for gc in range(n_chunks):
            while not bar_y.test_wait(ph_y):
                yield "wait"
            ph_y ^= 1
            seen[w].append((gc, "Y", last.get("Y")))
            yield "step"
            if u_warp:
                bar_u.arrive()
            else:
                bar_o.arrive()
                if w == 2:    # the storing O warp waits for the other three
                    while not bar_o.test_wait(ph_o):
                        yield "wait"
                ph_o ^= 1
            yield "step"
            while not bar_ds.test_wait(ph_ds):
                yield "wait"
            ph_ds ^= 1
            seen[w].append((gc, "dS", last.get("dS")))
            if gc + 1 < n_chunks:
                bar_s.arrive()
            yield "step"

    live = [mma_warp(), tensor_core()] + [compute(w) for w in range(8)]
    idle = 0
    while live:
        a = rng.choice(live)
        try:
            what = next(a)
        except StopIteration:
            live.remove(a)
            idle = 0
            continue
        idle = idle + 1 if what == "wait" else 0
        if idle > max_idle:
            raise AssertionError("hang in the chain CTA's MMA handshake")
    return seen


def test_chain_mma_handshake_each_warp_reads_each_product_once_in_order():
    """Y and dS on their own barriers, compute warps waiting independently: every
    warp sees each product as the latest completed one of its kind -- the next
    product of a kind cannot complete before every warp has arrived after reading
    this one -- and nothing hangs."""
    for seed in range(200):
        seen = chain_mma_run(12, random.Random(seed))
        for w in range(8):
            assert [(g, p) for g, p, _ in seen[w]] == [(g, p) for g in range(12) for p in ("Y", "dS")]
            for g, p, latest in seen[w]:
                assert latest == g, f"warp {w} read {p} of chunk {g} when chunk {latest}'s had completed"


def test_one_shared_commit_barrier_lets_a_lagging_warp_read_the_wrong_product():
    """With Y and dS on one barrier and no barrier across the compute warps, a
    warp that lags reads a later completion as the one it waits for (or waits
    for a phase that has come round again): the model must notice."""
    bad = 0
    for seed in range(300):
        try:
            seen = chain_mma_run(12, random.Random(seed), separate_barriers=False)
        except AssertionError:
            bad += 1
            continue
        for w in range(8):
            if [(g, p) for g, p, _ in seen[w]] != [(g, p) for g in range(12) for p in ("Y", "dS")] or \
                    any(latest != g for g, p, latest in seen[w]):
                bad += 1
                break
    assert bad > 0
