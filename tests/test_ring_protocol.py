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
