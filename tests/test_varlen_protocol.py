"""Model of the full-utterance attention kernel's mbarrier protocol (no GPU).

The kernel (chunked_block_self_b200/csrc/varlen_attn_sm100a.cu) runs one TMA
producer warp (each item's Q into one of two Q stages, then the utterance's
64-key K/V tiles into a ring), a V fix-up warp that releases each K/V stage
to the chains once it has landed, and four chains of four warps.  Every
chain walks every K/V tile of every item (a stage is freed by four
arrivals); a chain without query rows in an item only waits for each stage
to hold the item's data and releases it.  The chains learn each item, and
the end, from a ring of item descriptors that the producer fills (an entry
is freed by all sixteen chain warps: at once by a warp without rows in the
item, after the item's output otherwise).  Per tile a chain's first warp
waits for the stage and for its previous PV MMA, issues S, the chain's four
warps wait for S and write P, and the first warp issues PV.

A parity wait on an mbarrier answers correctly only for the barrier's
current phase or the one after it.  This model replays the kernel's waits,
arrivals and MMA commits (MMAs and TMA copies complete at random later
times, out of order too) under random interleavings, with every wait
carrying the absolute phase it means, and fails if a parity wait would
answer differently from the true one, if a barrier gets more arrivals in a
phase than its count, or if the roles deadlock.
"""
import random

import pytest

CHAINS, QROWS, KEYS = 4, 128, 64


class _Bar:
    def __init__(self, count):
        self.count, self.pending, self.phases = count, 0, 0

    def arrive(self):
        self.pending += 1
        assert self.pending <= self.count, "arrivals past the barrier's count"
        if self.pending == self.count:
            self.pending, self.phases = 0, self.phases + 1


def _simulate(items, nkv, seed, p_complete=0.3, p_out_of_order=0.2, early_release=False, ndesc=4):
    """items: (query rows L, utterance length T) of the CTA's items in order."""
    rnd = random.Random(seed)
    bars = {}

    def bar(name, count=1):
        return bars.setdefault(name, _Bar(count))

    for s in range(2):
        bar(f"q_full{s}"), bar(f"q_empty{s}", CHAINS)
    for s in range(nkv):
        bar(f"kv_full{s}"), bar(f"kv_ready{s}"), bar(f"kv_empty{s}", CHAINS)
    for c in range(CHAINS):
        bar(f"s_full{c}"), bar(f"wg_p{c}", 4), bar(f"o_done{c}")
    for j in range(ndesc):
        bar(f"desc_full{j}"), bar(f"desc_empty{j}", 4 * CHAINS)
    later = []   # async completions (TMA copies, MMA commits)

    def tiles(T):
        return (T + KEYS - 1) // KEYS

    def publish(n):
        j = n % ndesc
        if n >= ndesc:
            yield f"desc_empty{j}", n // ndesc - 1
        bars[f"desc_full{j}"].arrive()

    def producer():
        nkt = 0
        for nq, (L, T) in enumerate(items):
            yield from publish(nq)
            qs = nq & 1
            if nq >= 2:
                yield f"q_empty{qs}", (nq >> 1) - 1
            later.append(f"q_full{qs}")
            for _ in range(tiles(T)):
                s, u = nkt % nkv, nkt // nkv
                if u > 0:
                    yield f"kv_empty{s}", u - 1
                later.append(f"kv_full{s}")
                nkt += 1
        yield from publish(len(items))   # end marker

    def fixup():
        nkt = 0
        for L, T in items:
            for _ in range(tiles(T)):
                s = nkt % nkv
                yield f"kv_full{s}", nkt // nkv
                bars[f"kv_ready{s}"].arrive()
                nkt += 1

    def warp(c, leader):
        nkt, uses = 0, 0
        for n, (L, T) in enumerate(items):
            qs, nt = n & 1, tiles(T)
            dj = n % ndesc
            yield f"desc_full{dj}", n // ndesc
            if leader:
                yield f"q_full{qs}", n >> 1
            if L <= c * QROWS:
                # no rows of this chain: release the item's stages in order
                bars[f"desc_empty{dj}"].arrive()
                if leader:
                    bars[f"q_empty{qs}"].arrive()
                    for j in range(nt):
                        s = (nkt + j) % nkv
                        if not early_release:
                            yield f"kv_ready{s}", (nkt + j) // nkv
                        bars[f"kv_empty{s}"].arrive()
                nkt += nt
                continue
            for j in range(nt):
                s = nkt % nkv
                if leader:
                    yield f"kv_ready{s}", nkt // nkv
                    if uses > 0:
                        yield f"o_done{c}", uses - 1
                    later.append(f"s_full{c}")
                    if j == nt - 1:
                        later.append(f"q_empty{qs}")
                yield f"s_full{c}", uses
                bars[f"wg_p{c}"].arrive()
                if leader:
                    yield f"wg_p{c}", uses
                    later.append(f"o_done{c}")
                    later.append(f"kv_empty{s}")
                uses += 1
                nkt += 1
            yield f"o_done{c}", uses - 1
            bars[f"desc_empty{dj}"].arrive()   # the output step read the entry again
        n = len(items)
        yield f"desc_full{n % ndesc}", n // ndesc   # the end marker
        bars[f"desc_empty{n % ndesc}"].arrive()

    roles = {"producer": producer(), "fixup": fixup()}
    for c in range(CHAINS):
        for q in range(4):
            roles[f"c{c}w{q}"] = warp(c, q == 0)
    waiting = dict.fromkeys(roles)
    done = set()
    while len(done) < len(roles):
        ready = []
        for name in roles:
            if name in done:
                continue
            w = waiting[name]
            if w is None:
                ready.append(name)
                continue
            b = bars[w[0]]
            parity_says = (w[1] & 1) != (b.phases & 1)
            assert parity_says == (b.phases > w[1]), f"{name}: parity wait on {w} at phase {b.phases}"
            if parity_says:
                ready.append(name)
        if later and (not ready or rnd.random() < p_complete):
            bars[later.pop(rnd.randrange(len(later)) if rnd.random() < p_out_of_order else 0)].arrive()
            continue
        assert ready, f"deadlock: {[(k, waiting[k]) for k in roles if k not in done]}"
        name = rnd.choice(ready)
        waiting[name] = None
        try:
            waiting[name] = next(roles[name])
        except StopIteration:
            done.add(name)


def _items(rng, n):
    """A CTA's item sequence: (query rows, utterance length) with rows <= 512."""
    out = []
    for _ in range(n):
        T = rng.choice([1, 15, 64, 65, 127, 128, 129, 200, 257, 384, 513, 700])
        L = min(512, T - 512 * rng.randrange((T + 511) // 512))
        out.append((L, T))
    return out


@pytest.mark.parametrize("nkv", [2, 3, 5, 6])
def test_varlen_kernel_barrier_phases(nkv):
    rng = random.Random(nkv)
    for trial in range(150):
        items = _items(rng, rng.randint(1, 7))
        _simulate(items, nkv, trial)
        _simulate(items, nkv, trial, p_complete=0.05, p_out_of_order=1.0)


@pytest.mark.parametrize("ndesc", [1, 2, 3])
def test_shallow_descriptor_rings(ndesc):
    """The protocol holds for any ring depth (the kernel uses 4), up to one
    entry: the producer then waits for every chain warp's output step."""
    rng = random.Random(100 + ndesc)
    for trial in range(60):
        items = _items(rng, rng.randint(1, 7))
        _simulate(items, 3, trial, ndesc=ndesc)
        _simulate(items, 2, trial, p_complete=0.05, p_out_of_order=1.0, ndesc=ndesc)


def test_model_catches_an_early_stage_release():
    """A chain without rows that releases the item's K/V stages without first
    waiting for each to hold the item's data lets the producer refill a stage
    that other chains still read; the model must flag it."""
    rng = random.Random(7)
    caught = 0
    for trial in range(60):
        items = [(100, 700), (512, 700), (30, 300)] + _items(rng, 2)
        try:
            _simulate(items, 2, trial, p_complete=0.05, p_out_of_order=1.0, early_release=True)
        except AssertionError:
            caught += 1
    assert caught == 60   # every seeded trial
    _simulate([(100, 700), (512, 700), (30, 300)], 2, 0, p_complete=0.05, p_out_of_order=1.0)
