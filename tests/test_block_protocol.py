"""Model of the block-attention kernel's mbarrier protocol (no GPU).

The kernel (chunked_block_self_b200/csrc/block_attn_sm100a.cu) runs one Q/K
producer warp, one V producer warp and two tile warpgroups that take
alternate items; each warpgroup computes row tile 0 and, for blocks longer
than 128 frames, row tile 1 of its items.  Stages of the QK and V rings are
refilled when the item's last S / last PV MMA completes.

A parity wait on an mbarrier answers correctly only for the barrier's current
phase or the one after it.  This model replays the kernel's waits, arrivals
and MMA commits (MMAs and TMA copies complete at random later times) under
random interleavings, with every wait carrying the absolute phase it means,
and fails if a parity wait would answer differently from the true one, or if
the roles deadlock.  Ring depths are even, as the host code chooses them.
"""
import random

import pytest


class _Bar:
    def __init__(self, count):
        self.count, self.pending, self.phases = count, 0, 0

    def arrive(self):
        self.pending += 1
        assert self.pending <= self.count
        if self.pending == self.count:
            self.pending, self.phases = 0, self.phases + 1


def _simulate(lengths, sqk, nsv, seed, p_complete=0.3, p_out_of_order=0.2):
    rnd = random.Random(seed)
    bars = {}

    def bar(name, count=1):
        return bars.setdefault(name, _Bar(count))

    for s in range(sqk):
        bar(f"qk_full{s}"), bar(f"qk_empty{s}")
    for s in range(nsv):
        bar(f"v_full{s}"), bar(f"v_empty{s}")
    for t in range(2):
        bar(f"s_full{t}"), bar(f"wg_p{t}", 4), bar(f"o_full{t}"), bar(f"wg_o{t}", 4)
    later = []          # async completions (TMA copies, MMA commits)
    n_items = len(lengths)

    def producer(kind, depth):
        for n in range(n_items):
            s, u = n % depth, n // depth
            if u > 0:
                yield f"{kind}_empty{s}", u - 1
            later.append(f"{kind}_full{s}")

    def warp(t, leader):
        next_n, n, x, L, uses = 0, -1, 1, 0, 0
        while True:
            if not (x == 0 and L > 128):          # the warpgroup's next item
                while next_n < n_items and next_n % 2 != t:
                    next_n += 1
                if next_n >= n_items:
                    return
                n, L, x = next_n, lengths[next_n], 0
                next_n += 1
            else:                                   # row tile 1 of the item
                x = 1
            last_tile = x == 1 or L <= 128
            if leader:
                if x == 0:
                    yield f"qk_full{n % sqk}", n // sqk
                if uses > 0:
                    yield f"wg_o{t}", uses - 1
                later.append(f"s_full{t}")
                if last_tile:
                    later.append(f"qk_empty{n % sqk}")
            yield f"s_full{t}", uses
            bars[f"wg_p{t}"].arrive()
            if leader:
                yield f"wg_p{t}", uses
                if x == 0:
                    yield f"v_full{n % nsv}", n // nsv
                later.append(f"o_full{t}")
                if last_tile:
                    later.append(f"v_empty{n % nsv}")
            yield f"o_full{t}", uses
            bars[f"wg_o{t}"].arrive()
            uses += 1

    roles = {"qk": producer("qk", sqk), "v": producer("v", nsv)}
    for t in range(2):
        for q in range(4):
            roles[f"w{t}{q}"] = warp(t, q == 0)
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


@pytest.mark.parametrize("sqk,nsv", [(2, 2), (2, 4), (4, 2), (4, 4)])
def test_block_kernel_barrier_phases(sqk, nsv):
    rng = random.Random(sqk * 10 + nsv)
    for trial in range(400):
        lengths = [rng.choice([200, 193, 192, 150, 129, 128, 100, 40, 16, 1])
                   for _ in range(rng.randint(1, 14))]
        _simulate(lengths, sqk, nsv, trial)
        _simulate(lengths, sqk, nsv, trial, p_complete=0.05, p_out_of_order=1.0)


def test_model_catches_a_stage_shared_by_both_warpgroups():
    """With an odd V ring a stage serves both warpgroups' items, and a
    warpgroup that only waits on its own items' phases can run two phases
    ahead of the stage's barrier when copies complete late and out of order.
    The model must flag these cases (found by a seeded search)."""
    cases = [(157, [40, 150, 40, 40, 40, 100, 100, 200]),
             (455, [40, 100, 100, 40, 40, 100, 40, 150, 100, 150, 40, 200]),
             (523, [40, 100, 200, 40, 100, 40, 40, 100, 150])]
    for seed, lengths in cases:
        with pytest.raises(AssertionError, match="parity wait"):
            _simulate(lengths, 2, 3, seed, p_complete=0.05, p_out_of_order=1.0)
        _simulate(lengths, 2, 4, seed, p_complete=0.05, p_out_of_order=1.0)   # even ring: fine


def test_split_items_meet_the_protocol():
    """Split work items (one row tile each, for batches that do not fill the
    GPU) meet the protocol as items of at most 128 rows: a block of L > 128
    frames becomes two items, of 128 and L - 128 rows."""
    rng = random.Random(77)
    for trial in range(200):
        blocks = [rng.choice([200, 193, 150, 129, 128, 100, 40, 1]) for _ in range(rng.randint(1, 10))]
        items = []
        for L in blocks:
            items.append(min(L, 128))
            if L > 128:
                items.append(L - 128)
        _simulate(items, 2, 4, trial)
        _simulate(items, 2, 2, trial, p_complete=0.05, p_out_of_order=1.0)
