"""The library's host block/window plans are bit-identical to the oracle's
independent enumeration; shard plans cover the batch and balance cost."""
import json
import os

import numpy as np
import pytest

import oracle
from chunked_block_self_b200 import dp, nle
from chunked_block_self_b200 import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _cases():
    g = json.load(open(os.path.join(GOLDEN, "block_tables.json")))
    out = [c["lengths"] for c in g["cases"]]
    rng = np.random.default_rng(77)
    for _ in range(40):
        n = int(rng.integers(1, 40))
        out.append(list(rng.integers(0, 1300, n)))
    for cfg in (1, 2, 3, 4, 5):
        out.append(list(wl.draw_lengths(cfg)))
    return out


@pytest.mark.parametrize("B", [200, 1, 15, 128, 129, 256])
def test_block_plan_host_matches_oracle(B):
    for lens in _cases():
        cu = wl.cu_seqlens(lens)
        a = nle.nle_block_plan_host(cu, B)
        b = oracle.block_table(cu, B)
        for x, y in zip(a, b):
            np.testing.assert_array_equal(x, y)


def test_window_plan_host_matches_oracle():
    for lens in _cases():
        cu = wl.cu_seqlens(lens)
        a = nle.nle_window_plan_host(cu, 15, 3)
        b = oracle.window_table(cu, 15, 3)
        for x, y in zip(a, b):
            np.testing.assert_array_equal(x, y)
        assert nle.window_query_rows(cu, 15, 3) == 3 * len(b[0])


def test_window_plan_config5_counts():
    cu = wl.cu_seqlens(wl.draw_lengths(5))
    seq, w, start, ln, qrow = nle.nle_window_plan_host(cu, 15, 3)
    assert len(seq) == 64 * 314
    assert int((ln == 5).sum()) == 64 and int((ln == 15).sum()) == 64 * 313


def test_plan_rejects_bad_offsets():
    with pytest.raises(nle.NLEError):
        nle.nle_block_plan_host(np.array([0, 10, 5], np.int32), 200)
    with pytest.raises(nle.NLEError):
        nle.nle_block_plan_host(np.array([3, 10], np.int32), 200)


@pytest.mark.parametrize("world", [1, 2, 3, 8])
def test_shard_plan_covers_and_balances(world):
    lens = wl.draw_lengths(4)
    b = nle.nle_shard_plan_host(lens, world, 200)
    assert b[0] == 0 and b[-1] == len(lens) and np.all(np.diff(b) >= 0)
    cost = np.array([(t // 200) * 200.0 ** 2 + (t % 200) ** 2 for t in lens])
    per = np.array([cost[b[r]:b[r + 1]].sum() for r in range(world)])
    assert abs(per.sum() - cost.sum()) < 1e-6
    assert per.max() <= cost.sum() / world + cost.max()


def test_local_shard_rebases_offsets():
    cu = wl.cu_seqlens([5, 7, 0, 9])
    first, end, local = dp.local_shard(cu, [0, 2, 4], 1)
    assert (first, end) == (12, 21)
    np.testing.assert_array_equal(local, [0, 0, 9])
