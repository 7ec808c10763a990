"""Pins of the CTC greedy-decoding oracle (oracle/ctc.py) against hand-worked
cases and properties that hold whatever the implementation."""
import itertools
import json
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "ctc_greedy.json")


def _bf16_bits(a):
    f = np.asarray(a, np.float32)
    bits = f.view(np.uint32)
    assert np.all((bits & 0xFFFF) == 0), "fixture values must be exact in bf16"
    return (bits >> 16).astype(np.uint16)


@pytest.mark.parametrize("case", json.load(open(GOLDEN))["cases"], ids=lambda c: c["name"])
def test_golden(case):
    cls, toks = oracle.ctc_greedy(_bf16_bits(case["logits"]), case["cu"])
    assert cls.tolist() == case["classes"]
    assert toks == case["tokens"]


def _random_case(rng, n_utt, n_cls):
    lens = rng.integers(0, 40, n_utt)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    # few distinct values so that ties and repeated classes are common
    vals = rng.integers(-3, 4, (int(cu[-1]), n_cls)).astype(np.float32)
    return cu, vals


def test_matches_run_length_formulation():
    """Greedy CTC as the textbook run-length rule: split each utterance's
    class sequence into maximal runs, keep one class per run, drop blanks."""
    rng = np.random.default_rng(1)
    for _ in range(50):
        cu, vals = _random_case(rng, int(rng.integers(1, 6)), int(rng.integers(2, 7)))
        cls, toks = oracle.ctc_greedy(_bf16_bits(vals), cu)
        for u in range(len(cu) - 1):
            seq = cls[cu[u]:cu[u + 1]].tolist()
            runs = [c for c, _ in itertools.groupby(seq)]
            assert toks[u] == [c - 1 for c in runs if c != 0]


def test_argmax_is_first_maximum_and_shift_invariant():
    rng = np.random.default_rng(2)
    cu, vals = _random_case(rng, 4, 9)
    cls = oracle.ctc_frame_classes(_bf16_bits(vals))
    for i, row in enumerate(vals):
        m = row.max()
        assert row[cls[i]] == m and np.all(row[:cls[i]] < m)
    # adding a per-frame constant (exact in bf16 here) does not change the classes
    shifted = vals + rng.integers(-2, 3, (len(vals), 1)).astype(np.float32)
    assert np.array_equal(oracle.ctc_frame_classes(_bf16_bits(shifted)), cls)


def test_token_counts_bounded_and_no_blank_token():
    rng = np.random.default_rng(3)
    cu, vals = _random_case(rng, 8, 5)
    _, toks = oracle.ctc_greedy(_bf16_bits(vals), cu)
    for u, t in enumerate(toks):
        assert len(t) <= cu[u + 1] - cu[u]
        assert all(0 <= x <= 3 for x in t)   # classes 1..4 -> tokens 0..3; blank never emitted


def test_planted_mistake_is_caught():
    """Collapsing across the utterance boundary (a plausible slip) must fail
    the boundary fixture."""
    case = json.load(open(GOLDEN))["cases"][2]
    cls = oracle.ctc_frame_classes(_bf16_bits(case["logits"]))
    wrong = oracle.ctc_collapse(cls, [0, len(cls)])      # boundary ignored
    flat = [t for u in case["tokens"] for t in u]
    assert wrong[0] != flat


# Non-finite and signed-zero logits, worked by hand.  Reading taken where the
# page is silent: a NaN logit is no candidate; a frame of NaNs only takes the
# blank; -0 and +0 are equal (the lower class wins); infinities order as usual.
NONFINITE = [
    ([np.nan, 1.0, 1.0], 1),
    ([np.nan, np.nan, np.nan], 0),
    ([np.nan, -np.inf, -np.inf], 1),
    ([-np.inf, np.nan], 0),
    ([-np.inf, -np.inf, -np.inf], 0),
    ([2.0, np.inf, np.nan, np.inf], 1),
    ([-0.0, 0.0, -1.0], 0),
    ([-1.0, 0.0, -0.0], 1),
    ([np.nan, -3.0, np.nan, -2.0, np.nan], 3),
]


@pytest.mark.parametrize("row,cls", NONFINITE)
def test_nonfinite_and_signed_zero(row, cls):
    assert oracle.ctc_frame_classes(_bf16_bits([row])).tolist() == [cls]


def _brute_force_class(row):
    """Per-frame class by a plain scan: the first non-NaN logit that no later
    non-NaN logit exceeds (strictly), the blank when every logit is NaN."""
    best, cls = None, 0
    for c, z in enumerate(row):
        if z != z:          # NaN: no candidate
            continue
        if best is None or z > best:
            best, cls = z, c
    return cls


def test_frame_classes_match_a_plain_scan_on_small_rows():
    """The array formulation against a pure-Python scan on tiny rows that mix
    NaN, +-inf, -0/+0 and ties, over several pass sizes (including rows
    split across passes)."""
    rng = np.random.default_rng(17)
    pool = np.array([np.nan, np.inf, -np.inf, -0.0, 0.0, 1.0, -1.0, 2.0], np.float32)
    for n_cls in (1, 2, 3, 5, 9):
        vals = rng.choice(pool, size=(64, n_cls))
        want = [_brute_force_class(r.tolist()) for r in vals]
        for per_pass in (1, 7, 256):
            got = oracle.ctc_frame_classes(_bf16_bits(vals), rows_per_pass=per_pass)
            assert got.tolist() == want
