"""Pins of the posterior-weighted pooling oracle (oracle/pool.py): hand-worked
fixtures, the row count the ONNX README's parity table prints, an
independent library softmax, closed forms and invariants."""
import json
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
from chunked_block_self_b200 import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "posterior_pool.json")


def _bf16(a):
    import torch
    return torch.tensor(np.asarray(a, np.float32)).to(torch.bfloat16)


def _num(x):
    return float("-inf") if x == "-inf" else float(x)


@pytest.mark.parametrize("case", json.load(open(GOLDEN))["cases"], ids=lambda c: c["name"])
def test_golden(case):
    logits = _bf16([[_num(v) for v in row] for row in case["logits"]])
    hidden = _bf16(case["hidden"])
    pooled, w = oracle.posterior_pool(hidden, logits, case["cu"], case["pool_frames"])
    assert np.allclose(w, [float(Fraction(x)) for x in case["weights"]], rtol=1e-13, atol=1e-15)
    want = np.array([[float(Fraction(x)) for x in row] for row in case["pooled"]])
    assert pooled.shape == want.shape
    assert np.allclose(pooled, want, rtol=1e-13, atol=1e-13)


def test_row_count_of_the_parity_clip():
    """The ONNX README's parity clip: 844 mel frames -> 422 encoder frames ->
    211 rows of the BPE head with windows of 2 encoder frames."""
    assert oracle.pooled_rows([0, 422], 2)[-1] == 211
    assert oracle.pooled_rows([0, 5, 5, 9, 10], 2).tolist() == [0, 3, 3, 5, 6]
    assert oracle.pooled_rows([0, 5, 5, 9, 10], 4).tolist() == [0, 2, 2, 3, 4]


def test_weights_against_library_softmax():
    from scipy.special import softmax
    rng = np.random.default_rng(1)
    z = (rng.standard_normal((40, 37)) * 3).astype(np.float32)
    z = _bf16(z)
    p = softmax(z.float().double().numpy(), axis=1)
    assert np.allclose(oracle.blank_weights(z), 1.0 - p[:, 0], rtol=1e-12, atol=1e-14)


def test_far_apart_logits_keep_their_weight_ratio():
    """A blank logit 900 above the rest: w = C' e^-900, below float64's range,
    yet a window of two such frames is still their (exact) weighted mean."""
    z = np.full((2, 4), 0.0, np.float32)
    z[:, 0] = 896.0                       # exact in bf16
    z[1, 1:] = [1.0, -np.inf, -np.inf]    # frame 1: one non-blank class at 1
    h = np.array([[1.0, 0.0], [0.0, 1.0]], np.float32)
    pooled, _ = oracle.posterior_pool(_bf16(h), _bf16(z), [0, 2], 2)
    # log w0 = log 3 - 896, log w1 = 1 - 896 (to within e^-895): ratio w1/w0 = e/3
    r = np.e / 3.0
    assert np.allclose(pooled[0], [1 / (1 + r), r / (1 + r)], rtol=1e-12)


def test_equal_weights_give_the_plain_mean():
    rng = np.random.default_rng(2)
    T, D = 23, 16
    h = _bf16(rng.standard_normal((T, D)))
    z = _bf16(np.tile(rng.standard_normal(9), (T, 1)))   # every frame the same logits
    pooled, _ = oracle.posterior_pool(h, z, [0, T], 4)
    hf = h.float().double().numpy()
    want = np.stack([hf[a:a + 4].mean(axis=0) for a in range(0, T, 4)])
    assert np.allclose(pooled, want, rtol=1e-13, atol=1e-13)


def test_pool_of_one_frame_is_the_frame_or_zero():
    rng = np.random.default_rng(3)
    T, D = 9, 8
    h = _bf16(rng.standard_normal((T, D)))
    z = rng.standard_normal((T, 5)).astype(np.float32)
    z[4, 1:] = -np.inf   # weight 0
    pooled, w = oracle.posterior_pool(h, _bf16(z), [0, T], 1)
    hf = h.float().double().numpy()
    assert w[4] == 0.0 and np.all(pooled[4] == 0.0)
    keep = np.arange(T) != 4
    assert np.array_equal(pooled[keep], hf[keep])


def test_invariants_shift_permutation_packing():
    rng = np.random.default_rng(4)
    lens = [7, 0, 1, 12, 5]
    cu = wl.cu_seqlens(lens)
    T, D = int(cu[-1]), 6
    h = _bf16(rng.standard_normal((T, D)))
    zf = rng.integers(-4, 5, (T, 7)).astype(np.float32)
    pooled, w = oracle.posterior_pool(h, _bf16(zf), cu, 3)
    # a per-frame constant added to every logit changes no weight
    _, w2 = oracle.posterior_pool(h, _bf16(zf + rng.integers(-3, 4, (T, 1))), cu, 3)
    assert np.allclose(w, w2, rtol=1e-13, atol=1e-15)
    # swapping two frames inside one window (frames 0 and 2 of utterance 0)
    perm = np.arange(T)
    perm[[0, 2]] = perm[[2, 0]]
    p3, _ = oracle.posterior_pool(h[perm], _bf16(zf[perm]), cu, 3)
    assert np.allclose(p3, pooled, rtol=1e-13, atol=1e-13)
    # the packed batch is the per-utterance results stacked
    rows = oracle.pooled_rows(cu, 3)
    for i in range(len(lens)):
        a, b = int(cu[i]), int(cu[i + 1])
        pi, _ = oracle.posterior_pool(h[a:b], _bf16(zf[a:b]), [0, b - a], 3)
        assert np.array_equal(pi, pooled[rows[i]:rows[i + 1]])


def test_planted_mistakes_are_caught():
    """p_blank used in place of 1 - p_blank, and windows counted from the
    batch start instead of each utterance's, both fail the first fixture."""
    case = json.load(open(GOLDEN))["cases"][0]
    logits = _bf16([[_num(v) for v in row] for row in case["logits"]])
    hidden = _bf16(case["hidden"])
    want = np.array([[float(Fraction(x)) for x in row] for row in case["pooled"]])
    w_bad = 1.0 - oracle.blank_weights(logits)          # = p_blank
    hf = hidden.float().double().numpy()
    cu = case["cu"]
    bad = []
    for i in range(len(cu) - 1):
        for a in range(cu[i], cu[i + 1], 2):
            b = min(a + 2, cu[i + 1])
            s = w_bad[a:b].sum()
            bad.append((w_bad[a:b, None] * hf[a:b]).sum(0) / s if s > 0 else np.zeros(2))
    assert not np.allclose(np.array(bad), want)
    # windows from the batch start: [0,2) [2,4) [4,6) [6,8) -- a different row set
    whole, _ = oracle.posterior_pool(hidden, logits, [0, 8], 2)
    assert whole.shape != want.shape or not np.allclose(whole, want)
