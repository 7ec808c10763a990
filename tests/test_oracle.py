"""Pins for the fp64 CPU oracle, against things other than the oracle itself.

* hand-worked block / window tables (tests/golden, each with its citation);
* a closed form (two keys -> logistic weights), at d = 1 and at d = 64 with
  the default scale 1/sqrt(d);
* the special case that reduces to a library routine: an utterance that fits
  in one block (window) is plain full softmax attention, compared with
  torch's scaled_dot_product_attention in float64;
* invariants: block locality, probabilities summing to one, permutation
  equivariance / invariance inside a block, packing invariance, the L = 1
  block copying V, equal keys averaging V over exactly the block.
"""
import json
import os

import numpy as np
import pytest
import torch

import oracle
from chunked_block_self_b200 import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _f64(x):
    return x.to(torch.float64)


def _sdpa(q, k, v, scale=None):
    """Library full attention: [L, H, d] bf16 -> float64 numpy [L, H, d]."""
    qh, kh, vh = (_f64(t).permute(1, 0, 2).unsqueeze(0) for t in (q, k, v))
    o = torch.nn.functional.scaled_dot_product_attention(qh, kh, vh, is_causal=False,
                                                         scale=scale)
    return o.squeeze(0).permute(1, 0, 2).numpy()


# ---------------------------------------------------------------- tables
def test_block_tables_golden():
    g = _load("block_tables.json")
    for case in g["cases"]:
        cu = wl.cu_seqlens(case["lengths"])
        seq, j, start, ln = oracle.block_table(cu, g["block_frames"])
        got = np.stack([seq, j, start, ln], 1).tolist() if len(seq) else []
        assert got == case["blocks"], case


def test_window_tables_golden():
    g = _load("window_tables.json")
    W, Q = g["window_frames"], g["queries_per_window"]
    for case in g["cases"]:
        cu = wl.cu_seqlens(case["lengths"])
        got = np.stack(oracle.window_table(cu, W, Q), 1).tolist()
        assert got == case["windows"], case
    lc = g["long_case"]
    t = oracle.window_table(wl.cu_seqlens(lc["lengths"]), W, Q)
    assert len(t[0]) == lc["n_windows"]
    assert [int(a[-1]) for a in t] == lc["last"]


def test_block_table_rejects_bad_offsets():
    with pytest.raises(ValueError):
        oracle.block_table(np.array([0, 5, 3], np.int32), 200)
    with pytest.raises(ValueError):
        oracle.block_table(np.array([1, 5], np.int32), 200)


# ---------------------------------------------------------------- closed forms
def test_two_key_closed_form_d1():
    g = _load("two_key_closed_form.json")
    q = torch.tensor([[[1.0]], [[2.0]]], dtype=torch.bfloat16)
    k = torch.tensor([[[1.0]], [[-1.0]]], dtype=torch.bfloat16)
    v = torch.tensor([[[1.0]], [[3.0]]], dtype=torch.bfloat16)
    o = oracle.block_attn(q, k, v, np.array([0, 2], np.int32), block_frames=2, scale=1.0)
    assert o[0, 0, 0] == pytest.approx(g["a1"], rel=1e-14)
    assert o[1, 0, 0] == pytest.approx(g["a2"], rel=1e-14)


def test_two_key_closed_form_default_scale_d64():
    g = _load("two_key_closed_form.json")
    d = 64
    q = torch.zeros(2, 1, d, dtype=torch.bfloat16)
    q[:, 0, 0] = 8.0
    k = torch.zeros(2, 1, d, dtype=torch.bfloat16)
    k[0, 0, 0], k[1, 0, 0] = 1.0, -1.0
    v = torch.ones(2, 1, d, dtype=torch.bfloat16)
    v[1] = 3.0
    o = oracle.block_attn(q, k, v, np.array([0, 2], np.int32), block_frames=200)
    np.testing.assert_allclose(o[:, 0, :], g["a1"], rtol=1e-14)


# ---------------------------------------------------------------- library case
@pytest.mark.parametrize("T", [1, 7, 150, 200])
def test_one_block_equals_full_attention(T):
    x = wl.block_inputs(lengths=[T], heads=3, seed=T)
    o = oracle.block_attn(x["q"], x["k"], x["v"], x["cu"], block_frames=200)
    ref = _sdpa(x["q"], x["k"], x["v"])
    np.testing.assert_allclose(o, ref, rtol=1e-11, atol=1e-12)


def test_each_block_is_full_attention_over_its_frames():
    # lengths [450, 30]: blocks [0,200) [200,400) [400,450) [450,480) (hand-cut)
    x = wl.block_inputs(lengths=[450, 30], heads=2, seed=3)
    o = oracle.block_attn(x["q"], x["k"], x["v"], x["cu"], block_frames=200, scale=0.3)
    for a, b in [(0, 200), (200, 400), (400, 450), (450, 480)]:
        ref = _sdpa(x["q"][a:b], x["k"][a:b], x["v"][a:b], scale=0.3)
        np.testing.assert_allclose(o[a:b], ref, rtol=1e-11, atol=1e-12)


def test_one_window_equals_full_cross_attention():
    # two utterances of 15 and 9 frames: one window each, query rows 0-2 / 3-5
    x = wl.window_inputs(6, cfg=None, lengths=[15, 9], heads=4, seed=2)
    o = oracle.window_xattn(x["q"], x["k"], x["v"], x["cu"], 15, 3)
    for (qa, qb), (ka, kb) in [((0, 3), (0, 15)), ((3, 6), (15, 24))]:
        ref = _sdpa(x["q"][qa:qb], x["k"][ka:kb], x["v"][ka:kb])
        np.testing.assert_allclose(o[qa:qb], ref, rtol=1e-11, atol=1e-12)


# ---------------------------------------------------------------- invariants
def test_single_frame_block_copies_v():
    x = wl.block_inputs(lengths=[201], heads=2, seed=5)
    o = oracle.block_attn(x["q"], x["k"], x["v"], x["cu"])
    np.testing.assert_array_equal(o[200], _f64(x["v"][200]).numpy())


def test_constant_v_gives_constant():
    x = wl.block_inputs(lengths=[260, 7], heads=2, seed=6)
    v = torch.empty_like(x["v"])
    v[:, 0, :] = 0.75
    v[:, 1, :] = -2.5
    o = oracle.block_attn(x["q"], x["k"], v, x["cu"])
    np.testing.assert_allclose(o[:, 0, :], 0.75, rtol=1e-14)
    np.testing.assert_allclose(o[:, 1, :], -2.5, rtol=1e-14)


def test_equal_keys_average_v_over_exactly_the_block():
    # lengths [250, 3, 401] -> blocks [0,200) [200,250) [250,253) [253,453) [453,653) [653,654)
    x = wl.block_inputs(lengths=[250, 3, 401], heads=2, seed=8)
    k = torch.empty_like(x["k"])
    k[:] = x["k"][0]
    o = oracle.block_attn(x["q"], k, x["v"], x["cu"])
    v = _f64(x["v"]).numpy()
    for a, b in [(0, 200), (200, 250), (250, 253), (253, 453), (453, 653), (653, 654)]:
        np.testing.assert_allclose(o[a:b], np.broadcast_to(v[a:b].mean(0), o[a:b].shape),
                                   rtol=1e-12, atol=1e-13)


def test_block_locality():
    x = wl.block_inputs(lengths=[530], heads=2, seed=9)
    o = oracle.block_attn(x["q"], x["k"], x["v"], x["cu"])
    q, k, v = x["q"].clone(), x["k"].clone(), x["v"].clone()
    for t in (q, k, v):  # perturb everything outside block 1 = [200, 400)
        t[:200] = -t[:200] * 3
        t[400:] = t[400:] + 1
    o2 = oracle.block_attn(q, k, v, x["cu"])
    np.testing.assert_array_equal(o2[200:400], o[200:400])
    assert np.abs(o2[:200] - o[:200]).max() > 1e-3
    assert np.abs(o2[400:] - o[400:]).max() > 1e-3


def test_probabilities_sum_to_one():
    x = wl.block_inputs(lengths=[90, 420], heads=3, seed=10)
    for row, head, ks, n in [(0, 0, 0, 90), (89, 2, 0, 90), (90, 1, 90, 200),
                             (350, 0, 290, 200), (509, 2, 490, 20)]:
        start, p, out = oracle.block_attn_probs(x["q"], x["k"], x["v"], x["cu"], row, head)
        assert (start, len(p)) == (ks, n)
        assert np.all(p >= 0)
        assert abs(p.sum() - 1.0) < 1e-12
        full = oracle.block_attn_rows(x["q"], x["k"], x["v"], x["cu"], [row], [head])
        np.testing.assert_array_equal(full[0], out)


def test_permutations_inside_a_block():
    x = wl.block_inputs(lengths=[200], heads=2, seed=11)
    o = oracle.block_attn(x["q"], x["k"], x["v"], x["cu"])
    rng = np.random.default_rng(0)
    pq = torch.from_numpy(rng.permutation(200))
    o_q = oracle.block_attn(x["q"][pq], x["k"], x["v"], x["cu"])
    np.testing.assert_allclose(o_q, o[pq.numpy()], rtol=1e-13, atol=1e-14)
    pk = torch.from_numpy(rng.permutation(200))
    o_kv = oracle.block_attn(x["q"], x["k"][pk], x["v"][pk], x["cu"])
    np.testing.assert_allclose(o_kv, o, rtol=1e-12, atol=1e-13)


def test_packing_invariance():
    lens = [17, 230, 0, 401]
    x = wl.block_inputs(lengths=lens, heads=2, seed=12)
    o = oracle.block_attn(x["q"], x["k"], x["v"], x["cu"])
    a = 0
    for t in lens:
        sub = oracle.block_attn(x["q"][a:a + t], x["k"][a:a + t], x["v"][a:a + t],
                                np.array([0, t], np.int32))
        np.testing.assert_array_equal(o[a:a + t], sub)
        a += t


def test_rows_and_threads_agree_with_full():
    x = wl.block_inputs(lengths=[333, 12, 250], heads=4, seed=13)
    o1 = oracle.block_attn(x["q"], x["k"], x["v"], x["cu"], n_threads=1)
    o8 = oracle.block_attn(x["q"], x["k"], x["v"], x["cu"], n_threads=0)
    np.testing.assert_array_equal(o1, o8)
    rows = np.array([0, 199, 200, 332, 333, 344, 345, 594])
    heads = np.array([0, 1, 2, 3, 0, 1, 2, 3])
    r = oracle.block_attn_rows(x["q"], x["k"], x["v"], x["cu"], rows, heads)
    np.testing.assert_array_equal(r, o1[rows, heads])


def test_window_locality_partial_window_and_rows():
    lens = [47, 15]
    # windows: [0,15) [15,30) [30,45) [45,47) | [47,62)  -> 5 windows, 15 query rows
    x = wl.window_inputs(15, cfg=None, lengths=lens, heads=2, seed=14)
    o = oracle.window_xattn(x["q"], x["k"], x["v"], x["cu"], 15, 3)
    ref = _sdpa(x["q"][9:12], x["k"][45:47], x["v"][45:47])  # the 2-frame window
    np.testing.assert_allclose(o[9:12], ref, rtol=1e-11, atol=1e-12)
    k = x["k"].clone()
    k[:45] += 2.0
    k[47:] *= -1
    o2 = oracle.window_xattn(x["q"], k, x["v"], x["cu"], 15, 3)
    np.testing.assert_array_equal(o2[9:12], o[9:12])
    r = oracle.window_xattn_rows(x["q"], x["k"], x["v"], x["cu"], [0, 5, 10, 14], [0, 1, 1, 0])
    np.testing.assert_array_equal(r, o[[0, 5, 10, 14], [0, 1, 1, 0]])


def test_window_equal_keys_average():
    lens = [20]  # windows [0,15) [15,20)
    x = wl.window_inputs(6, cfg=None, lengths=lens, heads=1, seed=15)
    k = torch.empty_like(x["k"])
    k[:] = x["k"][3]
    o = oracle.window_xattn(x["q"], k, x["v"], x["cu"], 15, 3)
    v = _f64(x["v"]).numpy()
    np.testing.assert_allclose(o[0:3], np.broadcast_to(v[0:15].mean(0), (3, 1, 64)),
                               rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(o[3:6], np.broadcast_to(v[15:20].mean(0), (3, 1, 64)),
                               rtol=1e-12, atol=1e-13)


def test_planted_mistake_is_caught():
    """A wrong scale in the oracle call must fail the library comparison."""
    x = wl.block_inputs(lengths=[64], heads=1, seed=16)
    o = oracle.block_attn(x["q"], x["k"], x["v"], x["cu"], scale=0.125 * 1.01)
    ref = _sdpa(x["q"], x["k"], x["v"])
    assert np.abs(o - ref).max() > 1e-4
