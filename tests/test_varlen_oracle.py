"""Pins of the full-utterance attention oracle (no blocks; the editor's
bidirectional attention, model card "Model Architecture" (3)) against
numpy's full softmax attention and invariants."""
import numpy as np

import oracle
from chunked_block_self_b200 import workloads as wl


def _f64(t):
    return t.float().double().numpy()


def _numpy_full(q, k, v, cu, scale):
    q, k, v = _f64(q), _f64(k), _f64(v)
    out = np.zeros_like(q)
    for i in range(len(cu) - 1):
        a, b = int(cu[i]), int(cu[i + 1])
        for h in range(q.shape[1] if b > a else 0):
            s = scale * q[a:b, h] @ k[a:b, h].T
            s -= s.max(axis=1, keepdims=True)
            p = np.exp(s)
            p /= p.sum(axis=1, keepdims=True)
            out[a:b, h] = p @ v[a:b, h]
    return out


def test_long_utterances_equal_numpy_full_attention():
    lens = [517, 1, 0, 300, 129]
    x = wl.block_inputs(None, seed=5, lengths=lens, heads=2)
    got = oracle.varlen_attn(x["q"], x["k"], x["v"], x["cu"])
    want = _numpy_full(x["q"], x["k"], x["v"], x["cu"], 0.125)
    assert np.allclose(got, want, rtol=1e-12, atol=1e-12)


def test_rows_match_whole_and_other_utterances_do_not_leak():
    lens = [400, 250]
    x = wl.block_inputs(None, seed=6, lengths=lens, heads=2)
    full = oracle.varlen_attn(x["q"], x["k"], x["v"], x["cu"])
    rows = [0, 399, 400, 649, 123]
    heads = [0, 1, 1, 0, 1]
    r = oracle.varlen_attn_rows(x["q"], x["k"], x["v"], x["cu"], rows, heads)
    assert np.array_equal(r, full[rows, heads])
    # utterance 1 changed entirely: utterance 0 unchanged, bit for bit
    k2 = x["k"].clone()
    k2[400:] = -k2[400:]
    again = oracle.varlen_attn(x["q"], k2, x["v"], x["cu"])
    assert np.array_equal(again[:400], full[:400])
    assert not np.allclose(again[400:], full[400:])


def test_packing_invariance():
    lens = [230, 31, 257]
    x = wl.block_inputs(None, seed=7, lengths=lens, heads=1)
    full = oracle.varlen_attn(x["q"], x["k"], x["v"], x["cu"])
    cu = x["cu"]
    for i in range(len(lens)):
        a, b = int(cu[i]), int(cu[i + 1])
        one = oracle.varlen_attn(x["q"][a:b], x["k"][a:b], x["v"][a:b], [0, b - a])
        assert np.array_equal(one, full[a:b])
