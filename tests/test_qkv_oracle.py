"""Pins of the QKV-projection + block-attention oracle (oracle/qkv.py):
reductions to the pinned block-attention oracle, a hand-worked case in
closed form, bias and linearity properties, and a planted mistake."""
import math

import numpy as np
import torch

import oracle
from oracle import qkv
from chunked_block_self_b200 import workloads as wl


def _bf16(a):
    return torch.tensor(np.asarray(a, np.float32)).to(torch.bfloat16)


def test_fp64_block_attention_matches_the_c_oracle():
    x = wl.block_inputs(lengths=[230, 1, 57], heads=2, seed=41)
    want = oracle.block_attn(x["q"], x["k"], x["v"], x["cu"], block_frames=200)
    got = qkv.block_attn_f64(x["q"].double().numpy(), x["k"].double().numpy(), x["v"].double().numpy(),
                             x["cu"], 200)
    assert np.allclose(got, want, rtol=1e-12, atol=1e-12)


def test_identity_projection_reduces_to_block_attention():
    """D = 3*H*64 and W = I: Q, K and V are the three column blocks of X, so
    the result is the pinned block attention of those blocks."""
    H, lens = 2, [260, 40]
    rng = np.random.default_rng(42)
    T = sum(lens)
    x = _bf16(rng.standard_normal((T, 3 * H * 64)))
    w = _bf16(np.eye(3 * H * 64))
    cu = wl.cu_seqlens(lens)
    got = qkv.block_attn_qkv(x, w, cu, H)
    q, k, v = (x[:, i * H * 64:(i + 1) * H * 64].reshape(T, H, 64).contiguous() for i in range(3))
    want = oracle.block_attn(q, k, v, cu, block_frames=200)
    assert np.allclose(got, want, rtol=1e-12, atol=1e-12)


def test_swapped_weight_blocks_swap_the_operands():
    """Exchanging W's q and k row blocks is attention with Q and K exchanged;
    a projection that used W instead of W^T (the inverse permutation) would
    differ (planted below)."""
    H, lens = 1, [150]
    rng = np.random.default_rng(43)
    T = sum(lens)
    x = _bf16(rng.standard_normal((T, 3 * 64)))
    perm = np.concatenate([np.arange(64, 128), np.arange(0, 64), np.arange(128, 192)])
    cyc = np.concatenate([np.arange(64, 128), np.arange(128, 192), np.arange(0, 64)])   # not an involution
    cu = wl.cu_seqlens(lens)
    q, k, v = (x[:, i * 64:(i + 1) * 64].reshape(T, 1, 64).contiguous() for i in range(3))
    got = qkv.block_attn_qkv(x, _bf16(np.eye(192)[perm]), cu, H)
    assert np.allclose(got, oracle.block_attn(k, q, v, cu), rtol=1e-12, atol=1e-12)
    # W's row blocks (k, v, q): Q = K-block, K = V-block, V = Q-block
    got = qkv.block_attn_qkv(x, _bf16(np.eye(192)[cyc]), cu, H)
    want = oracle.block_attn(k, v, q, cu)
    assert np.allclose(got, want, rtol=1e-12, atol=1e-12)
    # planted mistake: X W (not X W^T) applies the inverse permutation
    xf, wf = x.double().numpy(), np.eye(192)[cyc]
    y = xf @ wf
    bad = qkv.block_attn_f64(y[:, :64].reshape(T, 1, 64), y[:, 64:128].reshape(T, 1, 64),
                             y[:, 128:].reshape(T, 1, 64), cu, 200)
    assert not np.allclose(bad, want, rtol=1e-6, atol=1e-6)


def test_hand_worked_single_feature():
    """d = 1, D = 1, W = [2, 1, 3]^T, X = [1, 2] (one block, scale 1):
    q = [2, 4], k = [1, 2], v = [3, 6]; row r's scores are q_r * k, so
    o_0 = 3 + 3 e^2 / (1 + e^2) and o_1 = 3 + 3 e^4 / (1 + e^4)."""
    x = _bf16([[1.0], [2.0]])
    w = _bf16([[2.0], [1.0], [3.0]])
    q, k, v = qkv.qkv_project(x, w, heads=1, d_head=1)
    out = qkv.block_attn_f64(q, k, v, [0, 2], 200, scale=1.0)
    e2, e4 = math.exp(2.0), math.exp(4.0)
    assert np.allclose(out[:, 0, 0], [3 + 3 * e2 / (1 + e2), 3 + 3 * e4 / (1 + e4)], rtol=1e-14)


def test_bias_and_linearity():
    H, lens = 2, [90, 210]
    rng = np.random.default_rng(44)
    T, D = sum(lens), H * 64
    cu = wl.cu_seqlens(lens)
    x = _bf16(rng.standard_normal((T, D)))
    w = rng.standard_normal((3 * D, D)) * 0.05
    w[2 * D:] = 0.0
    bias = np.zeros(3 * D)
    bias[2 * D:] = rng.integers(-3, 4, D)          # V = the bias: every row's output is it
    out = qkv.block_attn_qkv(x, _bf16(w), cu, H, bias=bias)
    assert np.allclose(out, np.broadcast_to(bias[2 * D:].reshape(H, 64), out.shape), rtol=0, atol=1e-12)
    # doubling W_v (exact in bf16) doubles the output
    w = rng.standard_normal((3 * D, D)) * 0.05
    w2 = w.copy()
    w2[2 * D:] *= 2.0
    a = qkv.block_attn_qkv(x, _bf16(w), cu, H)
    b = qkv.block_attn_qkv(x, _bf16(w2), cu, H)
    assert np.allclose(b, 2.0 * a, rtol=1e-12, atol=1e-12)
