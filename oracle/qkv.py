"""QKV projection followed by block self-attention -- TEST INFRASTRUCTURE ONLY.

Written from the model card, "Model Architecture" (1) CTC Speech Encoder:
each conformer layer's self-attention projects the layer's hidden states to
queries, keys and values and attends within 4 s blocks.  This is the fused
step that starts from the hidden states X instead of from Q, K and V.

Readings taken where the pages are silent:
- X is bf16 [T_total, D] (D = heads x 64 = 1024 for the encoder), frame-major;
- the projection weight is one bf16 matrix W [3 * heads * 64, D] in the
  layout of a linear layer (output features x input features): rows
  [0, H*64) give Q, [H*64, 2*H*64) K and [2*H*64, 3*H*64) V, head h taking
  the 64 rows h*64 .. h*64+63 of each; Q = X W_q^T (+ b_q), and so on;
- no bias unless one is given (the pages do not say whether the layers
  have one);
- the attention is the block definition of the block kernel (200-frame
  blocks cut per utterance, scale 1/sqrt(64), no positional term).

Everything is float64 from the exact bf16 inputs.  Only the test suite
uses this module; it shares no code with the CUDA library.
"""
from __future__ import annotations

import numpy as np

from .ctc import _as_f64


def qkv_project(x, w_qkv, heads: int, d_head: int = 64, bias=None):
    """(Q, K, V), each float64 [T, heads, d_head]: X W^T (+ bias), split into
    the q, k and v row blocks of W and then into heads."""
    xf = _as_f64(x)
    wf = _as_f64(w_qkv)
    hd = heads * d_head
    if wf.shape != (3 * hd, xf.shape[1]):
        raise ValueError("w_qkv must be [3 * heads * d_head, D]")
    y = xf @ wf.T
    if bias is not None:
        y = y + np.asarray(bias, np.float64)[None, :]
    t = xf.shape[0]
    return tuple(y[:, i * hd:(i + 1) * hd].reshape(t, heads, d_head) for i in range(3))


def block_attn_f64(q, k, v, cu, block_frames: int = 200, scale: float | None = None) -> np.ndarray:
    """Block self-attention on float64 Q, K, V [T, H, d]: for each block of
    each utterance and each head, softmax(scale * Q K^T) V over the block."""
    q, k, v = (np.asarray(a, np.float64) for a in (q, k, v))
    d = q.shape[2]
    scale = 1.0 / np.sqrt(d) if scale is None else scale
    out = np.zeros_like(q)
    cu = np.asarray(cu, np.int64)
    for i in range(len(cu) - 1):
        s0, e0 = int(cu[i]), int(cu[i + 1])
        for a in range(s0, e0, block_frames):
            b = min(a + block_frames, e0)
            for h in range(q.shape[1]):
                s = scale * q[a:b, h] @ k[a:b, h].T
                s -= s.max(axis=1, keepdims=True)
                p = np.exp(s)
                p /= p.sum(axis=1, keepdims=True)
                out[a:b, h] = p @ v[a:b, h]
    return out


def block_attn_qkv(x, w_qkv, cu, heads: int, block_frames: int = 200, bias=None,
                   scale: float | None = None) -> np.ndarray:
    """O [T, heads, 64] float64 of block self-attention of X's projections."""
    q, k, v = qkv_project(x, w_qkv, heads, bias=bias)
    return block_attn_f64(q, k, v, cu, block_frames, scale)
