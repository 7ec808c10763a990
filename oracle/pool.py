"""Posterior-weighted pooling for the BPE CTC head -- TEST INFRASTRUCTURE ONLY.

Written from the model card, "Model Architecture" (1) CTC Speech Encoder: the
BPE head pools the encoder's frames over windows of size 4, each frame
weighted by an importance weight of 1 - blank probability, the blank
probability coming from the mid-layer (character) CTC head.

Readings taken where the page is silent:
- the window of 4 counts 10 ms input (log-mel) frames.  Two-frame stacking
  puts the encoder at 50 Hz, so a window is 2 encoder frames.  The ONNX
  README's parity table supports this: an 8.43 s clip of 844 mel frames (422
  encoder frames) gives 211 rows of `bpe_logits_dense`.  The window, in
  encoder frames, is the parameter `pool_frames`;
- windows are cut per utterance from its frame 0 and do not overlap; the
  last one may be partial; window g of the packed batch is pooled row g;
- the blank is class 0 of the mid-layer head, and its probability is the
  softmax over that head's classes, so w_t = 1 - p_blank(t) =
  sum_{c>=1} exp(z_c) / sum_c exp(z_c).  The weight is 0 when every
  non-blank logit is -inf;
- a pooled row is the weighted mean sum_t w_t h_t / sum_t w_t over the
  window's frames.  A window whose weights are all 0 gives a zero row;
- hidden states and logits are bf16 inputs, widened exactly; the oracle
  works in float64.  Weights are formed in the log domain,
  log w_t = logsumexp(z[1:]) - logsumexp(z), and the mean divides
  exp(log w_t - max log w) by its sum.  That is the same quantity without
  underflow when logits are far apart.  Logits are finite or -inf (NaN and
  +inf are outside the definition).

Only the test suite, the smoke check and the bench use this module; it
shares no code with the CUDA library.
"""
from __future__ import annotations

import numpy as np

from .ctc import _as_f64


def _logsumexp(x: np.ndarray) -> float:
    m = np.max(x) if x.size else -np.inf
    if m == -np.inf:
        return -np.inf
    return float(m + np.log(np.sum(np.exp(x - m))))


def log_weights(logits) -> np.ndarray:
    """log(1 - p_blank) of each frame ([T, C] -> [T] float64, -inf for a
    weight of 0)."""
    z = _as_f64(logits)
    out = np.empty(z.shape[0])
    for t in range(z.shape[0]):
        nb = _logsumexp(z[t, 1:])
        out[t] = -np.inf if nb == -np.inf else nb - _logsumexp(z[t])
    return out


def blank_weights(logits) -> np.ndarray:
    """w_t = 1 - p_blank(t) of each frame ([T] float64)."""
    return np.exp(log_weights(logits))


def pooled_rows(cu, pool_frames: int) -> np.ndarray:
    """First pooled row of each utterance and the total ([n_seq + 1]):
    utterance i owns ceil(T_i / pool_frames) rows."""
    cu = np.asarray(cu, np.int64)
    out = np.zeros(len(cu), np.int64)
    for i in range(len(cu) - 1):
        t = int(cu[i + 1] - cu[i])
        out[i + 1] = out[i] + (t + pool_frames - 1) // pool_frames
    return out


def posterior_pool(hidden, logits, cu, pool_frames: int = 2):
    """(pooled [G, D] float64, w [T] float64) for hidden [T, D] and the
    mid-layer head's logits [T, C]."""
    h = _as_f64(hidden)
    lw = log_weights(logits)
    cu = np.asarray(cu, np.int64)
    rows = pooled_rows(cu, pool_frames)
    out = np.zeros((int(rows[-1]), h.shape[1]))
    for i in range(len(cu) - 1):
        s, e = int(cu[i]), int(cu[i + 1])
        for g, a in enumerate(range(s, e, pool_frames)):
            b = min(a + pool_frames, e)
            m = np.max(lw[a:b])
            if m == -np.inf:
                continue   # all weights 0: a zero row
            r = np.exp(lw[a:b] - m)
            out[rows[i] + g] = (r[:, None] * h[a:b]).sum(axis=0) / r.sum()
    return out, np.exp(lw)
