"""Seeded synthetic inputs shaped like the pages' workloads.

This module is shared by the tests, the bench and the smoke check; it feeds
both the CUDA path and the CPU oracle.  It holds no attention arithmetic:
only utterance lengths, packed offsets (``cu_seqlens``) and bf16 tensors
drawn from a seeded ``numpy.random.default_rng``.

Recipe (all inputs synthetic; no audio, no trained weights):

* lengths are drawn first from the config's length rule, then Q, K, V as
  float32 N(0, 1) times the config's factor, rounded to bf16
  round-to-nearest-even (torch's float32 -> bf16 conversion).
* default seed = 1000 + config number.

The five workloads stand in for the pages' ones by shape only:

1. one utterance of 400 frames (8 s at 50 Hz), 8 heads x 64;
2. the fixed 800-frame encoder bucket of the portable ONNX README, 16 x 64,
   values N(0,1) * 0.5;
3. 16 utterances of 39-94 s (1950-4700 frames, never a multiple of the
   200-frame block, so each ends in a partial block), 16 x 64;
4. 128 utterances of 2-16 s (100-800 frames), 16 x 64 -- the batch-128
   throughput setting of the model card;
5. the projector: 64 utterances of 4700 frames; K/V 16 x 64, three query
   rows per 15-frame window.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch


@dataclass(frozen=True)
class Workload:
    name: str
    n_seq: int
    t_min: int
    t_max: int
    heads: int
    d_head: int
    factor: float
    block_frames: int = 200
    avoid_multiple_of: int = 0      # redraw lengths divisible by this (0: never)
    window_frames: int = 0          # > 0 for the windowed cross-attention
    queries_per_window: int = 0


CONFIGS = {
    1: Workload("single utterance T=400, 8x64", 1, 400, 400, 8, 64, 1.0),
    2: Workload("800-frame bucket, 16x64, x0.5", 1, 800, 800, 16, 64, 0.5),
    3: Workload("16 utts 1950-4700 frames, 16x64", 16, 1950, 4700, 16, 64, 1.0,
                avoid_multiple_of=200),
    4: Workload("128 utts 100-800 frames, 16x64", 128, 100, 800, 16, 64, 1.0),
    5: Workload("projector 64 x 4700 frames, 15-frame windows x 3 queries, 16x64",
                64, 4700, 4700, 16, 64, 1.0, window_frames=15, queries_per_window=3),
}


def default_seed(cfg: int) -> int:
    return 1000 + int(cfg)


def draw_lengths(cfg: int, seed: int | None = None) -> np.ndarray:
    """Utterance lengths in frames for config ``cfg`` (int64 numpy)."""
    w = CONFIGS[cfg]
    rng = np.random.default_rng(default_seed(cfg) if seed is None else seed)
    out = np.empty(w.n_seq, np.int64)
    for i in range(w.n_seq):
        while True:
            t = int(rng.integers(w.t_min, w.t_max + 1))
            if not w.avoid_multiple_of or t % w.avoid_multiple_of:
                break
        out[i] = t
    return out


def cu_seqlens(lengths) -> np.ndarray:
    """Packed offsets: int32 [n_seq + 1], cu[0] = 0, cu[i+1] = cu[i] + T_i."""
    lengths = np.asarray(lengths, np.int64)
    cu = np.zeros(len(lengths) + 1, np.int64)
    np.cumsum(lengths, out=cu[1:])
    if cu[-1] >= 2**31:
        raise ValueError("total frames exceed int32")
    return cu.astype(np.int32)


def bf16_normal(rng: np.random.Generator, shape, factor: float = 1.0) -> torch.Tensor:
    """float32 N(0,1) * factor from ``rng``, rounded to bf16 (CPU tensor)."""
    x = rng.standard_normal(size=shape, dtype=np.float32)
    if factor != 1.0:
        x *= np.float32(factor)
    return torch.from_numpy(x).to(torch.bfloat16)


def block_inputs(cfg: int | None = None, seed: int | None = None, *, lengths=None,
                 heads: int | None = None, d_head: int = 64, factor: float | None = None,
                 block_frames: int | None = None, device=None) -> dict:
    """Q, K, V (bf16 CPU, [total_frames, heads, d_head]) plus offsets.

    Either a config number, or explicit ``lengths``/``heads`` for custom cases.
    With ``device``, Q, K and V are drawn there instead (see device_normal).
    """
    if cfg is not None:
        w = CONFIGS[cfg]
        seed = default_seed(cfg) if seed is None else seed
        if lengths is None:
            lengths = draw_lengths(cfg, seed)
        heads = w.heads if heads is None else heads
        d_head = w.d_head
        factor = w.factor if factor is None else factor
        block_frames = w.block_frames if block_frames is None else block_frames
    lengths = np.asarray(lengths, np.int64)
    heads = 1 if heads is None else heads
    factor = 1.0 if factor is None else factor
    block_frames = 200 if block_frames is None else block_frames
    cu = cu_seqlens(lengths)
    total = int(cu[-1])
    if device is not None:
        s0 = 12345 if seed is None else seed + 7
        q, k, v = (device_normal((total, heads, d_head), factor, s0 + i, device) for i in range(3))
        return dict(q=q, k=k, v=v, cu=cu, lengths=lengths, heads=heads, d_head=d_head,
                    block_frames=block_frames, total=total)
    rng = np.random.default_rng(12345 if seed is None else seed + 7)
    q = bf16_normal(rng, (total, heads, d_head), factor)
    k = bf16_normal(rng, (total, heads, d_head), factor)
    v = bf16_normal(rng, (total, heads, d_head), factor)
    return dict(q=q, k=k, v=v, cu=cu, lengths=lengths, heads=heads, d_head=d_head,
                block_frames=block_frames, total=total)


def device_normal(shape, factor: float, seed: int, device) -> torch.Tensor:
    """bf16 N(0,1) * factor drawn on ``device`` from a torch generator seeded
    with ``seed`` (other values than the host generator, same distribution):
    for benchmark inputs too large to draw on the host quickly."""
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    x = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    if factor != 1.0:
        x *= factor
    return x.to(torch.bfloat16)


def window_inputs(n_query_rows: int, cfg: int | None = 5, seed: int | None = None, *,
                  lengths=None, heads: int | None = None, d_head: int = 64,
                  factor: float | None = None, device=None) -> dict:
    """Inputs of the windowed cross-attention.

    ``n_query_rows`` is the number of query rows the caller's window plan asks
    for (this module does not cut windows).  K and V are [total_frames, heads,
    d_head]; Q is [n_query_rows, heads, d_head]; bf16 CPU tensors, or tensors
    drawn on ``device`` (see device_normal) when one is given.
    """
    w = CONFIGS[cfg] if cfg is not None else None
    if w is not None:
        seed = default_seed(cfg) if seed is None else seed
        if lengths is None:
            lengths = draw_lengths(cfg, seed)
        heads = w.heads if heads is None else heads
        factor = w.factor if factor is None else factor
    lengths = np.asarray(lengths, np.int64)
    heads = 1 if heads is None else heads
    factor = 1.0 if factor is None else factor
    cu = cu_seqlens(lengths)
    total = int(cu[-1])
    if device is not None:
        s0 = 54321 if seed is None else seed + 11
        k = device_normal((total, heads, d_head), factor, s0, device)
        v = device_normal((total, heads, d_head), factor, s0 + 1, device)
        q = device_normal((int(n_query_rows), heads, d_head), factor, s0 + 2, device)
        return dict(q=q, k=k, v=v, cu=cu, lengths=lengths, heads=heads, d_head=d_head, total=total)
    rng = np.random.default_rng(54321 if seed is None else seed + 11)
    k = bf16_normal(rng, (total, heads, d_head), factor)
    v = bf16_normal(rng, (total, heads, d_head), factor)
    q = bf16_normal(rng, (int(n_query_rows), heads, d_head), factor)
    return dict(q=q, k=k, v=v, cu=cu, lengths=lengths, heads=heads, d_head=d_head,
                total=total)


# ------------------------------------------------------------------ CTC head logits
CTC_CLASSES = 100353   # vocab + 1, blank at class 0 (q4-RTN ONNX page, decode note)


def ctc_logits(lengths, n_classes: int = CTC_CLASSES, seed: int = 2000, row_stride: int | None = None,
               device=None) -> torch.Tensor:
    """bf16 [frames, row_stride] logits shaped like a CTC head's output (only
    the first n_classes of a row are meaningful; padding is random too):
    N(0, 1) everywhere, then frames are drawn in runs of 1-4 -- about 60 %
    of the runs boost the blank (class 0) by 6, the rest boost one random
    class by 6 -- so that blanks, repeated classes and separated repeats all
    occur.  A few frames get an exact tie between two boosted classes.
    With device=None the values come from numpy's default_rng(seed) on the
    host; with a CUDA device, from a seeded torch generator on the device
    (other values, same structure)."""
    frames = int(np.sum(lengths))
    stride = n_classes if row_stride is None else row_stride
    if device is None:
        rng = np.random.default_rng(seed)
        x = torch.from_numpy(rng.standard_normal((frames, stride), dtype=np.float32))
        # runs of boosted classes
        cls = np.empty(frames, np.int64)
        i = 0
        while i < frames:
            run = int(rng.integers(1, 5))
            c = 0 if rng.random() < 0.6 else int(rng.integers(1, n_classes))
            cls[i:i + run] = c
            i += run
        ties = rng.random(frames) < 0.02
        tie_cls = rng.integers(0, n_classes, frames)
        x[np.arange(frames), cls] = 6.0
        x[np.nonzero(ties)[0], tie_cls[ties]] = 6.0
        return x.to(torch.bfloat16)
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    x = torch.randn((frames, stride), generator=g, device=device, dtype=torch.float32).to(torch.bfloat16)
    runs = torch.randint(1, 5, (frames,), generator=g, device=device)
    starts = torch.cumsum(runs, 0) - runs
    starts = starts[starts < frames]
    run_id = torch.zeros(frames, dtype=torch.int64, device=device)
    run_id[starts[1:]] = 1
    run_id = torch.cumsum(run_id, 0)
    n_runs = int(starts.numel())
    blank = torch.rand((n_runs,), generator=g, device=device) < 0.6
    rcls = torch.where(blank, torch.zeros((), dtype=torch.int64, device=device),
                       torch.randint(1, n_classes, (n_runs,), generator=g, device=device))
    x[torch.arange(frames, device=device), rcls[run_id]] = 6.0
    return x


# ------------------------------------------------------------------ posterior-weighted pooling
POOL_FRAMES = 2       # a window of 4 10-ms input frames = 2 encoder frames at 50 Hz
HIDDEN_DIM = 1024     # encoder width: 16 heads x 64
CHAR_CLASSES = 256    # mid-layer (character) head classes: not on the pages; a stand-in


def pool_inputs(lengths, dim: int = HIDDEN_DIM, n_classes: int = CHAR_CLASSES, seed: int = 3000,
                hidden_stride: int | None = None, logits_stride: int | None = None, device=None) -> dict:
    """Inputs of the posterior-weighted pooling: hidden bf16 [frames,
    hidden_stride] (N(0, 1); the first dim columns used) and the mid-layer
    head's logits bf16 [frames, logits_stride] (N(0, 2^2); the first
    n_classes used).  Frames come in runs of 1-6: about half of the runs
    boost the blank (class 0) by 2-10, so blank probabilities range from
    near 0 to near 1; 2 % of frames get every non-blank logit -inf (weight
    exactly 0) and 1 % get a -inf blank (weight exactly 1).  With
    device=None the values come from numpy's default_rng(seed) on the host,
    else from a seeded torch generator on that device (same structure)."""
    frames = int(np.sum(lengths))
    hs = dim if hidden_stride is None else hidden_stride
    zs = n_classes if logits_stride is None else logits_stride
    if device is None:
        rng = np.random.default_rng(seed)
        h = torch.from_numpy(rng.standard_normal((frames, hs), dtype=np.float32))
        z = rng.standard_normal((frames, zs), dtype=np.float32) * 2.0
        i = 0
        while i < frames:
            run = int(rng.integers(1, 7))
            if rng.random() < 0.5:
                z[i:i + run, 0] += np.float32(rng.uniform(2.0, 10.0))
            i += run
        if n_classes > 1:
            dead = rng.random(frames) < 0.02
            z[np.ix_(np.nonzero(dead)[0], np.arange(1, n_classes))] = -np.inf
        z[rng.random(frames) < 0.01, 0] = -np.inf
        return dict(hidden=h.to(torch.bfloat16), logits=torch.from_numpy(z).to(torch.bfloat16))
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    h = torch.randn((frames, hs), generator=g, device=device, dtype=torch.float32).to(torch.bfloat16)
    z = torch.randn((frames, zs), generator=g, device=device, dtype=torch.float32) * 2.0
    runs = torch.randint(1, 7, (frames,), generator=g, device=device)
    starts = torch.cumsum(runs, 0) - runs
    starts = starts[starts < frames]
    run_id = torch.zeros(frames, dtype=torch.int64, device=device)
    run_id[starts[1:]] = 1
    run_id = torch.cumsum(run_id, 0)
    n_runs = int(starts.numel())
    boost = torch.where(torch.rand((n_runs,), generator=g, device=device) < 0.5,
                        2.0 + 8.0 * torch.rand((n_runs,), generator=g, device=device),
                        torch.zeros((), device=device))
    z[:, 0] += boost[run_id]
    if n_classes > 1:
        dead = torch.rand((frames,), generator=g, device=device) < 0.02
        z[dead, 1:n_classes] = -float("inf")
    z[torch.rand((frames,), generator=g, device=device) < 0.01, 0] = -float("inf")
    return dict(hidden=h, logits=z.to(torch.bfloat16))
