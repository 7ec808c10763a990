"""CTC greedy decoding of the encoder's CTC head -- TEST INFRASTRUCTURE ONLY.

Written from the q4-RTN ONNX page ("Inference note (NAR decode)"): the head
emits vocab + 1 = 100353 classes per frame with the blank at class 0, and a
non-blank class c is LLM token c - 1.  Decoding takes, per frame, the class
of the largest logit, collapses runs of equal consecutive classes into one,
drops the blank, and subtracts 1.  Readings taken where the page is silent:
- the logits are bf16 (the model card's inference is bf16) and are compared
  exactly; among equal largest logits the lowest class wins;
- a NaN logit is no candidate (it carries no ordering); a frame whose logits
  are all NaN takes the blank;
- runs are collapsed within one utterance of the packed batch only;
- a blank frame between two equal classes separates them (both are kept).

Only the test suite, the smoke check and the bench's CPU-baseline leg use
this module; it shares no code with the CUDA library.
"""
from __future__ import annotations

import numpy as np


def _as_f64(logits) -> np.ndarray:
    """bf16 bit patterns (uint16) or a torch bf16 tensor -> exact float64."""
    try:
        import torch
        if isinstance(logits, torch.Tensor):
            logits = logits.contiguous().view(torch.int16).numpy().view(np.uint16)
    except ImportError:
        pass
    a = np.asarray(logits)
    if a.dtype == np.uint16:
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


def frame_classes(logits, rows_per_pass: int = 256) -> np.ndarray:
    """Class of the largest logit of each frame ([T, C] -> [T] int64): the
    first (lowest) class among equal maxima, NaN logits skipped, the blank
    when a frame has no other candidate.

    Written with whole-array operations over ``rows_per_pass`` frames at a
    time (the definition is per frame; passes only bound the memory)."""
    try:
        import torch
        if isinstance(logits, torch.Tensor):
            logits = logits.contiguous().view(torch.int16).numpy().view(np.uint16)
    except ImportError:
        pass
    src = np.asarray(logits)
    out = np.zeros(src.shape[0], np.int64)
    for a in range(0, src.shape[0], rows_per_pass):
        x = _as_f64(src[a:a + rows_per_pass])
        cand = ~np.isnan(x)                                   # the candidate classes
        best = np.where(cand, x, -np.inf).max(axis=1, initial=-np.inf)
        hit = cand & (x == best[:, None])                     # candidates holding the maximum
        any_hit = hit.any(axis=1)
        out[a:a + x.shape[0]] = np.where(any_hit, hit.argmax(axis=1), 0)   # lowest such class
    return out


def collapse(classes, cu, blank: int = 0) -> list[list[int]]:
    """Token ids of each utterance: runs of equal consecutive classes of the
    utterance become one, blanks are dropped, and class c becomes c - 1."""
    cu = np.asarray(cu, np.int64)
    out = []
    for u in range(len(cu) - 1):
        toks, prev = [], None
        for i in range(int(cu[u]), int(cu[u + 1])):
            c = int(classes[i])
            if c != prev and c != blank:
                toks.append(c - 1)
            prev = c
        out.append(toks)
    return out


def ctc_greedy(logits, cu, blank: int = 0):
    """(per-frame classes, token ids per utterance)."""
    cls = frame_classes(logits)
    return cls, collapse(cls, cu, blank)
