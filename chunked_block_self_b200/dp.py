"""Data-parallel replicas by utterance (no collective on the data path).

Blocks and windows never cross an utterance, so a packed batch splits into
per-rank sub-batches of whole utterances with no exchange step.  The split
itself (``nle_shard_plan_host``, balancing sum over blocks of len^2) is in
libnle; this module only re-bases the offsets of one rank's range.
"""
from __future__ import annotations

import numpy as np


def local_shard(cu_host, bounds, rank: int):
    """Frame range and re-based offsets of rank ``rank``'s utterances.

    Returns ``(first_frame, end_frame, local_cu)`` where ``local_cu`` is the
    int32 cu_seqlens of utterances ``bounds[rank] .. bounds[rank+1]`` starting
    at 0; the rank's q/k/v rows are ``[first_frame, end_frame)``.
    """
    cu = np.asarray(cu_host, np.int64)
    a, b = int(bounds[rank]), int(bounds[rank + 1])
    first, end = int(cu[a]), int(cu[b])
    local = (cu[a:b + 1] - first).astype(np.int32)
    return first, end, local
