"""fp64 CPU oracle for block self-attention and windowed cross-attention.

TEST INFRASTRUCTURE ONLY.  The product path (``chunked_block_self_b200``)
never imports this package; only ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py``'s CPU-baseline leg do.  The arithmetic lives in ``oracle.c``
(plain C, double precision, POSIX threads over (block, head) pairs); this
module only compiles it with gcc and marshals numpy arrays.

What it computes, and the readings taken where the pages are silent, is
stated in the header of ``oracle.c`` (granite-speech-4.1-2b-nar model card,
"Model Architecture" (1) CTC Speech Encoder and (2) Q-Former Projector).

Every public function takes bf16 tensors as their raw 16-bit patterns
(``uint16`` numpy arrays, or torch bf16 CPU tensors which are viewed as such)
and returns float64 numpy arrays.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

_i32p = ctypes.POINTER(ctypes.c_int32)
_i64p = ctypes.POINTER(ctypes.c_int64)
_u16p = ctypes.POINTER(ctypes.c_uint16)
_f64p = ctypes.POINTER(ctypes.c_double)


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so next to it (gcc, -O2, no fast-math)."""
    stale = (not os.path.exists(_LIB_PATH)
             or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC))
    if force or stale:
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-D_POSIX_C_SOURCE=200809L", "-fPIC",
             "-shared", "-o", tmp, _SRC, "-lm", "-lpthread"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            lib.orc_block_table.argtypes = [_i32p, ctypes.c_int, ctypes.c_int,
                                            _i32p, _i32p, _i32p, _i32p, ctypes.c_int]
            lib.orc_window_table.argtypes = [_i32p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                             _i32p, _i32p, _i32p, _i32p, _i32p, ctypes.c_int]
            lib.orc_block_attn.argtypes = [_u16p, _u16p, _u16p, _i32p, ctypes.c_int,
                                           ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                           ctypes.c_double, _f64p, ctypes.c_int]
            lib.orc_block_attn_rows.argtypes = [_u16p, _u16p, _u16p, _i32p, ctypes.c_int,
                                                ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                                ctypes.c_double, _i64p, _i32p, ctypes.c_int,
                                                _f64p]
            lib.orc_block_attn_probs.argtypes = [_u16p, _u16p, _u16p, _i32p, ctypes.c_int,
                                                 ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                                 ctypes.c_double, ctypes.c_int64, ctypes.c_int,
                                                 _f64p, ctypes.POINTER(ctypes.c_int), _i64p,
                                                 _f64p]
            lib.orc_window_xattn.argtypes = [_u16p, _u16p, _u16p, _i32p, ctypes.c_int,
                                             ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                             ctypes.c_int, ctypes.c_double, _f64p, ctypes.c_int]
            lib.orc_window_xattn_rows.argtypes = [_u16p, _u16p, _u16p, _i32p, ctypes.c_int,
                                                  ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                                  ctypes.c_int, ctypes.c_double, _i64p, _i32p,
                                                  ctypes.c_int, _f64p]
            for name in ("orc_block_table", "orc_window_table", "orc_block_attn",
                         "orc_block_attn_rows", "orc_block_attn_probs",
                         "orc_window_xattn", "orc_window_xattn_rows"):
                getattr(lib, name).restype = ctypes.c_int
            _lib = lib
    return _lib


def _bits(x) -> np.ndarray:
    """bf16 tensor / uint16 array -> contiguous uint16 numpy array."""
    if hasattr(x, "view") and hasattr(x, "dtype") and str(x.dtype) == "torch.bfloat16":
        import torch
        x = x.detach().cpu().contiguous().view(torch.int16).numpy()
    a = np.ascontiguousarray(np.asarray(x))
    if a.dtype == np.int16:
        a = a.view(np.uint16)
    if a.dtype != np.uint16:
        raise TypeError("oracle inputs are bf16 bit patterns (uint16)")
    return a


def _cu(cu) -> np.ndarray:
    if hasattr(cu, "detach"):
        cu = cu.detach().cpu().numpy()
    return np.ascontiguousarray(np.asarray(cu, dtype=np.int32))


def _p(a, t):
    return a.ctypes.data_as(t)


def block_table(cu, block_frames: int):
    """Blocks of the packed batch: (seq, j, start, len) int32 arrays."""
    lib = _load()
    cu = _cu(cu)
    n_seq = len(cu) - 1
    n = lib.orc_block_table(_p(cu, _i32p), n_seq, block_frames, None, None, None, None, 0)
    if n < 0:
        raise ValueError("invalid cu_seqlens")
    out = [np.zeros(max(n, 1), np.int32) for _ in range(4)]
    lib.orc_block_table(_p(cu, _i32p), n_seq, block_frames, *[_p(o, _i32p) for o in out], n)
    return tuple(o[:n] for o in out)


def window_table(cu, window_frames: int, queries_per_window: int):
    """Windows of the packed batch: (seq, w, start, len, q_row) int32 arrays."""
    lib = _load()
    cu = _cu(cu)
    n_seq = len(cu) - 1
    n = lib.orc_window_table(_p(cu, _i32p), n_seq, window_frames, queries_per_window,
                             None, None, None, None, None, 0)
    if n < 0:
        raise ValueError("invalid cu_seqlens")
    out = [np.zeros(max(n, 1), np.int32) for _ in range(5)]
    lib.orc_window_table(_p(cu, _i32p), n_seq, window_frames, queries_per_window,
                         *[_p(o, _i32p) for o in out], n)
    return tuple(o[:n] for o in out)


def _check_shapes(q, k, v):
    if q.ndim != 3 or k.shape != v.shape or q.shape[1:] != k.shape[1:]:
        raise ValueError("expected [rows, heads, d] tensors with matching heads and d")


def block_attn(q, k, v, cu, block_frames: int = 200, scale: float | None = None,
               n_threads: int = 0) -> np.ndarray:
    """All outputs of block self-attention, float64 [total_frames, heads, d]."""
    lib = _load()
    q, k, v, cu = _bits(q), _bits(k), _bits(v), _cu(cu)
    _check_shapes(q, k, v)
    heads, d = q.shape[1], q.shape[2]
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    out = np.zeros(q.shape, np.float64)
    rc = lib.orc_block_attn(_p(q, _u16p), _p(k, _u16p), _p(v, _u16p), _p(cu, _i32p),
                            len(cu) - 1, heads, d, block_frames, float(scale),
                            _p(out, _f64p), n_threads)
    if rc < 0:
        raise ValueError("oracle block_attn failed (invalid cu_seqlens?)")
    return out


def block_attn_rows(q, k, v, cu, rows, heads_sel, block_frames: int = 200,
                    scale: float | None = None) -> np.ndarray:
    """Outputs at selected (frame, head) pairs, float64 [n, d]."""
    lib = _load()
    q, k, v, cu = _bits(q), _bits(k), _bits(v), _cu(cu)
    _check_shapes(q, k, v)
    heads, d = q.shape[1], q.shape[2]
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    rows = np.ascontiguousarray(np.asarray(rows, np.int64))
    hs = np.ascontiguousarray(np.asarray(heads_sel, np.int32))
    out = np.zeros((len(rows), d), np.float64)
    rc = lib.orc_block_attn_rows(_p(q, _u16p), _p(k, _u16p), _p(v, _u16p), _p(cu, _i32p),
                                 len(cu) - 1, heads, d, block_frames, float(scale),
                                 _p(rows, _i64p), _p(hs, _i32p), len(rows), _p(out, _f64p))
    if rc < 0:
        raise ValueError("oracle block_attn_rows failed")
    return out


def block_attn_probs(q, k, v, cu, row: int, head: int, block_frames: int = 200,
                     scale: float | None = None):
    """(key_start, probabilities, output) of one (frame, head)."""
    lib = _load()
    q, k, v, cu = _bits(q), _bits(k), _bits(v), _cu(cu)
    heads, d = q.shape[1], q.shape[2]
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    probs = np.zeros(block_frames, np.float64)
    out = np.zeros(d, np.float64)
    nk = ctypes.c_int(0)
    ks = ctypes.c_int64(0)
    rc = lib.orc_block_attn_probs(_p(q, _u16p), _p(k, _u16p), _p(v, _u16p), _p(cu, _i32p),
                                  len(cu) - 1, heads, d, block_frames, float(scale),
                                  int(row), int(head), _p(probs, _f64p), ctypes.byref(nk),
                                  ctypes.byref(ks), _p(out, _f64p))
    if rc < 0:
        raise ValueError("oracle block_attn_probs failed")
    return ks.value, probs[:nk.value].copy(), out


def window_xattn(q, k, v, cu, window_frames: int = 15, queries_per_window: int = 3,
                 scale: float | None = None, n_threads: int = 0) -> np.ndarray:
    """All outputs of the windowed cross-attention, float64 shaped like q."""
    lib = _load()
    q, k, v, cu = _bits(q), _bits(k), _bits(v), _cu(cu)
    _check_shapes(q, k, v)
    heads, d = q.shape[1], q.shape[2]
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    n_win = len(window_table(cu, window_frames, queries_per_window)[0])
    if q.shape[0] != queries_per_window * n_win:
        raise ValueError("q must hold queries_per_window rows per window")
    out = np.zeros(q.shape, np.float64)
    rc = lib.orc_window_xattn(_p(q, _u16p), _p(k, _u16p), _p(v, _u16p), _p(cu, _i32p),
                              len(cu) - 1, heads, d, window_frames, queries_per_window,
                              float(scale), _p(out, _f64p), n_threads)
    if rc < 0:
        raise ValueError("oracle window_xattn failed")
    return out


def window_xattn_rows(q, k, v, cu, qrows, heads_sel, window_frames: int = 15,
                      queries_per_window: int = 3, scale: float | None = None) -> np.ndarray:
    """Windowed cross-attention outputs at selected (query row, head) pairs."""
    lib = _load()
    q, k, v, cu = _bits(q), _bits(k), _bits(v), _cu(cu)
    heads, d = q.shape[1], q.shape[2]
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    qrows = np.ascontiguousarray(np.asarray(qrows, np.int64))
    hs = np.ascontiguousarray(np.asarray(heads_sel, np.int32))
    out = np.zeros((len(qrows), d), np.float64)
    rc = lib.orc_window_xattn_rows(_p(q, _u16p), _p(k, _u16p), _p(v, _u16p), _p(cu, _i32p),
                                   len(cu) - 1, heads, d, window_frames, queries_per_window,
                                   float(scale), _p(qrows, _i64p), _p(hs, _i32p), len(qrows),
                                   _p(out, _f64p))
    if rc < 0:
        raise ValueError("oracle window_xattn_rows failed")
    return out


def _one_block(cu) -> int:
    """A block length that holds every utterance of cu whole."""
    cu = np.asarray(cu, np.int64)
    return max(1, int(np.max(np.diff(cu)))) if len(cu) > 1 else 1


def varlen_attn(q, k, v, cu, scale: float | None = None, n_threads: int = 0) -> np.ndarray:
    """Full bidirectional attention inside each packed utterance (no blocks;
    the editor's attention with the causal mask removed, granite-speech-
    4.1-2b-nar model card, "Model Architecture" (3)): the block definition
    with one block per utterance, float64 [total_frames, heads, d]."""
    return block_attn(q, k, v, cu, block_frames=_one_block(cu), scale=scale, n_threads=n_threads)


def varlen_attn_rows(q, k, v, cu, rows, heads_sel, scale: float | None = None) -> np.ndarray:
    """Full-utterance attention outputs at selected (frame, head) pairs."""
    return block_attn_rows(q, k, v, cu, rows, heads_sel, block_frames=_one_block(cu), scale=scale)


def threads_used(n_threads: int = 0) -> int:
    """How many threads a call with ``n_threads`` uses (0 = all online cores)."""
    return n_threads if n_threads > 0 else (os.cpu_count() or 1)


from .ctc import collapse as ctc_collapse, ctc_greedy, frame_classes as ctc_frame_classes  # noqa: E402,F401
from .pool import (blank_weights, log_weights as pool_log_weights,  # noqa: E402,F401
                   pooled_rows, posterior_pool)
from .qkv import block_attn_f64, block_attn_qkv, qkv_project  # noqa: E402,F401
