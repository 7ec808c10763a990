"""Thin ctypes binding of libnle.so (declared in include/nle.h).

Argument marshalling only: every step of the computation runs in the CUDA
kernels of libnle.so.  Importing this module loads the library and raises
ImportError if it is missing -- there is no fallback path.  Build it with
``python -m chunked_block_self_b200.build`` (``__graft_entry__.build()``).

Functions named ``nle_*`` mirror the C entry points one to one; they take
torch CUDA tensors (or, for the host table functions, numpy arrays) and the
stream defaults to torch's current stream.  A non-zero status raises
:class:`NLEError`.  The few helpers without the prefix (``block_attn``,
``window_xattn``, ``window_query_rows``) only allocate outputs with torch
and call the entry points.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libnle.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"libnle.so not found at {LIB_PATH}: run `python -m chunked_block_self_b200.build` "
                      "(the CUDA library is required; there is no CPU fallback)")
_lib = ctypes.CDLL(LIB_PATH)

_vp = ctypes.c_void_p
_i32 = ctypes.c_int32
_int = ctypes.c_int
_i64 = ctypes.c_int64
_f32 = ctypes.c_float
_i32p = ctypes.POINTER(ctypes.c_int32)

class PathBuffers(ctypes.Structure):
    """nle_path_buffers: host tensors, then their device copies."""
    _fields_ = [(n, _vp) for n in ("q", "k", "v", "out", "qw", "kw", "vw", "out_w", "cu",
                                    "d_q", "d_k", "d_v", "d_out", "d_qw", "d_kw", "d_vw", "d_out_w", "d_cu",
                                    "d_status")]


_SIGS = {
    "nle_version": ([], _int),
    "nle_path_fwd_host": ([ctypes.POINTER(PathBuffers), _int, _i64, _i64, _int, _int, _int, _int, _int, _int,
                           _vp], _int),
    "nle_status_string": ([_int], ctypes.c_char_p),
    "nle_block_attn_fwd": ([_vp, _vp, _vp, _vp, _vp, _int, _i64, _int, _int, _int, _vp], _int),
    "nle_block_attn_fwd_ex": ([_vp, _vp, _vp, _vp, _vp, _int, _i64, _int, _int, _int, _f32, _i64, _vp,
                               _int, _i64, _vp], _int),
    "nle_block_attn_qkv_fwd": ([_vp, _vp, _vp, _vp, _vp, _int, _i64, _int, _int, _int, _int, _vp], _int),
    "nle_block_attn_qkv_fwd_ex": ([_vp, _vp, _vp, _vp, _vp, _int, _i64, _int, _int, _int, _int, _f32, _vp, _int,
                                   _i64, _vp], _int),
    "nle_window_xattn_fwd": ([_vp, _vp, _vp, _vp, _vp, _int, _i64, _i64, _int, _int, _int, _int, _vp], _int),
    "nle_window_xattn_fwd_ex": ([_vp, _vp, _vp, _vp, _vp, _int, _i64, _i64, _int, _int, _int, _int, _f32,
                                 _vp, _int, _i64, _vp], _int),
    "nle_block_plan_host": ([_vp, _int, _int, _vp, _vp, _vp, _vp, _int, ctypes.POINTER(_int)], _int),
    "nle_block_plan_dev": ([_vp, _int, _i64, _int, _vp, _vp, _vp, _vp, _int, _vp, _vp], _int),
    "nle_window_plan_host": ([_vp, _int, _int, _int, _vp, _vp, _vp, _vp, _vp, _int, ctypes.POINTER(_int)],
                             _int),
    "nle_shard_plan_host": ([_vp, _int, _int, _int, _vp], _int),
    "nle_varlen_attn_fwd": ([_vp, _vp, _vp, _vp, _vp, _int, _i64, _int, _int, _vp], _int),
    "nle_varlen_attn_fwd_ex": ([_vp, _vp, _vp, _vp, _vp, _int, _i64, _int, _int, _f32, _i64, _vp, _int, _i64,
                                _vp], _int),
    "nle_ctc_greedy_fwd": ([_vp, _i64, _int, _vp, _int, _i64, _vp, _vp, _vp, _vp], _int),
    "nle_posterior_pool_fwd": ([_vp, _i64, _int, _vp, _i64, _int, _vp, _int, _i64, _int, _i64, _vp, _vp, _vp,
                                _vp], _int),
}
for _name, (_args, _res) in _SIGS.items():
    _fn = getattr(_lib, _name)
    _fn.argtypes = _args
    _fn.restype = _res

EXPORTS = tuple(_SIGS)

NLE_OK = 0
NLE_ERR_INVALID_ARG = -1
NLE_ERR_UNSUPPORTED = -2
NLE_ERR_MISALIGNED = -3
NLE_ERR_CUDA = -4
NLE_ERR_TIMEOUT = -5
NLE_FLAG_TEST_SKIP_FIRST_LOAD = 1
NLE_FLAG_WHOLE_ITEMS = 2    # block attention: never run row tiles as separate items
NLE_FLAG_SPLIT_ITEMS = 4    # block attention: always run row tiles as separate items


class NLEError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {nle_status_string(status)} ({status})")
        self.status = status


def _check(rc: int, where: str) -> None:
    if rc != NLE_OK:
        raise NLEError(rc, where)


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, torch.Tensor):
        return t.data_ptr()
    if isinstance(t, np.ndarray):
        return t.ctypes.data
    return int(t)


def _stream(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _dev_tensor(t, name, dtype):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}")


def nle_version() -> int:
    return _lib.nle_version()


def nle_status_string(status: int) -> str:
    return _lib.nle_status_string(int(status)).decode()


# ------------------------------------------------------------------ block attention
def nle_block_attn_fwd(q, k, v, out, cu_seqlens, n_seq: int | None = None, total_frames: int | None = None,
                       heads: int | None = None, d_head: int | None = None, block_frames: int = 200,
                       stream=None) -> None:
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (out, "out")):
        _dev_tensor(t, n, torch.bfloat16)
    _dev_tensor(cu_seqlens, "cu_seqlens", torch.int32)
    n_seq = cu_seqlens.numel() - 1 if n_seq is None else n_seq
    total_frames = q.shape[0] if total_frames is None else total_frames
    heads = q.shape[1] if heads is None else heads
    d_head = q.shape[2] if d_head is None else d_head
    _check(_lib.nle_block_attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(cu_seqlens), n_seq,
                                   total_frames, heads, d_head, block_frames, _stream(stream)),
           "nle_block_attn_fwd")


def nle_block_attn_fwd_ex(q, k, v, out, cu_seqlens, n_seq: int | None = None, total_frames: int | None = None,
                          heads: int | None = None, d_head: int = 64, block_frames: int = 200,
                          softmax_scale: float = 0.0, row_stride_qkv: int = 0, dev_status=None, flags: int = 0,
                          wait_limit_ns: int = 0, stream=None) -> None:
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (out, "out")):
        _dev_tensor(t, n, torch.bfloat16)
    _dev_tensor(cu_seqlens, "cu_seqlens", torch.int32)
    if dev_status is not None:
        _dev_tensor(dev_status, "dev_status", torch.int32)
    n_seq = cu_seqlens.numel() - 1 if n_seq is None else n_seq
    total_frames = out.shape[0] if total_frames is None else total_frames
    heads = out.shape[1] if heads is None else heads
    _check(_lib.nle_block_attn_fwd_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(cu_seqlens), n_seq,
                                      total_frames, heads, d_head, block_frames, float(softmax_scale),
                                      row_stride_qkv, _ptr(dev_status), flags, wait_limit_ns, _stream(stream)),
           "nle_block_attn_fwd_ex")


def block_attn(q, k, v, cu_seqlens, block_frames: int = 200, out=None, stream=None) -> torch.Tensor:
    """O = block attention of packed q/k/v ([frames, heads, 64] bf16 CUDA)."""
    if out is None:
        out = torch.empty_like(q)
    nle_block_attn_fwd(q, k, v, out, cu_seqlens, block_frames=block_frames, stream=stream)
    return out


# ------------------------------------------------------------------ QKV projection + block attention
def nle_block_attn_qkv_fwd_ex(x, w_qkv, bias, out, cu_seqlens, n_seq: int | None = None,
                              total_frames: int | None = None, heads: int | None = None, d_head: int = 64,
                              block_frames: int = 200, softmax_scale: float = 0.0, dev_status=None, flags: int = 0,
                              wait_limit_ns: int = 0, stream=None) -> None:
    """x: CUDA bf16 [frames, d_model]; w_qkv: bf16 [3 * heads * 64, d_model];
    bias: None or bf16 [3 * heads * 64]; out: bf16 [frames, heads, 64]."""
    _dev_tensor(x, "x", torch.bfloat16)
    _dev_tensor(w_qkv, "w_qkv", torch.bfloat16)
    _dev_tensor(out, "out", torch.bfloat16)
    if bias is not None:
        _dev_tensor(bias, "bias", torch.bfloat16)
    _dev_tensor(cu_seqlens, "cu_seqlens", torch.int32)
    if dev_status is not None:
        _dev_tensor(dev_status, "dev_status", torch.int32)
    if x.dim() != 2 or not x.is_contiguous() or not w_qkv.is_contiguous():
        raise ValueError("x: contiguous [frames, d_model]; w_qkv: contiguous [3 * heads * 64, d_model]")
    n_seq = cu_seqlens.numel() - 1 if n_seq is None else n_seq
    total_frames = x.shape[0] if total_frames is None else total_frames
    heads = out.shape[1] if heads is None else heads
    _check(_lib.nle_block_attn_qkv_fwd_ex(_ptr(x), _ptr(w_qkv), _ptr(bias), _ptr(out), _ptr(cu_seqlens), n_seq,
                                          total_frames, x.shape[1], heads, d_head, block_frames,
                                          float(softmax_scale), _ptr(dev_status), flags, wait_limit_ns,
                                          _stream(stream)),
           "nle_block_attn_qkv_fwd_ex")


def nle_block_attn_qkv_fwd(x, w_qkv, bias, out, cu_seqlens, block_frames: int = 200, stream=None) -> None:
    _dev_tensor(x, "x", torch.bfloat16)
    _dev_tensor(w_qkv, "w_qkv", torch.bfloat16)
    _dev_tensor(out, "out", torch.bfloat16)
    if bias is not None:
        _dev_tensor(bias, "bias", torch.bfloat16)
    _dev_tensor(cu_seqlens, "cu_seqlens", torch.int32)
    if x.dim() != 2 or not x.is_contiguous() or not w_qkv.is_contiguous():
        raise ValueError("x: contiguous [frames, d_model]; w_qkv: contiguous [3 * heads * 64, d_model]")
    _check(_lib.nle_block_attn_qkv_fwd(_ptr(x), _ptr(w_qkv), _ptr(bias), _ptr(out), _ptr(cu_seqlens),
                                       cu_seqlens.numel() - 1, x.shape[0], x.shape[1], out.shape[1], 64,
                                       block_frames, _stream(stream)),
           "nle_block_attn_qkv_fwd")


def block_attn_qkv(x, w_qkv, cu_seqlens, heads: int, bias=None, block_frames: int = 200, out=None,
                   stream=None) -> torch.Tensor:
    """O [frames, heads, 64] of block attention of X's QKV projection."""
    if out is None:
        out = torch.empty((x.shape[0], heads, 64), dtype=torch.bfloat16, device=x.device)
    nle_block_attn_qkv_fwd(x, w_qkv, bias, out, cu_seqlens, block_frames=block_frames, stream=stream)
    return out


# ------------------------------------------------------------------ full-utterance attention
def nle_varlen_attn_fwd(q, k, v, out, cu_seqlens, n_seq: int | None = None, total_frames: int | None = None,
                        heads: int | None = None, d_head: int | None = None, stream=None) -> None:
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (out, "out")):
        _dev_tensor(t, n, torch.bfloat16)
    _dev_tensor(cu_seqlens, "cu_seqlens", torch.int32)
    n_seq = cu_seqlens.numel() - 1 if n_seq is None else n_seq
    total_frames = q.shape[0] if total_frames is None else total_frames
    heads = q.shape[1] if heads is None else heads
    d_head = q.shape[2] if d_head is None else d_head
    _check(_lib.nle_varlen_attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(cu_seqlens), n_seq,
                                    total_frames, heads, d_head, _stream(stream)),
           "nle_varlen_attn_fwd")


def nle_varlen_attn_fwd_ex(q, k, v, out, cu_seqlens, n_seq: int | None = None, total_frames: int | None = None,
                           heads: int | None = None, d_head: int = 64, softmax_scale: float = 0.0,
                           row_stride_qkv: int = 0, dev_status=None, flags: int = 0, wait_limit_ns: int = 0,
                           stream=None) -> None:
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (out, "out")):
        _dev_tensor(t, n, torch.bfloat16)
    _dev_tensor(cu_seqlens, "cu_seqlens", torch.int32)
    if dev_status is not None:
        _dev_tensor(dev_status, "dev_status", torch.int32)
    n_seq = cu_seqlens.numel() - 1 if n_seq is None else n_seq
    total_frames = out.shape[0] if total_frames is None else total_frames
    heads = out.shape[1] if heads is None else heads
    _check(_lib.nle_varlen_attn_fwd_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(cu_seqlens), n_seq,
                                       total_frames, heads, d_head, float(softmax_scale), row_stride_qkv,
                                       _ptr(dev_status), flags, wait_limit_ns, _stream(stream)),
           "nle_varlen_attn_fwd_ex")


def varlen_attn(q, k, v, cu_seqlens, out=None, stream=None) -> torch.Tensor:
    """O = full attention inside each packed utterance ([frames, heads, 64] bf16 CUDA)."""
    if out is None:
        out = torch.empty_like(q)
    nle_varlen_attn_fwd(q, k, v, out, cu_seqlens, stream=stream)
    return out


# ------------------------------------------------------------------ windowed cross-attention
def nle_window_xattn_fwd(q, k, v, out, cu_seqlens_kv, n_seq: int | None = None, total_frames: int | None = None,
                         n_query_rows: int | None = None, heads: int | None = None, d_head: int | None = None,
                         window_frames: int = 15, queries_per_window: int = 3, stream=None) -> None:
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (out, "out")):
        _dev_tensor(t, n, torch.bfloat16)
    _dev_tensor(cu_seqlens_kv, "cu_seqlens_kv", torch.int32)
    n_seq = cu_seqlens_kv.numel() - 1 if n_seq is None else n_seq
    total_frames = k.shape[0] if total_frames is None else total_frames
    n_query_rows = q.shape[0] if n_query_rows is None else n_query_rows
    heads = q.shape[1] if heads is None else heads
    d_head = q.shape[2] if d_head is None else d_head
    _check(_lib.nle_window_xattn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(cu_seqlens_kv), n_seq,
                                     total_frames, n_query_rows, heads, d_head, window_frames,
                                     queries_per_window, _stream(stream)),
           "nle_window_xattn_fwd")


def nle_window_xattn_fwd_ex(q, k, v, out, cu_seqlens_kv, n_seq: int | None = None,
                            total_frames: int | None = None, n_query_rows: int | None = None,
                            heads: int | None = None, d_head: int = 64, window_frames: int = 15,
                            queries_per_window: int = 3, softmax_scale: float = 0.0, dev_status=None,
                            flags: int = 0, wait_limit_ns: int = 0, stream=None) -> None:
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (out, "out")):
        _dev_tensor(t, n, torch.bfloat16)
    _dev_tensor(cu_seqlens_kv, "cu_seqlens_kv", torch.int32)
    if dev_status is not None:
        _dev_tensor(dev_status, "dev_status", torch.int32)
    n_seq = cu_seqlens_kv.numel() - 1 if n_seq is None else n_seq
    total_frames = k.shape[0] if total_frames is None else total_frames
    n_query_rows = q.shape[0] if n_query_rows is None else n_query_rows
    heads = q.shape[1] if heads is None else heads
    _check(_lib.nle_window_xattn_fwd_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(cu_seqlens_kv), n_seq,
                                        total_frames, n_query_rows, heads, d_head, window_frames,
                                        queries_per_window, float(softmax_scale), _ptr(dev_status), flags,
                                        wait_limit_ns, _stream(stream)),
           "nle_window_xattn_fwd_ex")


def window_xattn(q, k, v, cu_seqlens_kv, window_frames: int = 15, queries_per_window: int = 3, out=None,
                 stream=None) -> torch.Tensor:
    if out is None:
        out = torch.empty_like(q)
    nle_window_xattn_fwd(q, k, v, out, cu_seqlens_kv, window_frames=window_frames,
                         queries_per_window=queries_per_window, stream=stream)
    return out


# ------------------------------------------------------------------ plans (host / device)
def _host_cu(cu) -> np.ndarray:
    if isinstance(cu, torch.Tensor):
        cu = cu.detach().cpu().numpy()
    return np.ascontiguousarray(np.asarray(cu, np.int32))


def nle_block_plan_host(cu_host, block_frames: int = 200):
    """(seq, j, start, len) int32 numpy arrays of the blocks."""
    cu = _host_cu(cu_host)
    n = _int(0)
    _check(_lib.nle_block_plan_host(_ptr(cu), len(cu) - 1, block_frames, None, None, None, None, 0,
                                    ctypes.byref(n)), "nle_block_plan_host")
    outs = [np.zeros(max(n.value, 1), np.int32) for _ in range(4)]
    _check(_lib.nle_block_plan_host(_ptr(cu), len(cu) - 1, block_frames, *[_ptr(o) for o in outs], n.value,
                                    ctypes.byref(n)), "nle_block_plan_host")
    return tuple(o[:n.value] for o in outs)


def nle_window_plan_host(cu_host, window_frames: int = 15, queries_per_window: int = 3):
    """(seq, w, start, len, q_row) int32 numpy arrays of the windows."""
    cu = _host_cu(cu_host)
    n = _int(0)
    _check(_lib.nle_window_plan_host(_ptr(cu), len(cu) - 1, window_frames, queries_per_window, None, None, None,
                                     None, None, 0, ctypes.byref(n)), "nle_window_plan_host")
    outs = [np.zeros(max(n.value, 1), np.int32) for _ in range(5)]
    _check(_lib.nle_window_plan_host(_ptr(cu), len(cu) - 1, window_frames, queries_per_window,
                                     *[_ptr(o) for o in outs], n.value, ctypes.byref(n)), "nle_window_plan_host")
    return tuple(o[:n.value] for o in outs)


def window_query_rows(cu_host, window_frames: int = 15, queries_per_window: int = 3) -> int:
    """Rows of the query tensor the windowed cross-attention expects."""
    cu = _host_cu(cu_host)
    n = _int(0)
    _check(_lib.nle_window_plan_host(_ptr(cu), len(cu) - 1, window_frames, queries_per_window, None, None, None,
                                     None, None, 0, ctypes.byref(n)), "nle_window_plan_host")
    return queries_per_window * n.value


def nle_block_plan_dev(cu_dev, total_frames: int, block_frames: int = 200, capacity: int | None = None,
                       stream=None):
    """Device copy of the block table: (seq, j, start, len) int32 CUDA tensors and the count tensor."""
    _dev_tensor(cu_dev, "cu_dev", torch.int32)
    n_seq = cu_dev.numel() - 1
    if capacity is None:
        capacity = n_seq + total_frames // block_frames
    dev = cu_dev.device
    outs = [torch.full((max(capacity, 1),), -7, dtype=torch.int32, device=dev) for _ in range(4)]
    count = torch.zeros(1, dtype=torch.int32, device=dev)
    _check(_lib.nle_block_plan_dev(_ptr(cu_dev), n_seq, total_frames, block_frames, *[_ptr(o) for o in outs],
                                   capacity, _ptr(count), _stream(stream)), "nle_block_plan_dev")
    return tuple(outs), count


def nle_shard_plan_host(lengths, world_size: int, block_frames: int = 200) -> np.ndarray:
    """Utterance ranges per rank: bounds[r]..bounds[r+1] (numpy int32 [world_size+1])."""
    ln = np.ascontiguousarray(np.asarray(lengths, np.int32))
    bounds = np.zeros(world_size + 1, np.int32)
    _check(_lib.nle_shard_plan_host(_ptr(ln), len(ln), block_frames, world_size, _ptr(bounds)),
           "nle_shard_plan_host")
    return bounds


# ------------------------------------------------------------------ whole path from host memory
_PATH_NAMES = ("q", "k", "v", "out", "qw", "kw", "vw", "out_w")


def nle_path_fwd_host(host: dict, dev: dict, block_frames: int = 200, window_frames: int = 15,
                      queries_per_window: int = 3, n_chunks: int = 0, stream=None, dev_status=None) -> None:
    """Both kernels from host memory (nle_path_fwd_host).  ``host`` and ``dev``
    map q, k, v, out, qw, kw, vw, out_w to bf16 [rows, heads, 64] tensors on the
    CPU (pinned for overlap) and on the GPU, and cu to int32 [n_seq + 1].
    ``dev_status`` (optional CUDA int32 [1]) receives the first in-kernel
    error (a wait that ran out).  Returns once the work is queued on
    ``stream``."""
    for name in _PATH_NAMES:
        h, d = host[name], dev[name]
        if h.device.type != "cpu" or h.dtype != torch.bfloat16 or not h.is_contiguous():
            raise ValueError(f"host {name}: contiguous CPU bf16 tensor required")
        _dev_tensor(d, f"dev {name}", torch.bfloat16)
        if h.shape != d.shape:
            raise ValueError(f"{name}: host {tuple(h.shape)} and device {tuple(d.shape)} differ")
    hcu, dcu = host["cu"], dev["cu"]
    if hcu.device.type != "cpu" or hcu.dtype != torch.int32 or not hcu.is_contiguous():
        raise ValueError("host cu: contiguous CPU int32 tensor required")
    _dev_tensor(dcu, "dev cu", torch.int32)
    if dev_status is not None:
        _dev_tensor(dev_status, "dev_status", torch.int32)
    b = PathBuffers(*[host[n].data_ptr() for n in _PATH_NAMES], hcu.data_ptr(),
                    *[dev[n].data_ptr() for n in _PATH_NAMES], dcu.data_ptr(),
                    dev_status.data_ptr() if dev_status is not None else None)
    heads = host["q"].shape[1]
    _check(_lib.nle_path_fwd_host(ctypes.byref(b), hcu.numel() - 1, host["q"].shape[0], host["qw"].shape[0],
                                  heads, host["q"].shape[2], block_frames, window_frames, queries_per_window,
                                  n_chunks, _stream(stream)),
           "nle_path_fwd_host")


# ------------------------------------------------------------------ CTC greedy decoding
def nle_ctc_greedy_fwd(logits, cu_seqlens, frame_class, tokens, n_tokens, n_classes: int | None = None,
                       stream=None) -> None:
    """logits: CUDA bf16 [frames, row_stride] (the first n_classes used);
    frame_class, tokens: int32 [frames]; n_tokens: int32 [n_seq]."""
    _dev_tensor(logits, "logits", torch.bfloat16)
    if logits.dim() != 2 or logits.stride(1) != 1:
        raise ValueError("logits: [frames, classes] with unit stride along classes")
    for t, n in ((cu_seqlens, "cu_seqlens"), (frame_class, "frame_class"), (tokens, "tokens"),
                 (n_tokens, "n_tokens")):
        _dev_tensor(t, n, torch.int32)
    n_classes = logits.shape[1] if n_classes is None else n_classes
    _check(_lib.nle_ctc_greedy_fwd(_ptr(logits), logits.stride(0), n_classes, _ptr(cu_seqlens),
                                   cu_seqlens.numel() - 1, logits.shape[0], _ptr(frame_class), _ptr(tokens),
                                   _ptr(n_tokens), _stream(stream)),
           "nle_ctc_greedy_fwd")


def ctc_greedy(logits, cu_seqlens, n_classes: int | None = None, stream=None):
    """(frame_class, tokens, n_tokens) of CTC greedy decoding on the GPU."""
    frames, n_seq = logits.shape[0], cu_seqlens.numel() - 1
    frame_class = torch.empty(frames, dtype=torch.int32, device=logits.device)
    tokens = torch.full((frames,), -1, dtype=torch.int32, device=logits.device)
    n_tokens = torch.empty(n_seq, dtype=torch.int32, device=logits.device)
    nle_ctc_greedy_fwd(logits, cu_seqlens, frame_class, tokens, n_tokens, n_classes, stream)
    return frame_class, tokens, n_tokens


# ------------------------------------------------------------------ posterior-weighted pooling
def pooled_rows(cu_host, pool_frames: int = 2) -> int:
    """Rows of the pooled output: one per window of pool_frames frames."""
    return window_query_rows(cu_host, pool_frames, 1)


def nle_posterior_pool_fwd(hidden, logits, cu_seqlens, pooled, weights=None, pool_frames: int = 2,
                           n_classes: int | None = None, dev_status=None, stream=None) -> None:
    """hidden: CUDA bf16 [frames, hidden_stride] (the first pooled.shape[1]
    columns used); logits: CUDA bf16 [frames, logits_stride] of the mid-layer
    head (the first n_classes used, blank at 0); pooled: bf16 [rows, dim];
    weights: None or float32 [frames]; dev_status: None or int32 [1]."""
    _dev_tensor(hidden, "hidden", torch.bfloat16)
    _dev_tensor(logits, "logits", torch.bfloat16)
    _dev_tensor(pooled, "pooled", torch.bfloat16)
    _dev_tensor(cu_seqlens, "cu_seqlens", torch.int32)
    for t, n in ((hidden, "hidden"), (logits, "logits"), (pooled, "pooled")):
        if t.dim() != 2 or t.stride(1) != 1:
            raise ValueError(f"{n}: 2-D with unit stride along its last dimension")
    if not pooled.is_contiguous():
        raise ValueError("pooled: contiguous [rows, dim] required")
    if weights is not None:
        _dev_tensor(weights, "weights", torch.float32)
    if dev_status is not None:
        _dev_tensor(dev_status, "dev_status", torch.int32)
    if hidden.shape[0] != logits.shape[0]:
        raise ValueError("hidden and logits: different frame counts")
    n_classes = logits.shape[1] if n_classes is None else n_classes
    _check(_lib.nle_posterior_pool_fwd(_ptr(hidden), hidden.stride(0), pooled.shape[1], _ptr(logits),
                                       logits.stride(0), n_classes, _ptr(cu_seqlens), cu_seqlens.numel() - 1,
                                       hidden.shape[0], pool_frames, pooled.shape[0], _ptr(pooled),
                                       _ptr(weights), _ptr(dev_status), _stream(stream)),
           "nle_posterior_pool_fwd")


def posterior_pool(hidden, logits, cu_seqlens, pool_frames: int = 2, n_rows: int | None = None,
                   dim: int | None = None, n_classes: int | None = None, stream=None):
    """(pooled bf16 [rows, dim], weights float32 [frames]) on the GPU.  n_rows
    defaults to the windows of cu_seqlens (read back to the host)."""
    if n_rows is None:
        n_rows = pooled_rows(cu_seqlens.cpu(), pool_frames)
    dim = hidden.shape[1] if dim is None else dim
    pooled = torch.empty((n_rows, dim), dtype=torch.bfloat16, device=hidden.device)
    weights = torch.empty(hidden.shape[0], dtype=torch.float32, device=hidden.device)
    nle_posterior_pool_fwd(hidden, logits, cu_seqlens, pooled, weights, pool_frames, n_classes, None, stream)
    return pooled, weights
