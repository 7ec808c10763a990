"""nle_path_fwd_host: both kernels from host memory, pipelined over chunks
of utterances, must give exactly the device-path results (same kernels on
the same rows; chunks only split the batch between utterances)."""
import ctypes

import numpy as np
import pytest
import torch

from chunked_block_self_b200 import nle
from chunked_block_self_b200 import workloads as wl

W, QW, B = 15, 3, 200


def _inputs(n_utt, seed):
    lengths = wl.draw_lengths(4)[:n_utt]
    x = wl.block_inputs(lengths=lengths, heads=16, seed=seed)
    n_win = sum(-(-int(t) // W) for t in lengths)
    y = wl.window_inputs(QW * n_win, cfg=None, lengths=lengths, heads=16, seed=seed + 1)
    host = {"q": x["q"], "k": x["k"], "v": x["v"], "qw": y["q"], "kw": y["k"], "vw": y["v"],
            "out": torch.empty_like(x["q"]), "out_w": torch.empty_like(y["q"]),
            "cu": torch.from_numpy(np.ascontiguousarray(x["cu"]))}
    return host


def _device_reference(host, dev):
    d = {n: host[n].to(dev) for n in ("q", "k", "v", "qw", "kw", "vw", "cu")}
    out = nle.block_attn(d["q"], d["k"], d["v"], d["cu"], block_frames=B)
    out_w = nle.window_xattn(d["qw"], d["kw"], d["vw"], d["cu"], window_frames=W, queries_per_window=QW)
    torch.cuda.synchronize()
    return out.cpu(), out_w.cpu()


@pytest.mark.gpu
@pytest.mark.parametrize("chunks,pinned", [(1, True), (3, True), (8, True), (0, False)])
def test_host_path_equals_device_path(chunks, pinned, cuda_device):
    host = _inputs(40, seed=501)
    if pinned:
        host = {n: t.pin_memory() for n, t in host.items()}
    ref, ref_w = _device_reference(host, cuda_device)
    dev = {n: torch.empty(t.shape, dtype=t.dtype, device=cuda_device) for n, t in host.items()}
    host["out"].fill_(float("nan"))
    host["out_w"].fill_(float("nan"))
    status = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    nle.nle_path_fwd_host(host, dev, block_frames=B, window_frames=W, queries_per_window=QW, n_chunks=chunks,
                          dev_status=status)
    torch.cuda.current_stream().synchronize()
    assert int(status.item()) == 0
    assert torch.equal(host["out"], ref)
    assert torch.equal(host["out_w"], ref_w)


@pytest.mark.gpu
def test_host_path_orders_after_and_before_the_stream(cuda_device):
    """Work queued before the call is finished before its copies start, and
    work queued after it sees its outputs."""
    host = {n: t.pin_memory() for n, t in _inputs(12, seed=502).items()}
    ref, _ = _device_reference(host, cuda_device)
    dev = {n: torch.empty(t.shape, dtype=t.dtype, device=cuda_device) for n, t in host.items()}
    stream = torch.cuda.Stream(device=cuda_device)
    with torch.cuda.stream(stream):
        dev["out"].fill_(0)                       # queued before: must not overwrite the result
        nle.nle_path_fwd_host(host, dev, n_chunks=4)
        echo = dev["out"].clone()                 # queued after: must see the result
    stream.synchronize()
    assert torch.equal(host["out"], ref)
    assert torch.equal(echo.cpu(), ref)


def test_host_path_rejects_bad_tables():
    """Argument checks made on the host before any CUDA call."""
    lengths = [30, 0, 17]
    cu = np.array([0, 30, 30, 47], np.int32)
    n_win = sum(-(-t // W) for t in lengths)
    dummy = 1 << 20   # never dereferenced: the checks return first
    b = nle.PathBuffers(*([dummy] * 8), cu.ctypes.data, *([dummy] * 9))
    call = lambda b_, rows, total=47: nle._lib.nle_path_fwd_host(ctypes.byref(b_), 3, total, rows, 16, 64, B, W,
                                                                QW, 0, None)
    assert call(b, QW * n_win + 3) == nle.NLE_ERR_INVALID_ARG          # query rows do not match
    assert call(b, QW * n_win, total=50) == nle.NLE_ERR_INVALID_ARG    # cu[n_seq] != total_frames
    bad = np.array([0, 30, 20, 47], np.int32)                          # decreasing offsets
    b2 = nle.PathBuffers(*([dummy] * 8), bad.ctypes.data, *([dummy] * 9))
    assert call(b2, QW * n_win) == nle.NLE_ERR_INVALID_ARG
    b3 = nle.PathBuffers(*([dummy] * 8), cu.ctypes.data, *([dummy] * 8), None)   # no device cu
    assert call(b3, QW * n_win) == nle.NLE_ERR_INVALID_ARG


@pytest.mark.gpu
def test_host_path_full_batch_against_oracle(cuda_device):
    """The whole batch-128 workload (128 utterances, 58,903 frames, 3,992
    windows) through the host-memory entry point with its default chunking:
    bit-equal to the device path, and every output of both kernels within
    the path's tolerance of the fp64 oracle (rel-L2 <= 5e-3, max-abs <= 2e-2
    per tensor)."""
    import oracle

    host = {n: t.pin_memory() for n, t in _inputs(128, seed=503).items()}
    ref, ref_w = _device_reference(host, cuda_device)
    dev = {n: torch.empty(t.shape, dtype=t.dtype, device=cuda_device) for n, t in host.items()}
    host["out"].fill_(float("nan"))
    host["out_w"].fill_(float("nan"))
    status = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    nle.nle_path_fwd_host(host, dev, block_frames=B, window_frames=W, queries_per_window=QW, dev_status=status)
    torch.cuda.current_stream().synchronize()
    assert int(status.item()) == 0
    assert torch.equal(host["out"], ref)
    assert torch.equal(host["out_w"], ref_w)
    cu = host["cu"].numpy()
    want = oracle.block_attn(host["q"], host["k"], host["v"], cu, block_frames=B)
    want_w = oracle.window_xattn(host["qw"], host["kw"], host["vw"], cu, window_frames=W, queries_per_window=QW)
    for got, exp in ((host["out"], want), (host["out_w"], want_w)):
        g = got.float().numpy().astype(np.float64)
        err = g - exp
        rel = np.linalg.norm(err) / np.linalg.norm(exp)
        assert rel <= 5e-3 and np.abs(err).max() <= 2e-2, f"rel_l2={rel:.3e} max_abs={np.abs(err).max():.3e}"
