"""GPU parity of the windowed cross-attention kernel against the fp64 oracle
(same tolerance as the block attention: rel-L2 <= 5e-3, max-abs <= 2e-2)."""
import numpy as np
import pytest
import torch

import oracle
from chunked_block_self_b200 import workloads as wl

pytestmark = pytest.mark.gpu

REL_L2 = 5e-3
MAX_ABS = 2e-2


def _nle():
    from chunked_block_self_b200 import nle
    return nle


def _inputs(lengths, heads, seed, W=15, Qw=3):
    nq = Qw * len(oracle.window_table(wl.cu_seqlens(lengths), W, Qw)[0])
    return wl.window_inputs(nq, cfg=None, lengths=lengths, heads=heads, seed=seed)


def _run(x, dev, W=15, Qw=3, **kw):
    nle = _nle()
    q, k, v = (x[n].to(dev) for n in ("q", "k", "v"))
    cu = torch.from_numpy(x["cu"]).to(dev)
    out = torch.full_like(q, float("nan"))
    if kw:
        nle.nle_window_xattn_fwd_ex(q, k, v, out, cu, window_frames=W, queries_per_window=Qw, **kw)
    else:
        nle.nle_window_xattn_fwd(q, k, v, out, cu, window_frames=W, queries_per_window=Qw)
    torch.cuda.synchronize()
    return out


def _compare(got, ref):
    g = got.float().cpu().double().numpy()
    assert np.isfinite(g).all(), "non-finite output"
    err = g - ref
    rel = np.linalg.norm(err) / max(np.linalg.norm(ref), 1e-30)
    mx = np.abs(err).max() if err.size else 0.0
    assert rel <= REL_L2 and mx <= MAX_ABS, f"rel_l2={rel:.3e} max_abs={mx:.3e}"


@pytest.mark.parametrize("lengths,heads", [
    ([15], 16), ([4700], 16), ([1, 14, 15, 16, 29, 30, 31], 5), ([0, 47, 0, 3], 2), ([200] * 9, 16),
])
def test_window_full_parity(lengths, heads, cuda_device):
    x = _inputs(lengths, heads, seed=sum(lengths))
    out = _run(x, cuda_device)
    _compare(out, oracle.window_xattn(x["q"], x["k"], x["v"], x["cu"], 15, 3))


@pytest.mark.parametrize("W,Qw", [(1, 1), (8, 2), (16, 3), (17, 3), (32, 8), (15, 5)])
def test_window_shape_variants(W, Qw, cuda_device):
    x = _inputs([3 * W + 2, W, 1], 3, seed=W * 10 + Qw, W=W, Qw=Qw)
    out = _run(x, cuda_device, W=W, Qw=Qw)
    _compare(out, oracle.window_xattn(x["q"], x["k"], x["v"], x["cu"], W, Qw))


def test_config5_full_size_sampled(cuda_device):
    cu = wl.cu_seqlens(wl.draw_lengths(5))
    nq = 3 * len(oracle.window_table(cu, 15, 3)[0])
    x = wl.window_inputs(nq, cfg=5)
    out = _run(x, cuda_device)
    rng = np.random.default_rng(5)
    rows = np.concatenate([rng.integers(0, nq, 3000), np.arange(939, nq, 942)])  # + every partial window
    hs = rng.integers(0, 16, len(rows))
    ref = oracle.window_xattn_rows(x["q"], x["k"], x["v"], x["cu"], rows, hs, 15, 3)
    got = out[torch.from_numpy(rows).to(cuda_device), torch.from_numpy(hs).to(cuda_device)]
    _compare(got, ref)
    assert torch.isfinite(out.float()).all()


def test_config5_full_size_every_output(cuda_device):
    """Config 5 (64 utterances of 4700 frames, 20,096 windows, 16 heads) at
    full size: every query row of the launch against the oracle, as one
    tensor within the tolerance and window by window (every (window, head)
    within twice it)."""
    cu = wl.cu_seqlens(wl.draw_lengths(5))
    nq = 3 * len(oracle.window_table(cu, 15, 3)[0])
    x = wl.window_inputs(nq, cfg=5)
    out = _run(x, cuda_device)
    ref = oracle.window_xattn(x["q"], x["k"], x["v"], x["cu"], 15, 3)
    _compare(out, ref)
    g = out.float().cpu().double().numpy().reshape(nq // 3, 3, 16, 64)
    r = ref.reshape(nq // 3, 3, 16, 64)
    e = np.linalg.norm(g - r, axis=(1, 3)) / np.maximum(np.linalg.norm(r, axis=(1, 3)), 1e-30)
    assert e.max() <= 2 * REL_L2, f"worst window rel_l2={e.max():.3e}"


def test_window_locality_bit_exact(cuda_device):
    x = _inputs([47, 15], 4, seed=41)
    out = _run(x, cuda_device)
    for n in ("k", "v"):
        x[n][:45] = float("nan")
        x[n][47:] = float("inf")
    out2 = _run(x, cuda_device)
    assert torch.equal(out2[9:12], out[9:12])   # window [45, 47)


def test_window_scale_and_status(cuda_device):
    nle = _nle()
    x = _inputs([40, 7], 2, seed=42)
    status = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    out = _run(x, cuda_device, softmax_scale=0.2, dev_status=status)
    assert int(status.item()) == 0
    _compare(out, oracle.window_xattn(x["q"], x["k"], x["v"], x["cu"], 15, 3, scale=0.2))


def test_window_short_query_tensor_is_reported(cuda_device):
    nle = _nle()
    x = _inputs([45, 30], 2, seed=43)           # 5 windows -> 15 query rows
    dev = cuda_device
    q = x["q"][:12].to(dev)                     # one window short
    k, v = x["k"].to(dev), x["v"].to(dev)
    big = torch.full((12 + 8, 2, 64), 9.0, dtype=torch.bfloat16, device=dev)
    out = big[:12]
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    nle.nle_window_xattn_fwd_ex(q, k, v, out, torch.from_numpy(x["cu"]).to(dev), dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == nle.NLE_ERR_INVALID_ARG
    assert (big[12:] == 9.0).all()
    ref = oracle.window_xattn(x["q"], x["k"], x["v"], x["cu"], 15, 3)
    _compare(out, ref[:12])


def test_window_timeout_path(cuda_device):
    nle = _nle()
    x = _inputs([150, 60], 2, seed=44)
    status = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    _run(x, cuda_device, dev_status=status, flags=nle.NLE_FLAG_TEST_SKIP_FIRST_LOAD, wait_limit_ns=2_000_000)
    assert int(status.item()) == nle.NLE_ERR_TIMEOUT
    out = _run(x, cuda_device)
    _compare(out, oracle.window_xattn(x["q"], x["k"], x["v"], x["cu"], 15, 3))
