"""GPU parity of the QKV projection fused with block self-attention
(nle_block_attn_qkv_fwd) against the fp64 oracle (oracle/qkv.py: X W^T (+ b)
in fp64, then the block definition in fp64).

Tolerance: relative L2 error <= 5e-3 and max-abs <= 2e-2, as for the block
kernel.  The fused path rounds once more than the block kernel (Q, K and V to
bf16 after the fp32 projection); with unit-variance Q and K that adds about
2e-3 relative to S and V, well inside the bound.  Block locality is compared
bit for bit: rows of other blocks (NaN and Inf included) never reach a
block's output."""
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


def _inputs(lengths, heads, d_model, seed, bias=False):
    rng = np.random.default_rng(seed)
    cu = wl.cu_seqlens(lengths)
    T = int(cu[-1])
    x = torch.from_numpy(rng.standard_normal((T, d_model), dtype=np.float32)).to(torch.bfloat16)
    w = torch.from_numpy((rng.standard_normal((3 * heads * 64, d_model), dtype=np.float32)
                          / np.float32(np.sqrt(d_model)))).to(torch.bfloat16)
    b = None
    if bias:
        b = torch.from_numpy(rng.standard_normal(3 * heads * 64, dtype=np.float32) * np.float32(0.5)).to(
            torch.bfloat16)
    return dict(x=x, w=w, b=b, cu=cu, heads=heads, T=T)


def _run(a, dev, B=200, **kw):
    nle = _nle()
    x, w = a["x"].to(dev), a["w"].to(dev)
    b = a["b"].to(dev) if a["b"] is not None else None
    cu = torch.from_numpy(a["cu"]).to(dev)
    out = torch.full((a["T"], a["heads"], 64), float("nan"), dtype=torch.bfloat16, device=dev)
    if kw:
        nle.nle_block_attn_qkv_fwd_ex(x, w, b, out, cu, block_frames=B, **kw)
    else:
        nle.nle_block_attn_qkv_fwd(x, w, b, out, cu, block_frames=B)
    torch.cuda.synchronize()
    return out


def _ref(a, B=200, scale=None):
    bias = None if a["b"] is None else a["b"].double().numpy()
    return oracle.block_attn_qkv(a["x"], a["w"], a["cu"], a["heads"], block_frames=B, bias=bias, scale=scale)


def _compare(got, ref):
    g = got.float().cpu().double().numpy()
    assert np.isfinite(g).all(), "non-finite output"
    err = g - ref
    rel = np.linalg.norm(err) / max(np.linalg.norm(ref), 1e-30)
    mx = np.abs(err).max() if err.size else 0.0
    assert rel <= REL_L2 and mx <= MAX_ABS, f"rel_l2={rel:.3e} max_abs={mx:.3e}"
    return rel, mx


@pytest.mark.parametrize("lengths,heads,d_model,bias", [
    ([400], 2, 128, False),
    ([1], 1, 64, True),
    ([127, 128, 129], 3, 192, True),
    ([200, 201, 55, 0, 399], 2, 256, False),
    ([0, 5, 0, 333, 1, 0], 4, 256, True),
])
def test_ragged_full_parity(lengths, heads, d_model, bias, cuda_device):
    a = _inputs(lengths, heads, d_model, seed=sum(lengths) + heads + d_model, bias=bias)
    _compare(_run(a, cuda_device), _ref(a))


@pytest.mark.parametrize("seed", range(10))
def test_random_batches(seed, cuda_device):
    """Seeded random batches: many short utterances (a projection tile of 128
    frames then holds many blocks, some of them a frame long) mixed with long
    ones, block lengths from 16 to 256, 1 to 4 heads, d_model 64 to 256,
    with and without a bias."""
    rng = np.random.default_rng(900 + seed)
    B = int(rng.choice([16, 64, 100, 129, 200, 256]))
    n = int(rng.integers(1, 40))
    lengths = [int(x) for x in rng.choice([0, 1, 2, 3, 7, 15, 64, 127, 128, 129, 200, 257, 600], n)]
    if sum(lengths) == 0:
        lengths[0] = 5
    heads = int(rng.integers(1, 5))
    d_model = int(rng.choice([64, 128, 192, 256]))
    a = _inputs(lengths, heads, d_model, seed=1000 + seed, bias=bool(seed % 2))
    _compare(_run(a, cuda_device, B=B), _ref(a, B=B))


def test_encoder_shape_batch_slice(cuda_device):
    """The encoder's shape (d_model 1024, 16 heads) on 24 utterances of the
    batch-128 workload, with a bias."""
    a = _inputs(wl.draw_lengths(4)[:24], 16, 1024, seed=401, bias=True)
    _compare(_run(a, cuda_device), _ref(a))


def test_batch128_full_size_every_output(cuda_device):
    """The batch-128 workload at full size (128 utterances, 58,903 frames,
    d_model 1024, 16 heads): every output against the oracle, as one tensor
    and (block, head) by (block, head) within twice the tolerance."""
    a = _inputs(wl.draw_lengths(4), 16, 1024, seed=402, bias=True)
    out = _run(a, cuda_device)
    ref = _ref(a)
    _compare(out, ref)
    g = out.float().cpu().double().numpy()
    seq, j, start, ln = oracle.block_table(a["cu"], 200)
    worst = 0.0
    for s0, n in zip(start.tolist(), ln.tolist()):
        e = np.linalg.norm(g[s0:s0 + n] - ref[s0:s0 + n], axis=(0, 2))
        r = np.maximum(np.linalg.norm(ref[s0:s0 + n], axis=(0, 2)), 1e-30)
        worst = max(worst, float((e / r).max()))
    assert worst <= 2 * REL_L2, f"worst item rel_l2={worst:.3e}"


@pytest.mark.parametrize("B", [1, 16, 100, 128, 129, 208, 256])
def test_block_frames_variants(B, cuda_device):
    a = _inputs([3 * B + 5, B, 2], 2, 128, seed=B + 7)
    _compare(_run(a, cuda_device, B=B), _ref(a, B=B))


def test_scale_and_status(cuda_device):
    """A scale other than 1/sqrt(64).  The bf16 rounding of Q and K moves S
    by an amount proportional to the scale, so the check uses 0.1 (a softmax
    a little flatter than the default's); at 0.3 the max-abs error reaches
    about 2.3e-2 on this input."""
    a = _inputs([250, 90], 2, 128, seed=9, bias=True)
    status = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    out = _run(a, cuda_device, softmax_scale=0.1, dev_status=status)
    assert int(status.item()) == 0
    _compare(out, _ref(a, scale=0.1))


def test_block_locality_bit_exact(cuda_device):
    """Changing every input row outside block [200, 400) of utterance 0 (to
    NaN and Inf too) leaves that block's outputs unchanged bit for bit: the
    projection's rows of other frames never reach the block's keys, values
    or queries."""
    a = _inputs([530, 90], 4, 128, seed=10)
    out = _run(a, cuda_device)
    b = dict(a)
    x = a["x"].clone()
    x[:200] = -3 * x[:200]
    x[400:] = x[400:] + 1
    x[400:402] = float("nan")
    x[402:404] = float("inf")
    x[150:200] = float("inf")
    b["x"] = x
    out2 = _run(b, cuda_device)
    assert torch.equal(out2[200:400], out[200:400])
    assert not torch.equal(out2[:150], out[:150])


def test_invalid_offsets_reported_without_stray_writes(cuda_device):
    nle = _nle()
    a = _inputs([100, 100], 2, 128, seed=11)
    x, w = a["x"].to(cuda_device), a["w"].to(cuda_device)
    big = torch.full((200 + 16, 2, 64), 55.0, dtype=torch.bfloat16, device=cuda_device)
    out = big[8:208]
    status = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    bad_cu = torch.tensor([0, 100, 400], dtype=torch.int32, device=cuda_device)   # beyond total
    nle.nle_block_attn_qkv_fwd_ex(x, w, None, out, bad_cu, total_frames=200, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == nle.NLE_ERR_INVALID_ARG
    assert (big[:8] == 55.0).all() and (big[208:] == 55.0).all()
    first = dict(a, x=a["x"][:100], cu=np.array([0, 100], np.int32), T=100)
    _compare(out[:100], _ref(first))
    assert (out[100:] == 55.0).all()


def test_timeout_path_reports_and_recovers(cuda_device):
    """The test hook withholds the first load: the bounded waits expire, the
    kernel reports NLE_ERR_TIMEOUT and the next launch is correct."""
    nle = _nle()
    a = _inputs([400, 300], 2, 128, seed=12)
    status = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    _run(a, cuda_device, dev_status=status, flags=nle.NLE_FLAG_TEST_SKIP_FIRST_LOAD, wait_limit_ns=2_000_000)
    assert int(status.item()) == nle.NLE_ERR_TIMEOUT
    _compare(_run(a, cuda_device), _ref(a))
