"""GPU parity of posterior-weighted pooling (nle_posterior_pool_fwd) against
the fp64 oracle.  Pooled rows are bf16: rel-L2 <= 5e-3 and max-abs <= 2e-2
per tensor (the path's tolerance; the kernel's error is the final bf16
rounding, <= 2^-9 relative, plus fp32 sums).  Weights are fp32: within
1e-5 relative + 1e-6 absolute (one exp, two logs and fp32 sums of <= 1000
terms)."""
import json
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from chunked_block_self_b200 import workloads as wl

pytestmark = pytest.mark.gpu
GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "posterior_pool.json")
REL_L2, MAX_ABS = 5e-3, 2e-2


def _nle():
    from chunked_block_self_b200 import nle
    return nle


def _run(hidden, logits, cu, dev, P, dim=None, n_classes=None, n_rows=None):
    nle = _nle()
    cu_d = torch.from_numpy(np.asarray(cu, np.int32)).to(dev)
    if n_rows is None:
        n_rows = int(oracle.pooled_rows(cu, P)[-1])
    pooled, w = nle.posterior_pool(hidden.to(dev), logits.to(dev), cu_d, P, n_rows=n_rows, dim=dim,
                                   n_classes=n_classes)
    torch.cuda.synchronize()
    return pooled.float().cpu().double().numpy(), w.cpu().double().numpy()


def _compare(got, ref):
    if ref.size == 0:
        assert got.size == 0
        return
    nrm = np.linalg.norm(ref)
    err = np.linalg.norm(got - ref)
    assert err <= REL_L2 * max(nrm, 1e-30) or err == 0.0, f"rel-L2 {err / nrm:.3e}"
    assert np.abs(got - ref).max() <= MAX_ABS


def _check(x, cu, dev, P, dim, n_classes):
    got, gw = _run(x["hidden"], x["logits"], cu, dev, P, dim, n_classes)
    ref, rw = oracle.posterior_pool(x["hidden"][:, :dim], x["logits"][:, :n_classes], cu, P)
    _compare(got, ref)
    np.testing.assert_allclose(gw, rw, rtol=1e-5, atol=1e-6)
    # zero-weight windows are exact zero rows
    lw = oracle.pool_log_weights(x["logits"][:, :n_classes])
    rows = oracle.pooled_rows(cu, P)
    for i in range(len(cu) - 1):
        for j, a in enumerate(range(int(cu[i]), int(cu[i + 1]), P)):
            if np.all(lw[a:min(a + P, int(cu[i + 1]))] == -np.inf):
                assert np.all(got[rows[i] + j] == 0.0)


@pytest.mark.parametrize("case", json.load(open(GOLDEN))["cases"], ids=lambda c: c["name"])
def test_golden_cases(case, cuda_device):
    # the fixtures have 2 hidden columns; the kernel pools 16-byte chunks, so
    # they ride in the first 2 of 8 columns (the other 6 are zero)
    z = [[float("-inf") if v == "-inf" else float(v) for v in row] for row in case["logits"]]
    logits = torch.tensor(z, dtype=torch.float32).to(torch.bfloat16)
    h = np.zeros((len(case["hidden"]), 8), np.float32)
    h[:, :2] = case["hidden"]
    got, gw = _run(torch.from_numpy(h).to(torch.bfloat16), logits, case["cu"], cuda_device, case["pool_frames"])
    want = np.array([[float(Fraction(x)) for x in row] for row in case["pooled"]])
    assert np.all(got[:, 2:] == 0.0)
    # bf16 rounding of the pooled values (|x| <= 8: <= 2^-6 absolute)
    np.testing.assert_allclose(got[:, :2], want, rtol=2 ** -8, atol=1e-7)
    np.testing.assert_allclose(gw, [float(Fraction(x)) for x in case["weights"]], rtol=1e-6, atol=1e-7)


@pytest.mark.parametrize("P,dim,n_classes,pads", [
    (2, 1024, 256, (0, 0)), (1, 8, 1, (0, 0)), (2, 8, 2, (8, 1)), (3, 24, 37, (16, 3)), (4, 1024, 256, (8, 5)),
    (7, 64, 1000, (0, 7)), (2, 1032, 2, (0, 0)), (16, 128, 5, (0, 2)),
    # the pipelined path (P <= 2, dim <= 1024, classes <= 256 in 16-byte chunks), with 1-4
    # hidden chunks per lane, some lanes without a chunk, and fewer than 32 logit chunks
    (1, 1024, 256, (0, 0)), (3, 64, 8, (8, 8)), (4, 1024, 256, (8, 0)), (2, 8, 16, (0, 0)),
    (4, 1000, 248, (16, 8)), (2, 512, 64, (0, 0)), (2, 640, 128, (8, 8)), (1, 264, 8, (0, 0)),
    (2, 776, 200, (24, 16)), (2, 1000, 256, (0, 0))])
def test_random_shapes(P, dim, n_classes, pads, cuda_device):
    lengths = [37, 0, 1, 200, 5, 64, 3]
    cu = wl.cu_seqlens(lengths)
    x = wl.pool_inputs(lengths, dim, n_classes, seed=P * 1000 + dim + n_classes,
                       hidden_stride=dim + pads[0], logits_stride=n_classes + pads[1])
    _check(x, cu, cuda_device, P, dim, n_classes)


@pytest.mark.parametrize("C", [6, 8])   # the general and the pipelined path
def test_degenerate_weights(C, cuda_device):
    """Only the blank (every weight 0 -> zero rows), a -inf blank (weight
    exactly 1), and a blank far above the rest (weights below fp32's range;
    their window is still their weighted mean)."""
    lengths = [6, 4, 5]
    cu = wl.cu_seqlens(lengths)
    T, D = 15, 16
    rng = np.random.default_rng(7)
    z = rng.standard_normal((T, C)).astype(np.float32)
    z[0:6, 1:] = -np.inf          # utterance 0: every weight 0
    z[6:8, 0] = -np.inf           # weight 1
    z[10:12, 0] = 800.0           # utterance 2, window 0: both weights ~e^-800
    z[11, 1] = 3.0
    h = rng.standard_normal((T, D)).astype(np.float32)
    x = dict(hidden=torch.from_numpy(h).to(torch.bfloat16), logits=torch.from_numpy(z).to(torch.bfloat16))
    _check(x, cu, cuda_device, 2, D, C)
    got, gw = _run(x["hidden"], x["logits"], cu, cuda_device, 2)
    assert np.all(got[:3] == 0.0) and np.all(gw[:6] == 0.0)
    assert np.all(gw[6:8] == 1.0)


@pytest.mark.parametrize("n_classes", [4, 8])   # the general and the pipelined path
def test_rows_short_reported_and_untouched(n_classes, cuda_device):
    """Too few pooled rows for the windows: rows past the buffer are never
    written and the status says so."""
    nle = _nle()
    lengths = [9, 7]
    cu = wl.cu_seqlens(lengths)
    x = wl.pool_inputs(lengths, 16, n_classes, seed=5)
    n_rows = int(oracle.pooled_rows(cu, 2)[-1])
    guard = torch.full((n_rows + 4, 16), 7.0, dtype=torch.bfloat16, device=cuda_device)
    status = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    cu_d = torch.from_numpy(cu).to(cuda_device)
    short = guard[:n_rows - 3]
    nle.nle_posterior_pool_fwd(x["hidden"].to(cuda_device), x["logits"].to(cuda_device), cu_d, short,
                               None, 2, None, status)
    torch.cuda.synchronize()
    assert int(status.item()) == -1
    assert torch.all(guard[n_rows - 3:] == 7.0)
    ref, _ = oracle.posterior_pool(x["hidden"], x["logits"], cu, 2)
    _compare(short.float().cpu().double().numpy(), ref[:n_rows - 3])


@pytest.mark.parametrize("n_classes", [4, 8])   # the general and the pipelined path
def test_invalid_offsets_reported(n_classes, cuda_device):
    nle = _nle()
    x = wl.pool_inputs([8], 16, n_classes, seed=6)
    cu_bad = torch.tensor([0, 9], dtype=torch.int32, device=cuda_device)   # past total_frames
    out = torch.full((4, 16), 7.0, dtype=torch.bfloat16, device=cuda_device)
    status = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    nle.nle_posterior_pool_fwd(x["hidden"].to(cuda_device), x["logits"].to(cuda_device), cu_bad, out, None, 2,
                               None, status)
    torch.cuda.synchronize()
    assert int(status.item()) == -1
    assert torch.all(out == 7.0)


def test_full_size_sampled(cuda_device):
    """Batch-128 workload at full size (58,903 frames x 1024, 256 mid-layer
    classes, windows of 2 -> 29,4xx rows), generated on the device: 300
    sampled windows against the oracle, and every weight of the batch."""
    nle = _nle()
    lengths = wl.draw_lengths(4)
    cu = wl.cu_seqlens(lengths)
    x = wl.pool_inputs(lengths, seed=77, device=cuda_device)
    cu_d = torch.from_numpy(cu).to(cuda_device)
    pooled, w = nle.posterior_pool(x["hidden"], x["logits"], cu_d, 2, n_rows=int(oracle.pooled_rows(cu, 2)[-1]))
    torch.cuda.synchronize()
    rows = oracle.pooled_rows(cu, 2)
    rng = np.random.default_rng(8)
    got, ref = [], []
    for _ in range(300):
        i = int(rng.integers(0, len(lengths)))
        j = int(rng.integers(0, rows[i + 1] - rows[i]))
        a = int(cu[i]) + 2 * j
        b = min(a + 2, int(cu[i + 1]))
        r, _ = oracle.posterior_pool(x["hidden"][a:b].cpu(), x["logits"][a:b].cpu(), [0, b - a], 2)
        ref.append(r[0])
        got.append(pooled[rows[i] + j].float().cpu().double().numpy())
    _compare(np.array(got), np.array(ref))
    rw = oracle.blank_weights(x["logits"][:2000].cpu())
    np.testing.assert_allclose(w[:2000].cpu().double().numpy(), rw, rtol=1e-5, atol=1e-6)


def test_full_size_every_row(cuda_device):
    """Batch-128 workload at full size (58,903 frames x 1024, 256 mid-layer
    classes, windows of 2), generated on the device: every pooled row and
    every weight against the oracle."""
    nle = _nle()
    lengths = wl.draw_lengths(4)
    cu = wl.cu_seqlens(lengths)
    x = wl.pool_inputs(lengths, seed=77, device=cuda_device)
    cu_d = torch.from_numpy(cu).to(cuda_device)
    n_rows = int(oracle.pooled_rows(cu, 2)[-1])
    pooled, w = nle.posterior_pool(x["hidden"], x["logits"], cu_d, 2, n_rows=n_rows)
    torch.cuda.synchronize()
    ref, rw = oracle.posterior_pool(x["hidden"].cpu(), x["logits"].cpu(), cu, 2)
    _compare(pooled.float().cpu().double().numpy(), ref)
    np.testing.assert_allclose(w.cpu().double().numpy(), rw, rtol=1e-5, atol=1e-6)


@pytest.mark.parametrize("P", [3072, 3073, 4096])
def test_largest_pool_windows(P, cuda_device):
    """Windows of up to 4096 frames (the documented maximum), whose per-warp
    weight buffers need more than the default 48 KB of shared memory."""
    lengths = [2 * P + 5, P, 17]
    cu = wl.cu_seqlens(lengths)
    x = wl.pool_inputs(lengths, 64, 37, seed=P)
    _check(x, cu, cuda_device, P, 64, 37)
