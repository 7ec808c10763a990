"""GPU parity of CTC greedy decoding (nle_ctc_greedy_fwd) against the oracle:
integer results, compared exactly."""
import json
import os

import numpy as np
import pytest
import torch

import oracle
from chunked_block_self_b200 import workloads as wl

pytestmark = pytest.mark.gpu
GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "ctc_greedy.json")


def _nle():
    from chunked_block_self_b200 import nle
    return nle


def _decode(logits_host, cu, dev, n_classes=None):
    nle = _nle()
    lg = logits_host.to(dev)
    cu_d = torch.from_numpy(np.asarray(cu, np.int32)).to(dev)
    fc, tok, nt = nle.ctc_greedy(lg, cu_d, n_classes=n_classes)
    torch.cuda.synchronize()
    return fc.cpu().numpy(), tok.cpu().numpy(), nt.cpu().numpy()


def _check(logits_host, cu, dev, n_classes=None):
    fc, tok, nt = _decode(logits_host, cu, dev, n_classes)
    ref_logits = logits_host if n_classes is None else logits_host[:, :n_classes]
    cls, toks = oracle.ctc_greedy(ref_logits, cu)
    np.testing.assert_array_equal(fc, cls)
    for u in range(len(cu) - 1):
        assert nt[u] == len(toks[u])
        assert tok[cu[u]:cu[u] + nt[u]].tolist() == toks[u]


@pytest.mark.parametrize("case", json.load(open(GOLDEN))["cases"], ids=lambda c: c["name"])
def test_golden_cases(case, cuda_device):
    logits = torch.tensor(case["logits"], dtype=torch.float32).to(torch.bfloat16)
    fc, tok, nt = _decode(logits, case["cu"], cuda_device)
    assert fc.tolist() == case["classes"]
    cu = case["cu"]
    assert [tok[cu[u]:cu[u] + nt[u]].tolist() for u in range(len(cu) - 1)] == case["tokens"]


@pytest.mark.parametrize("n_classes,pad", [(2, 0), (3, 1), (7, 0), (8, 5), (100, 0), (1000, 3), (4099, 8)])
def test_random_shapes_and_strides(n_classes, pad, cuda_device):
    lengths = [37, 0, 1, 200, 5, 64]
    cu = wl.cu_seqlens(lengths)
    # the row stride (n_classes + pad) puts rows at every 2-byte offset
    logits = wl.ctc_logits(lengths, n_classes=n_classes, seed=n_classes + pad, row_stride=n_classes + pad)
    _check(logits, cu, cuda_device, n_classes=n_classes)


def test_full_class_count_mid_batch(cuda_device):
    lengths = wl.draw_lengths(4)[:6]
    cu = wl.cu_seqlens(lengths)
    logits = wl.ctc_logits(lengths, seed=44)
    _check(logits, cu, cuda_device)


def test_last_row_ends_off_a_16_byte_boundary(cuda_device):
    # 3 classes, stride 3: rows of 6 bytes, the tensor ends 2 bytes past a
    # 16-byte boundary; the guard rows past it must not be read into any frame
    lengths = [11]
    logits = wl.ctc_logits(lengths, n_classes=3, seed=5)
    _check(logits, wl.cu_seqlens(lengths), cuda_device)


def test_full_size_sampled(cuda_device):
    """The batch-128 workload at full size (58,903 frames x 100,353 classes,
    11.8 GB of bf16 logits generated on the device): per-frame classes of
    sampled frames against the oracle on those rows."""
    nle = _nle()
    lengths = wl.draw_lengths(4)
    cu = torch.from_numpy(wl.cu_seqlens(lengths)).to(cuda_device)
    logits = wl.ctc_logits(lengths, seed=4004, device=cuda_device)
    fc, tok, nt = nle.ctc_greedy(logits, cu)
    torch.cuda.synchronize()
    rng = np.random.default_rng(9)
    rows = np.unique(np.concatenate([rng.integers(0, logits.shape[0], 200), [0, logits.shape[0] - 1]]))
    sample = logits[torch.from_numpy(rows).to(cuda_device)].cpu()
    np.testing.assert_array_equal(fc.cpu().numpy()[rows], oracle.ctc_frame_classes(sample))
    # counts are bounded by the frames of each utterance
    assert np.all(nt.cpu().numpy() <= np.asarray(lengths))
    del logits
    torch.cuda.empty_cache()


def test_full_size_every_frame_and_token(cuda_device):
    """The batch-128 workload at full size (58,903 frames x 100,353 classes,
    11.8 GB of bf16 logits generated on the device): the class of every
    frame and the token stream of every utterance, bit for bit against the
    oracle (which reads the logits in slices of 2,048 frames copied to the
    host and decodes its own classes)."""
    nle = _nle()
    lengths = wl.draw_lengths(4)
    cu_h = wl.cu_seqlens(lengths)
    cu = torch.from_numpy(cu_h).to(cuda_device)
    logits = wl.ctc_logits(lengths, seed=4004, device=cuda_device)
    fc, tok, nt = nle.ctc_greedy(logits, cu)
    torch.cuda.synchronize()
    T = logits.shape[0]
    ref_cls = np.empty(T, np.int64)
    for a in range(0, T, 2048):
        ref_cls[a:a + 2048] = oracle.ctc_frame_classes(logits[a:a + 2048].cpu())
    del logits
    torch.cuda.empty_cache()
    np.testing.assert_array_equal(fc.cpu().numpy(), ref_cls)
    ref_tok = oracle.ctc_collapse(ref_cls, cu_h)
    tok, nt = tok.cpu().numpy(), nt.cpu().numpy()
    for u in range(len(lengths)):
        assert nt[u] == len(ref_tok[u])
        assert tok[cu_h[u]:cu_h[u] + nt[u]].tolist() == ref_tok[u]


def test_invalid_offsets_give_zero_tokens(cuda_device):
    lengths = [10, 10]
    logits = wl.ctc_logits(lengths, n_classes=9, seed=6)
    cu = np.array([0, 10, 25], np.int32)   # past total_frames
    fc, tok, nt = _decode(logits, cu, cuda_device)
    cls, toks = oracle.ctc_greedy(logits, [0, 10])
    assert nt[0] == len(toks[0]) and tok[:nt[0]].tolist() == toks[0]
    assert nt[1] == 0


@pytest.mark.parametrize("n_classes,pad", [(1000, 3), (100353, 0), (13, 1)])
def test_nonfinite_signed_zero_and_ties(n_classes, pad, cuda_device):
    """Rows built to hit every branch of the argmax: NaN-only and -inf-only
    rows, NaN mixed with -inf, infinities, -0 against +0, the maximum repeated
    in several chunks, at the first and last class (the loose elements
    before and after the row's 16-byte chunks), and rows of few distinct
    values (ties everywhere).  NaN logits are no candidates."""
    rng = np.random.default_rng(n_classes)
    C = n_classes
    rows = []
    nan, inf = np.float32(np.nan), np.float32(np.inf)

    def r(fill=None):
        return (np.full(C, fill, np.float32) if fill is not None
                else rng.standard_normal(C).astype(np.float32))

    rows.append(r(nan))
    rows.append(r(-inf))
    x = r(nan); x[C * 2 // 3] = -inf; rows.append(x)
    x = r(-inf); x[::5] = nan; x[C - 2:] = inf; rows.append(x)
    x = -np.abs(r()) - 1; x[C // 2] = -0.0; x[C // 3] = 0.0; rows.append(x)
    x = r(); x[5 % C] = nan; rows.append(x)
    x = r(); x[[C // 7, C // 2, C - 1]] = 9.0; rows.append(x)
    x = r(); x[0] = 9.0; rows.append(x)
    x = r(); x[C - 1] = 9.0; rows.append(x)
    x = r(); x[min(3, C - 1)] = 9.0; x[C - 1] = 9.0; rows.append(x)
    for _ in range(8):
        rows.append(rng.integers(-2, 3, C).astype(np.float32))
    vals = np.stack(rows)
    full = np.concatenate([vals, rng.standard_normal((len(rows), pad)).astype(np.float32)], axis=1)
    logits = torch.from_numpy(full).to(torch.bfloat16)   # all values exact in bf16
    cu = wl.cu_seqlens([len(rows)])
    _check(logits, cu, cuda_device, n_classes=C)
