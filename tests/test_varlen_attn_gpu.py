"""GPU parity of the full-utterance attention kernel (nle_varlen_attn_fwd)
against the fp64 oracle (block attention with one block per utterance).

Tolerance as for the block kernel (bf16 inputs, fp32 accumulation and
softmax, bf16 P and O): relative L2 error <= 5e-3 and max-abs <= 2e-2.
Locality across utterances is compared bit for bit."""
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


def _run(x, dev, **kw):
    nle = _nle()
    q, k, v = (x[n].to(dev) for n in ("q", "k", "v"))
    cu = torch.from_numpy(x["cu"]).to(dev)
    out = torch.full_like(q, float("nan"))
    if kw:
        nle.nle_varlen_attn_fwd_ex(q, k, v, out, cu, **kw)
    else:
        nle.nle_varlen_attn_fwd(q, k, v, out, cu)
    torch.cuda.synchronize()
    return out


def _compare(got, ref):
    g = got.float().cpu().double().numpy()
    assert np.isfinite(g).all(), "non-finite output"
    err = g - ref
    rel = np.linalg.norm(err) / max(np.linalg.norm(ref), 1e-30)
    mx = np.abs(err).max() if err.size else 0.0
    assert rel <= REL_L2 and mx <= MAX_ABS, f"rel_l2={rel:.3e} max_abs={mx:.3e}"
    return rel, mx


@pytest.mark.parametrize("lengths", [
    [1], [15], [16], [17], [127], [128], [129], [255], [256], [257], [383], [384], [385],
    [0, 5, 0, 333, 1, 0], [600, 1, 129, 256, 40],
])
def test_ragged_full_parity(lengths, cuda_device):
    x = wl.block_inputs(lengths=lengths, heads=3, seed=sum(lengths) + 3 * len(lengths))
    out = _run(x, cuda_device)
    _compare(out, oracle.varlen_attn(x["q"], x["k"], x["v"], x["cu"]))


def test_long_utterances_full_parity(cuda_device):
    x = wl.block_inputs(lengths=[2011, 700, 3], heads=2, seed=91)
    out = _run(x, cuda_device)
    _compare(out, oracle.varlen_attn(x["q"], x["k"], x["v"], x["cu"]))


def test_long_clip_workload_sampled(cuda_device):
    """The long-clip workload (16 utterances of 1950-4700 frames, 16 heads)
    as full attention: sampled (frame, head) outputs against the oracle,
    biased to the first and last rows of each utterance."""
    x = wl.block_inputs(3)
    out = _run(x, cuda_device)
    assert torch.isfinite(out.float()).all()
    rng = np.random.default_rng(3)
    cu = x["cu"]
    edges = np.concatenate([cu[:-1], cu[1:] - 1, cu[:-1] + 255, cu[:-1] + 256])
    rows = np.concatenate([rng.integers(0, x["total"], 1500), edges])
    hs = rng.integers(0, x["heads"], len(rows))
    ref = oracle.varlen_attn_rows(x["q"], x["k"], x["v"], cu, rows, hs)
    got = out[torch.from_numpy(rows).to(out.device), torch.from_numpy(hs).to(out.device)]
    _compare(got, ref)


def test_long_clip_workload_every_output(cuda_device):
    """The long-clip workload (16 utterances of 1950-4700 frames, 16 heads)
    as full attention, every output against the oracle (about 0.76 TFLOP in
    fp64 on the host cores): as one tensor within the tolerance, and every
    (512-row query unit, head) within twice it."""
    x = wl.block_inputs(3)
    out = _run(x, cuda_device)
    ref = oracle.varlen_attn(x["q"], x["k"], x["v"], x["cu"])
    _compare(out, ref)
    g = out.float().cpu().double().numpy()
    cu = x["cu"]
    worst = 0.0
    for i in range(len(cu) - 1):
        for a in range(int(cu[i]), int(cu[i + 1]), 512):
            b = min(a + 512, int(cu[i + 1]))
            e = np.linalg.norm(g[a:b] - ref[a:b], axis=(0, 2))
            r = np.maximum(np.linalg.norm(ref[a:b], axis=(0, 2)), 1e-30)
            worst = max(worst, float((e / r).max()))
    assert worst <= 2 * REL_L2, f"worst unit rel_l2={worst:.3e}"


def test_utterance_locality_bit_exact(cuda_device):
    """Changing (and poisoning) every frame outside utterance 1 leaves its
    outputs bit for bit: keys past the utterance are masked by index and the
    V rows of its last partial key tile are zeroed before PV."""
    x = wl.block_inputs(lengths=[300, 450, 77], heads=4, seed=92)
    out = _run(x, cuda_device)
    y = {k: (v.clone() if isinstance(v, torch.Tensor) else v) for k, v in x.items()}
    for n in ("q", "k", "v"):
        y[n][:300] = -3 * y[n][:300]
        y[n][750:] = y[n][750:] + 1
    y["k"][750:752] = float("inf")
    y["v"][750:760] = float("nan")
    y["q"][750:] = float("inf")
    out2 = _run(y, cuda_device)
    assert torch.equal(out2[300:750], out[300:750])
    assert not torch.equal(out2[:300], out[:300])


@pytest.mark.parametrize("lengths,hot", [([900], [700, 701, 702]), ([520, 300], [515, 516]),
                                         ([140], [130, 131])])
def test_running_max_rescale_across_tiles(lengths, hot, cuda_device):
    """Keys in a late key tile dominate every row, so the running shift has
    to move after earlier tiles were summed into O: O, the row sum and the
    tile's P are rescaled by exact powers of two."""
    x = wl.block_inputs(lengths=lengths, heads=2, seed=93 + len(hot))
    k = x["k"].float()
    k[hot] *= 14.0
    x["k"] = k.to(torch.bfloat16)
    out = _run(x, cuda_device)
    _compare(out, oracle.varlen_attn(x["q"], x["k"], x["v"], x["cu"]))


def test_single_frame_copies_v(cuda_device):
    x = wl.block_inputs(lengths=[1, 2, 1], heads=4, seed=94)
    out = _run(x, cuda_device)
    assert torch.equal(out[0].cpu(), x["v"][0])
    assert torch.equal(out[3].cpu(), x["v"][3])


def test_empty_batch_is_noop(cuda_device):
    nle = _nle()
    q = torch.zeros(4, 2, 64, dtype=torch.bfloat16, device=cuda_device)
    out = torch.full_like(q, 7.0)
    cu2 = torch.zeros(3, dtype=torch.int32, device=cuda_device)   # two empty utterances
    nle.nle_varlen_attn_fwd(q, q, q, out, cu2, total_frames=0)
    cu3 = torch.tensor([0, 0, 4], dtype=torch.int32, device=cuda_device)
    nle.nle_varlen_attn_fwd(q, q, q, out, cu3)
    torch.cuda.synchronize()
    assert torch.isfinite(out.float()).all()


def test_strided_qkv_and_scale(cuda_device):
    nle = _nle()
    x = wl.block_inputs(lengths=[333, 45], heads=4, seed=95)
    T = x["total"]
    buf = torch.stack([x["q"], x["k"], x["v"]], 1).to(cuda_device)      # [T, 3, H, 64]
    cu = torch.from_numpy(x["cu"]).to(cuda_device)
    out = torch.empty(T, 4, 64, dtype=torch.bfloat16, device=cuda_device)
    nle.nle_varlen_attn_fwd_ex(buf[:, 0], buf[:, 1], buf[:, 2], out, cu, total_frames=T, heads=4,
                               softmax_scale=0.3, row_stride_qkv=3 * 4 * 64)
    torch.cuda.synchronize()
    _compare(out, oracle.varlen_attn(x["q"], x["k"], x["v"], x["cu"], scale=0.3))


def test_invalid_offsets_reported_without_stray_writes(cuda_device):
    nle = _nle()
    x = wl.block_inputs(lengths=[300, 100], heads=2, seed=96)
    q, k, v = (x[n].to(cuda_device) for n in ("q", "k", "v"))
    big = torch.full((400 + 16, 2, 64), 55.0, dtype=torch.bfloat16, device=cuda_device)
    out = big[8:408]
    status = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    bad_cu = torch.tensor([0, 300, 900], dtype=torch.int32, device=cuda_device)   # beyond total
    nle.nle_varlen_attn_fwd_ex(q, k, v, out, bad_cu, total_frames=400, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == nle.NLE_ERR_INVALID_ARG
    assert (big[:8] == 55.0).all() and (big[408:] == 55.0).all()
    ref = oracle.varlen_attn(x["q"][:300], x["k"][:300], x["v"][:300], np.array([0, 300], np.int32))
    _compare(out[:300], ref)          # the valid utterance is still computed
    assert (out[300:] == 55.0).all()  # the invalid one is skipped


def test_timeout_path_reports_and_recovers(cuda_device):
    """The test hook withholds the first Q load: the bounded waits expire,
    the kernel reports NLE_ERR_TIMEOUT and the context stays usable."""
    nle = _nle()
    x = wl.block_inputs(lengths=[600, 300], heads=2, seed=97)
    q, k, v = (x[n].to(cuda_device) for n in ("q", "k", "v"))
    cu = torch.from_numpy(x["cu"]).to(cuda_device)
    out = torch.zeros_like(q)
    status = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    nle.nle_varlen_attn_fwd_ex(q, k, v, out, cu, dev_status=status,
                               flags=nle.NLE_FLAG_TEST_SKIP_FIRST_LOAD, wait_limit_ns=2_000_000)
    torch.cuda.synchronize()
    assert int(status.item()) == nle.NLE_ERR_TIMEOUT
    out2 = _run(x, cuda_device)
    _compare(out2, oracle.varlen_attn(x["q"], x["k"], x["v"], x["cu"]))
