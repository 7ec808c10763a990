"""GPU parity of the block self-attention kernel against the fp64 oracle.

Tolerance (bf16 inputs, fp32 accumulation and softmax, bf16 P and O):
relative L2 error <= 5e-3 and max-abs error <= 2e-2 against the fp64
oracle on the same bf16 input bits.  Integer work (the block plan) and the
properties that hold exactly (block locality, a one-frame block copying V)
are compared bit for bit.
"""
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


def _dev(x, dev):
    return {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in x.items()}


def _run(x, dev, B=200, **kw):
    nle = _nle()
    q, k, v = (x[n].to(dev) for n in ("q", "k", "v"))
    cu = torch.from_numpy(x["cu"]).to(dev)
    out = torch.full_like(q, float("nan"))
    if kw:
        nle.nle_block_attn_fwd_ex(q, k, v, out, cu, block_frames=B, **kw)
    else:
        nle.nle_block_attn_fwd(q, k, v, out, cu, block_frames=B)
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


@pytest.mark.parametrize("cfg", [1, 2])
def test_config_full_parity(cfg, cuda_device):
    x = wl.block_inputs(cfg)
    out = _run(x, cuda_device)
    ref = oracle.block_attn(x["q"], x["k"], x["v"], x["cu"], block_frames=200)
    _compare(out, ref)


@pytest.mark.parametrize("lengths", [
    [1], [127], [128], [129], [199], [200], [201], [255], [256], [257], [400],
    [0, 5, 0, 333, 1, 0], [200, 200, 1, 399, 17, 1000, 3],
])
def test_ragged_full_parity(lengths, cuda_device):
    x = wl.block_inputs(lengths=lengths, heads=3, seed=sum(lengths) + len(lengths))
    out = _run(x, cuda_device)
    ref = oracle.block_attn(x["q"], x["k"], x["v"], x["cu"], block_frames=200)
    _compare(out, ref)


@pytest.mark.parametrize("B", [1, 16, 17, 64, 100, 128, 129, 192, 208, 256])
def test_block_frames_variants(B, cuda_device):
    x = wl.block_inputs(lengths=[3 * B + 5, B, 2], heads=2, seed=B)
    out = _run(x, cuda_device, B=B)
    ref = oracle.block_attn(x["q"], x["k"], x["v"], x["cu"], block_frames=B)
    _compare(out, ref)


def test_mid_size_ragged_batch_full(cuda_device):
    lens = wl.draw_lengths(4)[:24]
    x = wl.block_inputs(lengths=lens, heads=16, seed=404)
    out = _run(x, cuda_device)
    ref = oracle.block_attn(x["q"], x["k"], x["v"], x["cu"], block_frames=200)
    _compare(out, ref)


def _sampled(x, out, n, seed):
    """Compare n sampled (frame, head) outputs, biased to block edges."""
    rng = np.random.default_rng(seed)
    total, heads = x["total"], x["heads"]
    seq, j, start, ln = oracle.block_table(x["cu"], 200)
    edges = np.concatenate([start, start + ln - 1])
    rows = np.concatenate([rng.integers(0, total, n), rng.choice(edges, min(n, len(edges)))])
    hs = rng.integers(0, heads, len(rows))
    ref = oracle.block_attn_rows(x["q"], x["k"], x["v"], x["cu"], rows, hs, block_frames=200)
    got = out[torch.from_numpy(rows).to(out.device), torch.from_numpy(hs).to(out.device)]
    return _compare(got, ref)


@pytest.mark.parametrize("cfg", [3, 4])
def test_config_full_size_sampled(cfg, cuda_device):
    x = wl.block_inputs(cfg)
    out = _run(x, cuda_device)
    _sampled(x, out, 3000, cfg)
    assert torch.isfinite(out.float()).all()


def _per_item_rel_l2(got, ref, cu, B):
    """Largest relative L2 error of any single (block, head) item."""
    seq, j, start, ln = oracle.block_table(cu, B)
    g = got.float().cpu().double().numpy()
    worst = 0.0
    for s0, n in zip(start.tolist(), ln.tolist()):
        e = np.linalg.norm(g[s0:s0 + n] - ref[s0:s0 + n], axis=(0, 2))
        r = np.maximum(np.linalg.norm(ref[s0:s0 + n], axis=(0, 2)), 1e-30)
        worst = max(worst, float((e / r).max()))
    return worst


@pytest.mark.parametrize("cfg", [3, 4])
def test_config_full_size_every_output(cfg, cuda_device):
    """Configs 3 (16 long utterances) and 4 (batch of 128) at full size:
    every output of the launch against the oracle, as one tensor within the
    tolerance, and item by item (every (block, head) within twice it), so a
    single corrupted item among thousands cannot hide in the average."""
    x = wl.block_inputs(cfg)
    out = _run(x, cuda_device)
    ref = oracle.block_attn(x["q"], x["k"], x["v"], x["cu"], block_frames=200)
    _compare(out, ref)
    assert _per_item_rel_l2(out, ref, x["cu"], 200) <= 2 * REL_L2


def test_block_locality_bit_exact(cuda_device):
    x = wl.block_inputs(lengths=[530, 90], heads=4, seed=31)
    out = _run(x, cuda_device)
    y = {k: (v.clone() if isinstance(v, torch.Tensor) else v) for k, v in x.items()}
    for n in ("q", "k", "v"):  # everything outside block [200, 400) of utterance 0
        y[n][:200] = -3 * y[n][:200]
        y[n][400:] = y[n][400:] + 1
    y["k"][400:402] = float("inf")
    y["v"][400:402] = float("nan")
    y["v"][150:200] = float("inf")
    out2 = _run(y, cuda_device)
    assert torch.equal(out2[200:400], out[200:400])
    assert not torch.equal(out2[:200], out[:200])


def test_partial_block_ignores_nonfinite_neighbours(cuda_device):
    # utterance of 250 frames: its second block is [200, 250); the next
    # utterance starts at 250 and holds NaN/Inf values
    x = wl.block_inputs(lengths=[250, 60], heads=2, seed=32)
    ref = oracle.block_attn(x["q"], x["k"], x["v"], x["cu"])
    for n in ("k", "v"):
        x[n][250:] = float("nan")
    x["q"][250:] = float("inf")
    out = _run(x, cuda_device)
    _compare(out[:250], ref[:250])


def test_single_frame_block_copies_v(cuda_device):
    x = wl.block_inputs(lengths=[201, 1], heads=4, seed=33)
    out = _run(x, cuda_device)
    assert torch.equal(out[200].cpu(), x["v"][200])
    assert torch.equal(out[201].cpu(), x["v"][201])


def test_empty_batch_is_noop(cuda_device):
    nle = _nle()
    q = torch.zeros(4, 2, 64, dtype=torch.bfloat16, device=cuda_device)
    out = torch.full_like(q, 7.0)
    cu = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    nle.nle_block_attn_fwd(q, q, q, out, cu, n_seq=0, total_frames=0)
    cu2 = torch.zeros(3, dtype=torch.int32, device=cuda_device)   # two empty utterances
    nle.nle_block_attn_fwd(q, q, q, out, cu2, total_frames=0)
    torch.cuda.synchronize()
    assert (out == 7.0).all()


def test_fused_qkv_stride_and_scale(cuda_device):
    nle = _nle()
    x = wl.block_inputs(lengths=[333, 45], heads=4, seed=34)
    T = x["total"]
    buf = torch.stack([x["q"], x["k"], x["v"]], 1).to(cuda_device)      # [T, 3, H, 64]
    cu = torch.from_numpy(x["cu"]).to(cuda_device)
    out = torch.empty(T, 4, 64, dtype=torch.bfloat16, device=cuda_device)
    nle.nle_block_attn_fwd_ex(buf[:, 0], buf[:, 1], buf[:, 2], out, cu, total_frames=T, heads=4,
                              softmax_scale=0.3, row_stride_qkv=3 * 4 * 64)
    torch.cuda.synchronize()
    ref = oracle.block_attn(x["q"], x["k"], x["v"], x["cu"], scale=0.3)
    _compare(out, ref)


def test_output_guard_rows_untouched(cuda_device):
    nle = _nle()
    x = wl.block_inputs(lengths=[210, 7], heads=2, seed=35)
    T = x["total"]
    q, k, v = (x[n].to(cuda_device) for n in ("q", "k", "v"))
    big = torch.full((T + 16, 2, 64), 123.0, dtype=torch.bfloat16, device=cuda_device)
    out = big[8:8 + T]
    nle.nle_block_attn_fwd(q, k, v, out, torch.from_numpy(x["cu"]).to(cuda_device))
    torch.cuda.synchronize()
    assert (big[:8] == 123.0).all() and (big[8 + T:] == 123.0).all()


def test_non_default_stream(cuda_device):
    nle = _nle()
    x = wl.block_inputs(lengths=[450], heads=2, seed=36)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        q, k, v = (x[n].to(cuda_device) for n in ("q", "k", "v"))
        cu = torch.from_numpy(x["cu"]).to(cuda_device)
        out = nle.block_attn(q, k, v, cu)
    s.synchronize()
    _compare(out, oracle.block_attn(x["q"], x["k"], x["v"], x["cu"]))


def test_device_plan_bit_exact(cuda_device):
    nle = _nle()
    rng = np.random.default_rng(5)
    cases = [wl.draw_lengths(c) for c in (1, 2, 3, 4, 5)] + [rng.integers(0, 900, 70), [0], [1, 0, 0, 2]]
    for lens in cases:
        cu = wl.cu_seqlens(lens)
        total = int(cu[-1])
        for B in (200, 15, 1):
            (seq, j, st, ln), count = nle.nle_block_plan_dev(torch.from_numpy(cu).to(cuda_device), total, B)
            torch.cuda.synchronize()
            ref = oracle.block_table(cu, B)
            n = len(ref[0])
            assert int(count.item()) == n
            for a, b in zip((seq, j, st, ln), ref):
                np.testing.assert_array_equal(a[:n].cpu().numpy(), b)


def test_invalid_offsets_reported_without_stray_writes(cuda_device):
    nle = _nle()
    x = wl.block_inputs(lengths=[100, 100], heads=2, seed=37)
    q, k, v = (x[n].to(cuda_device) for n in ("q", "k", "v"))
    big = torch.full((200 + 16, 2, 64), 55.0, dtype=torch.bfloat16, device=cuda_device)
    out = big[8:208]
    status = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    bad_cu = torch.tensor([0, 100, 400], dtype=torch.int32, device=cuda_device)   # beyond total
    nle.nle_block_attn_fwd_ex(q, k, v, out, bad_cu, total_frames=200, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == nle.NLE_ERR_INVALID_ARG
    assert (big[:8] == 55.0).all() and (big[208:] == 55.0).all()
    ref = oracle.block_attn(x["q"][:100], x["k"][:100], x["v"][:100], np.array([0, 100], np.int32))
    _compare(out[:100], ref)          # the valid utterance is still computed
    assert (out[100:] == 55.0).all()  # the invalid one is skipped


def test_timeout_path_reports_and_recovers(cuda_device):
    """The test hook withholds the first load: every bounded wait expires, the
    kernel reports NLE_ERR_TIMEOUT and the context stays usable."""
    nle = _nle()
    x = wl.block_inputs(lengths=[400, 300], heads=2, seed=38)
    q, k, v = (x[n].to(cuda_device) for n in ("q", "k", "v"))
    cu = torch.from_numpy(x["cu"]).to(cuda_device)
    out = torch.zeros_like(q)
    status = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    nle.nle_block_attn_fwd_ex(q, k, v, out, cu, dev_status=status,
                              flags=nle.NLE_FLAG_TEST_SKIP_FIRST_LOAD, wait_limit_ns=2_000_000)
    torch.cuda.synchronize()
    assert int(status.item()) == nle.NLE_ERR_TIMEOUT
    out2 = _run(x, cuda_device)
    _compare(out2, oracle.block_attn(x["q"], x["k"], x["v"], x["cu"]))


@pytest.mark.parametrize("B,lengths", [(200, [200, 137]), (128, [128, 90]), (256, [250]), (64, [64, 40])])
def test_running_max_rescale(B, lengths, cuda_device):
    """Keys late in the row dominate, so the softmax's running maximum jumps by
    more than its slack after earlier columns were written and the P already
    written is rescaled (by an exact power of two)."""
    x = wl.block_inputs(lengths=lengths, heads=2, seed=B + 1)
    k = x["k"].float()
    for a in np.cumsum([0] + lengths[:-1]):
        hi = min(B, lengths[0]) - 4
        k[a + hi - 3:a + hi] *= 12.0
    x["k"] = k.to(torch.bfloat16)
    out = _run(x, cuda_device, B=B)
    _compare(out, oracle.block_attn(x["q"], x["k"], x["v"], x["cu"], block_frames=B))


def test_concurrent_launches_on_two_streams(cuda_device):
    """Two launches running at once on different streams (and a third
    queued behind one of them) must each compute every item exactly once."""
    nle = _nle()
    xs = [wl.block_inputs(lengths=wl.draw_lengths(4)[i * 20:(i + 1) * 20], heads=16, seed=70 + i)
          for i in range(3)]
    dev = [{n: x[n].to(cuda_device) for n in ("q", "k", "v")} for x in xs]
    cus = [torch.from_numpy(x["cu"]).to(cuda_device) for x in xs]
    outs = [torch.full_like(d["q"], float("nan")) for d in dev]
    streams = [torch.cuda.Stream(device=cuda_device) for _ in range(2)]
    torch.cuda.synchronize()
    for i, st in ((0, streams[0]), (1, streams[1]), (2, streams[0])):
        with torch.cuda.stream(st):
            nle.nle_block_attn_fwd(dev[i]["q"], dev[i]["k"], dev[i]["v"], outs[i], cus[i], block_frames=200)
    torch.cuda.synchronize()
    for x, out in zip(xs, outs):
        _compare(out, oracle.block_attn(x["q"], x["k"], x["v"], x["cu"], block_frames=200))


@pytest.mark.parametrize("B,lengths,heads", [
    (200, [400], 8),                          # config 1's shape: split by default
    (200, [800], 16),                         # config 2's shape
    (200, [201, 200, 199, 128, 129, 1, 0, 55, 350], 4),
    (129, [129, 130, 258, 400, 7], 3),
    (256, [256, 512, 300, 129, 128, 1000], 4),
    (200, list(wl.draw_lengths(4)[:20]), 16),  # whole items by default (320+ items)
])
def test_work_split_bit_equal(B, lengths, heads, cuda_device):
    """Row tiles as separate work items (split) and whole (block, head) items
    compute the same numbers bit for bit: each row tile's S, softmax, PV and
    output are the same instructions on the same data, only the CTA and
    chain that run them change.  Both are also within tolerance of the
    oracle."""
    nle = _nle()
    x = wl.block_inputs(lengths=lengths, heads=heads, seed=B + len(lengths))
    q, k, v = (x[n].to(cuda_device) for n in ("q", "k", "v"))
    cu = torch.from_numpy(x["cu"]).to(cuda_device)
    outs = {}
    for name, flags in (("whole", nle.NLE_FLAG_WHOLE_ITEMS), ("split", nle.NLE_FLAG_SPLIT_ITEMS), ("auto", 0)):
        out = torch.full_like(q, float("nan"))
        status = torch.zeros(1, dtype=torch.int32, device=cuda_device)
        nle.nle_block_attn_fwd_ex(q, k, v, out, cu, block_frames=B, dev_status=status, flags=flags)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        outs[name] = out
    assert torch.equal(outs["split"], outs["whole"])
    assert torch.equal(outs["auto"], outs["whole"])
    _compare(outs["split"], oracle.block_attn(x["q"], x["k"], x["v"], x["cu"], B))
