"""Host-side argument checks of the full-utterance attention, CTC decoding
and pooling entry points: every rejection below happens before a device is
touched (no GPU needed), and the pooled-row count helper agrees with the
oracle's window count."""
import numpy as np
import pytest
import torch

import oracle
from chunked_block_self_b200 import nle


def _varlen(**kw):
    a = dict(q=16, k=16, v=16, out=16, cu=16, n_seq=1, total=400, heads=8, d=64, stream=None)
    a.update(kw)
    return nle._lib.nle_varlen_attn_fwd(a["q"], a["k"], a["v"], a["out"], a["cu"], a["n_seq"], a["total"],
                                        a["heads"], a["d"], a["stream"])


def test_varlen_attn_host_validation():
    assert _varlen(d=65) == nle.NLE_ERR_UNSUPPORTED
    assert _varlen(heads=0) == nle.NLE_ERR_INVALID_ARG
    assert _varlen(n_seq=-1) == nle.NLE_ERR_INVALID_ARG
    assert _varlen(total=-1) == nle.NLE_ERR_INVALID_ARG
    assert _varlen(total=2**31) == nle.NLE_ERR_UNSUPPORTED
    assert _varlen(q=None) == nle.NLE_ERR_INVALID_ARG
    assert _varlen(cu=None) == nle.NLE_ERR_INVALID_ARG
    assert _varlen(v=40) == nle.NLE_ERR_MISALIGNED
    assert _varlen(n_seq=0, q=None, k=None, v=None, out=None, cu=None) == nle.NLE_OK
    assert _varlen(total=0) == nle.NLE_OK


def test_varlen_attn_ex_validation():
    f = nle._lib.nle_varlen_attn_fwd_ex
    args = [16, 16, 16, 16, 16, 1, 400, 8, 64, 0.0]
    assert f(*args, 8 * 64 - 8, None, 0, 0, None) == nle.NLE_ERR_INVALID_ARG    # stride below the row
    assert f(*args, 8 * 64 + 4, None, 0, 0, None) == nle.NLE_ERR_MISALIGNED     # stride not 16-byte
    assert f(*args, 0, None, 0, -1, None) == nle.NLE_ERR_INVALID_ARG            # negative wait limit


def _ctc(**kw):
    a = dict(logits=16, stride=100353, C=100353, cu=16, n_seq=2, total=50, fc=16, tok=16, nt=16, stream=None)
    a.update(kw)
    return nle._lib.nle_ctc_greedy_fwd(a["logits"], a["stride"], a["C"], a["cu"], a["n_seq"], a["total"], a["fc"],
                                       a["tok"], a["nt"], a["stream"])


def test_ctc_host_validation():
    assert _ctc(C=0) == nle.NLE_ERR_INVALID_ARG
    assert _ctc(stride=100352) == nle.NLE_ERR_INVALID_ARG
    assert _ctc(n_seq=-1) == nle.NLE_ERR_INVALID_ARG
    assert _ctc(total=-1) == nle.NLE_ERR_INVALID_ARG
    assert _ctc(total=2**31) == nle.NLE_ERR_UNSUPPORTED
    assert _ctc(logits=None) == nle.NLE_ERR_INVALID_ARG
    assert _ctc(fc=None) == nle.NLE_ERR_INVALID_ARG
    assert _ctc(nt=None) == nle.NLE_ERR_INVALID_ARG
    assert _ctc(logits=18) == nle.NLE_ERR_MISALIGNED
    assert _ctc(n_seq=0, total=0, logits=None, cu=None, fc=None, tok=None, nt=None) == nle.NLE_OK


def _pool(**kw):
    a = dict(h=16, hs=1024, dim=1024, z=16, zs=256, C=256, cu=16, n_seq=2, total=50, P=2, rows=26, out=16,
             w=None, status=None, stream=None)
    a.update(kw)
    return nle._lib.nle_posterior_pool_fwd(a["h"], a["hs"], a["dim"], a["z"], a["zs"], a["C"], a["cu"],
                                           a["n_seq"], a["total"], a["P"], a["rows"], a["out"], a["w"],
                                           a["status"], a["stream"])


def test_pool_host_validation():
    assert _pool(dim=12, hs=16) == nle.NLE_ERR_MISALIGNED
    assert _pool(hs=1028) == nle.NLE_ERR_MISALIGNED
    assert _pool(hs=1016) == nle.NLE_ERR_INVALID_ARG
    assert _pool(zs=255) == nle.NLE_ERR_INVALID_ARG
    assert _pool(C=0) == nle.NLE_ERR_INVALID_ARG
    assert _pool(P=0) == nle.NLE_ERR_INVALID_ARG
    assert _pool(P=5000) == nle.NLE_ERR_UNSUPPORTED
    assert _pool(rows=-1) == nle.NLE_ERR_INVALID_ARG
    assert _pool(total=2**31) == nle.NLE_ERR_UNSUPPORTED
    assert _pool(h=None) == nle.NLE_ERR_INVALID_ARG
    assert _pool(out=None) == nle.NLE_ERR_INVALID_ARG
    assert _pool(h=24) == nle.NLE_ERR_MISALIGNED
    assert _pool(z=17) == nle.NLE_ERR_MISALIGNED
    assert _pool(rows=0, h=None, z=None, cu=None, out=None) == nle.NLE_OK


@pytest.mark.parametrize("P", [1, 2, 3, 4, 15])
def test_pooled_rows_matches_oracle(P):
    rng = np.random.default_rng(P)
    lens = rng.integers(0, 900, 37)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    assert nle.pooled_rows(cu, P) == int(oracle.pooled_rows(cu, P)[-1])
    assert nle.pooled_rows(np.array([0, 422], np.int32), 2) == 211


def test_bindings_reject_cpu_tensors():
    x = torch.zeros(4, 1, 64, dtype=torch.bfloat16)
    cu = torch.tensor([0, 4], dtype=torch.int32)
    with pytest.raises(TypeError):
        nle.nle_varlen_attn_fwd(x, x, x, x, cu)
    z = torch.zeros(4, 8, dtype=torch.bfloat16)
    i = torch.zeros(4, dtype=torch.int32)
    with pytest.raises(TypeError):
        nle.nle_ctc_greedy_fwd(z, cu, i, i, i[:1])
    with pytest.raises(TypeError):
        nle.nle_posterior_pool_fwd(z, z, cu, z)
