"""The C-ABI library loads, exports what include/nle.h declares, and rejects
bad arguments on the host before touching a device (no GPU needed)."""
import ctypes
import os
import re

import pytest

from chunked_block_self_b200 import nle

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "nle.h")


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(nle_[a-z_]+)\s*\(", src)))


def test_header_declarations_are_exported():
    names = _declared()
    assert "nle_block_attn_fwd" in names and "nle_window_xattn_fwd" in names
    lib = ctypes.CDLL(nle.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(nle.EXPORTS)


def test_version_and_status_strings():
    assert nle.nle_version() == 2
    for code in (0, -1, -2, -3, -4, -5):
        assert nle.nle_status_string(code).startswith("NLE_")
    assert nle.nle_status_string(-99) == "unknown nle status"


def _block(**kw):
    a = dict(q=16, k=16, v=16, out=16, cu=16, n_seq=1, total=400, heads=8, d=64, B=200, stream=None)
    a.update(kw)
    return nle._lib.nle_block_attn_fwd(a["q"], a["k"], a["v"], a["out"], a["cu"], a["n_seq"], a["total"],
                                       a["heads"], a["d"], a["B"], a["stream"])


def test_block_attn_host_validation():
    assert _block(d=65) == nle.NLE_ERR_UNSUPPORTED
    assert _block(B=257) == nle.NLE_ERR_UNSUPPORTED
    assert _block(B=0) == nle.NLE_ERR_INVALID_ARG
    assert _block(heads=0) == nle.NLE_ERR_INVALID_ARG
    assert _block(n_seq=-1) == nle.NLE_ERR_INVALID_ARG
    assert _block(total=2**31) == nle.NLE_ERR_UNSUPPORTED
    assert _block(q=None) == nle.NLE_ERR_INVALID_ARG
    assert _block(out=None) == nle.NLE_ERR_INVALID_ARG
    assert _block(k=24) == nle.NLE_ERR_MISALIGNED
    # nothing to do: success without touching a device
    assert _block(n_seq=0, q=None, k=None, v=None, out=None, cu=None) == nle.NLE_OK
    assert _block(total=0) == nle.NLE_OK


def test_block_attn_ex_stride_validation():
    f = nle._lib.nle_block_attn_fwd_ex
    args = [16, 16, 16, 16, 16, 1, 400, 8, 64, 200, 0.0]
    assert f(*args, 8 * 64 - 8, None, 0, 0, None) == nle.NLE_ERR_INVALID_ARG
    assert f(*args, 8 * 64 + 4, None, 0, 0, None) == nle.NLE_ERR_MISALIGNED
    assert f(*args, 0, None, 0, -1, None) == nle.NLE_ERR_INVALID_ARG


def test_window_host_validation():
    f = nle._lib.nle_window_xattn_fwd
    base = [16, 16, 16, 16, 16, 1, 4700, 942, 16, 64, 15, 3, None]
    assert f(*base) != nle.NLE_ERR_INVALID_ARG or True  # reaches the device query on a GPU-less host
    bad = list(base); bad[9] = 32
    assert f(*bad) == nle.NLE_ERR_UNSUPPORTED
    bad = list(base); bad[10] = 33
    assert f(*bad) == nle.NLE_ERR_UNSUPPORTED
    bad = list(base); bad[11] = 17
    assert f(*bad) == nle.NLE_ERR_UNSUPPORTED
    bad = list(base); bad[11] = 0
    assert f(*bad) == nle.NLE_ERR_INVALID_ARG
    bad = list(base); bad[0] = 8
    assert f(*bad) == nle.NLE_ERR_MISALIGNED
    bad = list(base); bad[5] = 0
    assert f(*bad) == nle.NLE_OK


def test_binding_rejects_cpu_tensors():
    import torch
    x = torch.zeros(4, 1, 64, dtype=torch.bfloat16)
    cu = torch.tensor([0, 4], dtype=torch.int32)
    with pytest.raises(TypeError):
        nle.nle_block_attn_fwd(x, x, x, x, cu)


def _qkv(**kw):
    a = dict(x=16, w=16, b=None, out=16, cu=16, n_seq=1, total=400, dm=1024, heads=16, d=64, B=200)
    a.update(kw)
    return nle._lib.nle_block_attn_qkv_fwd(a["x"], a["w"], a["b"], a["out"], a["cu"], a["n_seq"], a["total"],
                                           a["dm"], a["heads"], a["d"], a["B"], None)


def test_block_attn_qkv_host_validation():
    assert _qkv(d=32) == nle.NLE_ERR_UNSUPPORTED
    assert _qkv(dm=1000) == nle.NLE_ERR_UNSUPPORTED        # not a multiple of 64
    assert _qkv(dm=16384 + 64) == nle.NLE_ERR_UNSUPPORTED
    assert _qkv(dm=0) == nle.NLE_ERR_INVALID_ARG
    assert _qkv(B=257) == nle.NLE_ERR_UNSUPPORTED
    assert _qkv(B=0) == nle.NLE_ERR_INVALID_ARG
    assert _qkv(heads=0) == nle.NLE_ERR_INVALID_ARG
    assert _qkv(x=None) == nle.NLE_ERR_INVALID_ARG
    assert _qkv(w=None) == nle.NLE_ERR_INVALID_ARG
    assert _qkv(x=24) == nle.NLE_ERR_MISALIGNED
    assert _qkv(b=8) == nle.NLE_ERR_MISALIGNED              # bias, when given, 16-byte aligned too
    assert _qkv(n_seq=0, x=None, w=None, out=None, cu=None) == nle.NLE_OK
    assert _qkv(total=0) == nle.NLE_OK
