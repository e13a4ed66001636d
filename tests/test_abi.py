"""The C ABI boundary without a GPU: the library loads, exports every symbol
include/relkl.h declares, and rejects bad arguments before any CUDA call."""
import ctypes
import os
import re

import pytest

from attention_relation_kl_b200 import _abi
from attention_relation_kl_b200._abi import relkl_desc

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _header_functions():
    src = open(os.path.join(ROOT, "include", "relkl.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(relkl_[a-z0-9_]+)\s*\(", src)))


def test_library_exports_every_declared_symbol():
    lib = _abi.lib()
    declared = _header_functions()
    assert declared, "no declarations parsed"
    assert sorted(_abi.EXPORTS) == declared
    for name in declared:
        assert hasattr(lib, name), name


def test_status_strings_and_workspace_size():
    lib = _abi.lib()
    for code in range(6):
        assert lib.relkl_status_string(code).startswith(b"RELKL_")
    assert lib.relkl_workspace_bytes() == 256


def _desc(B=1, H=2, N=256, d=128, dtype=_abi.RELKL_BF16, causal=1, scale=0.0):
    x = relkl_desc()
    x.B, x.H, x.N, x.d = B, H, N, d
    x.stride[0], x.stride[1], x.stride[2], x.stride[3] = H * N * d, N * d, d, 1
    x.dtype, x.causal, x.scale, x.reserved = dtype, causal, scale, 0
    return x


FAKE = 0x10000  # never dereferenced: every case below fails validation first


def _fwd(desc, xt=FAKE, xs=FAKE, kl=FAKE, st=FAKE, ws=FAKE, wsb=256):
    return _abi.lib().relkl_fwd(ctypes.byref(desc) if desc is not None else None,
                                xt, xs, kl, st, ws, wsb, None)


def test_path_selection():
    lib = _abi.lib()
    assert lib.relkl_path_for(ctypes.byref(_desc(d=128))) == 1
    assert lib.relkl_path_for(ctypes.byref(_desc(d=64))) == 1
    assert lib.relkl_path_for(ctypes.byref(_desc(d=96))) == 2
    assert lib.relkl_path_for(ctypes.byref(_desc(dtype=_abi.RELKL_FP32))) == 2
    assert lib.relkl_path_for(ctypes.byref(_desc(d=256))) == 0
    bad = _desc()
    bad.stride[3] = 2
    assert lib.relkl_path_for(ctypes.byref(bad)) == 0


@pytest.mark.parametrize("mutate", [
    lambda d: setattr(d, "dtype", 7),
    lambda d: setattr(d, "causal", 2),
    lambda d: setattr(d, "reserved", 1),
    lambda d: setattr(d, "scale", -1.0),
    lambda d: setattr(d, "scale", float("nan")),
    lambda d: setattr(d, "d", 0),
    lambda d: setattr(d, "N", -1),
    lambda d: d.stride.__setitem__(3, 2),
    lambda d: d.stride.__setitem__(1, -5),
])
def test_invalid_descriptors(mutate):
    d = _desc()
    mutate(d)
    assert _fwd(d) == _abi.RELKL_ERR_INVALID


def test_invalid_pointers_and_workspace():
    d = _desc()
    assert _fwd(None) == _abi.RELKL_ERR_INVALID
    assert _fwd(d, xt=None) == _abi.RELKL_ERR_INVALID
    assert _fwd(d, xs=FAKE + 1) == _abi.RELKL_ERR_INVALID        # misaligned bf16
    assert _fwd(d, kl=None) == _abi.RELKL_ERR_INVALID
    assert _fwd(d, st=FAKE + 4) == _abi.RELKL_ERR_INVALID        # stats must be 16-B aligned
    assert _fwd(d, ws=None) == _abi.RELKL_ERR_WORKSPACE
    assert _fwd(d, wsb=64) == _abi.RELKL_ERR_WORKSPACE
    assert _fwd(d, ws=FAKE + 16) == _abi.RELKL_ERR_WORKSPACE     # must be 256-B aligned
    assert _fwd(_desc(d=512)) == _abi.RELKL_ERR_UNSUPPORTED


def test_empty_problems_are_no_ops():
    # no unit or no row: nothing to do, nothing dereferenced, no CUDA call
    assert _fwd(_desc(N=0), xt=None, xs=None, kl=None, st=None, ws=None) == _abi.RELKL_OK
    assert _fwd(_desc(B=0), xt=None, xs=None, kl=None, st=None, ws=None) == _abi.RELKL_OK


def test_multi_relation_validation():
    lib = _abi.lib()
    P = ctypes.c_void_p * 3
    descs = (relkl_desc * 3)(_desc(H=4), _desc(H=2), _desc(H=2))
    ptrs = P(FAKE, FAKE, FAKE)
    assert lib.relkl_fwd_qkv(0, descs, ptrs, ptrs, ptrs, ptrs, FAKE, 256, None) == \
        _abi.RELKL_ERR_INVALID
    assert lib.relkl_fwd_qkv(4, descs, ptrs, ptrs, ptrs, ptrs, FAKE, 256, None) == \
        _abi.RELKL_ERR_INVALID
    mism = (relkl_desc * 2)(_desc(N=256), _desc(N=512))
    assert lib.relkl_fwd_qkv(2, mism, ptrs, ptrs, ptrs, ptrs, FAKE, 256, None) == \
        _abi.RELKL_ERR_INVALID
    assert lib.relkl_bwd_qkv(3, descs, ptrs, ptrs, ptrs, None, None, FAKE, 256, None) == \
        _abi.RELKL_ERR_INVALID


def test_wait_timeout_setting_roundtrip():
    lib = _abi.lib()
    old = lib.relkl_set_wait_timeout_ns(12345)
    assert lib.relkl_set_wait_timeout_ns(old) == 12345


def _rope(base=1e4, scale=0.25, offset=0.0, apply=1, reserved=0):
    return _abi.relkl_rope(base, scale, offset, apply, reserved)


def test_rope_bwd_validation():
    lib = _abi.lib()
    buf = ctypes.c_void_p(4096)   # never dereferenced: every case fails validation or is empty
    good = _rope()
    inv = _abi.RELKL_ERR_INVALID
    cases = [
        (1, 2, 8, 7, buf, good, _abi.RELKL_BF16, buf),          # odd d
        (1, 2, 8, 0, buf, good, _abi.RELKL_BF16, buf),          # d < 2
        (1, 2, 8, 514, buf, good, _abi.RELKL_BF16, buf),        # d > 512
        (-1, 2, 8, 64, buf, good, _abi.RELKL_BF16, buf),        # negative B
        (1, 2, 8, 64, buf, good, 7, buf),                       # unknown dtype
        (1, 2, 8, 64, None, good, _abi.RELKL_BF16, buf),        # null input with work
        (1, 2, 8, 64, buf, good, _abi.RELKL_BF16, None),        # null output with work
        (1, 2, 8, 64, buf, _rope(base=1.0), _abi.RELKL_BF16, buf),
        (1, 2, 8, 64, buf, _rope(base=float("nan")), _abi.RELKL_BF16, buf),
        (1, 2, 8, 64, buf, _rope(scale=float("inf")), _abi.RELKL_BF16, buf),
        (1, 2, 8, 64, buf, _rope(apply=2), _abi.RELKL_BF16, buf),
        (1, 2, 8, 64, buf, _rope(reserved=1), _abi.RELKL_BF16, buf),
        (1, 2, 8, 64, ctypes.c_void_p(4097), good, _abi.RELKL_FP32, buf),   # misaligned input
    ]
    for B, H, N, d, src, rope, dt, dst in cases:
        assert lib.relkl_rope_bwd(B, H, N, d, src, ctypes.byref(rope), dt, dst, None) == inv
    assert lib.relkl_rope_bwd(1, 2, 8, 64, buf, None, _abi.RELKL_BF16, buf, None) == inv
    # zero work: nothing to check, nothing enqueued
    assert lib.relkl_rope_bwd(0, 2, 8, 64, None, ctypes.byref(good), _abi.RELKL_BF16, None, None) == 0
    assert lib.relkl_rope_bwd(1, 0, 8, 64, None, ctypes.byref(good), _abi.RELKL_BF16, None, None) == 0


def test_weight_grad_validation():
    lib = _abi.lib()
    p = ctypes.c_void_p(4096)
    inv = _abi.RELKL_ERR_INVALID
    for rows, D, cols, h, dx, dw in [
        (0, 64, 64, p, p, p), (8, 0, 64, p, p, p), (8, 64, 0, p, p, p), (8, 60, 64, p, p, p),
        (8, 64, 12, p, p, p), (2 ** 31, 64, 64, p, p, p), (8, 64, 64, None, p, p),
        (8, 64, 64, p, None, p), (8, 64, 64, p, p, None), (8, 64, 64, ctypes.c_void_p(4104), p, p),
    ]:
        assert lib.relkl_weight_grad(rows, D, cols, h, dx, dw, p, 256, None) == inv
    # a missing workspace is refused after the shapes are accepted
    assert lib.relkl_weight_grad(8, 64, 64, p, p, p, None, 0, None) == _abi.RELKL_ERR_WORKSPACE


def test_binding_rejects_bad_outputs_before_the_call():
    """The binding checks caller-provided outputs (shape, dtype, contiguity,
    device) before handing raw pointers to the library, which writes B*H*N
    floats of kl and B*H*N*4 of stats through them."""
    import torch
    from attention_relation_kl_b200.ops import _check_out
    dev = torch.device("cpu")
    ok = torch.empty(2, 3, 5, dtype=torch.float32)
    _check_out(ok, (2, 3, 5), "kl", dev)
    for bad in (torch.empty(2, 3, 4), torch.empty(2, 3, 5, dtype=torch.float64),
                torch.empty(2, 5, 3).transpose(1, 2), torch.empty(2, 3, 5, device="meta")):
        with pytest.raises(ValueError):
            _check_out(bad, (2, 3, 5), "kl", dev)
    with pytest.raises(ValueError):
        _check_out(None, (2, 3, 5), "kl", dev)
