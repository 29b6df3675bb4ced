"""The C-ABI library on the CPU host: it builds, loads, exports every entry
point the header declares, and its host-side checks reject bad arguments
before touching the device (no call here reaches a kernel launch)."""
import ctypes
import os
import re

import pytest

import deformable_convolution_sampling_dcn_b200 as dcn
from deformable_convolution_sampling_dcn_b200 import _binding as B
from deformable_convolution_sampling_dcn_b200 import build as build_mod

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "dcn_b200.h")


@pytest.fixture(scope="module")
def lib():
    build_mod.build()
    return B.lib()


def header_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s*([a-z_][a-z0-9_]*)\s*\(", text, flags=re.M)
    return sorted(set(n for n in names if not n.startswith("DCN")))


def test_header_lists_all_entry_points():
    assert set(header_functions()) == set(B.EXPORTS)


def test_library_exports_every_symbol(lib):
    for name in header_functions():
        assert hasattr(lib, name), name
        assert ctypes.cast(getattr(lib, name), ctypes.c_void_p).value


def test_abi_version_and_strings(lib):
    assert lib.dcn_abi_version() == B.ABI_VERSION
    for s in range(6):
        assert lib.dcn_status_string(s).decode().startswith("DCN_")
    assert lib.dcn_status_string(99) == b"unknown dcn_status"


def params(**kw):
    base = dict(B=2, H=40, W=40, G=16, C=32, kh=3, kw=3, stride_h=1, stride_w=1, pad_h=1, pad_w=1, dil_h=1,
                dil_w=1, offset_scale=1.0, mask_mode=0, dtype=1)
    base.update(kw)
    return B.DcnParams(**base)


def test_output_hw(lib):
    assert dcn.dcn_core_output_hw(params()) == (40, 40)
    assert dcn.dcn_core_output_hw(params(stride_h=2, stride_w=3)) == (20, 14)
    assert dcn.dcn_core_output_hw(params(pad_h=2, pad_w=2, dil_h=2, dil_w=2)) == (40, 40)
    assert dcn.dcn_core_output_hw(params(kh=5, kw=1, pad_h=0, pad_w=0)) == (36, 40)
    with pytest.raises(dcn.DcnError) as e:
        dcn.dcn_core_output_hw(params(H=1, pad_h=0))
    assert e.value.status == B.DCN_ERR_SHAPE


@pytest.mark.parametrize("kw,status", [
    (dict(C=12), B.DCN_ERR_UNSUPPORTED),           # 24-byte rows
    (dict(C=4), B.DCN_ERR_UNSUPPORTED),            # 8-byte rows in fp16
    (dict(C=256), B.DCN_ERR_UNSUPPORTED),          # 512-byte rows
    (dict(dtype=7), B.DCN_ERR_UNSUPPORTED),
    (dict(mask_mode=2), B.DCN_ERR_UNSUPPORTED),
    (dict(G=0), B.DCN_ERR_SHAPE),
    (dict(B=-1), B.DCN_ERR_SHAPE),
    (dict(stride_h=0), B.DCN_ERR_SHAPE),
    (dict(dil_w=0), B.DCN_ERR_SHAPE),
    (dict(pad_h=-1), B.DCN_ERR_SHAPE),
    (dict(offset_scale=float("nan")), B.DCN_ERR_SHAPE),
    (dict(kh=99), B.DCN_ERR_SHAPE),
])
def test_bad_params_rejected(lib, kw, status):
    p = params(**kw)
    # fake, never-dereferenced pointers: the checks fail before any CUDA call
    r = lib.dcn_core_forward(ctypes.byref(p), 16, 16, 16, 16, None)
    assert r == status, lib.dcn_last_error_detail()
    assert lib.dcn_last_error_detail()


def test_null_and_alignment_checks(lib):
    p = params()
    assert lib.dcn_core_forward(None, 16, 16, 16, 16, None) == B.DCN_ERR_NULL
    assert lib.dcn_core_forward(ctypes.byref(p), 0, 16, 16, 16, None) == B.DCN_ERR_NULL
    assert lib.dcn_core_forward(ctypes.byref(p), 24, 16, 16, 16, None) == B.DCN_ERR_ALIGN
    assert lib.dcn_core_forward(ctypes.byref(p), 16, 18, 16, 16, None) == B.DCN_ERR_ALIGN  # fp16 pair: 4 B
    assert lib.dcn_core_forward(ctypes.byref(p), 16, 16, 17, 16, None) == B.DCN_ERR_ALIGN
    assert lib.dcn_core_backward(ctypes.byref(p), 16, 16, 16, 16, 0, 16, 16, None) == B.DCN_ERR_NULL
    assert lib.dcn_core_backward(ctypes.byref(p), 16, 16, 16, 16, 8, 16, 16, None) == B.DCN_ERR_ALIGN
    ps = params(mask_mode=1, kh=9, kw=9, pad_h=4, pad_w=4)
    assert lib.dcn_core_backward(ctypes.byref(ps), 16, 16, 16, 16, 16, 16, 16, None) == B.DCN_ERR_UNSUPPORTED


def test_empty_problem_is_noop(lib):
    p = params(B=0)
    assert lib.dcn_core_forward(ctypes.byref(p), None, None, None, None, None) == B.DCN_OK
    assert lib.dcn_core_backward(ctypes.byref(p), None, None, None, None, None, None, None, None) == B.DCN_OK
    a = B.DaggParams(0, 6, 4, 100, 900, 13, 8, 32, 0)
    assert lib.deform_agg_forward(ctypes.byref(a), None, None, None, None, None, None, None) == B.DCN_OK


def test_agg_checks(lib):
    a = B.DaggParams(1, 6, 4, 100, 900, 13, 8, 32, 0)
    assert lib.deform_agg_forward(ctypes.byref(a), 16, 16, 16, 16, 16, 0, None) == B.DCN_ERR_NULL
    assert lib.deform_agg_forward(ctypes.byref(a), 8, 16, 16, 16, 16, 16, None) == B.DCN_ERR_ALIGN
    assert lib.deform_agg_forward(ctypes.byref(a), 16, 16, 16, 4, 16, 16, None) == B.DCN_ERR_ALIGN
    bad = B.DaggParams(1, 6, 4, 100, 900, 13, 8, 6, 0)
    assert lib.deform_agg_forward(ctypes.byref(bad), 16, 16, 16, 16, 16, 16, None) == B.DCN_ERR_UNSUPPORTED
    bad = B.DaggParams(1, 0, 4, 100, 900, 13, 8, 32, 0)
    assert lib.deform_agg_forward(ctypes.byref(bad), 16, 16, 16, 16, 16, 16, None) == B.DCN_ERR_SHAPE
    assert lib.deform_agg_backward(ctypes.byref(a), 16, 16, 16, 16, 16, 16, 16, 12, 16, None) == B.DCN_ERR_ALIGN


def test_binding_refuses_cpu_tensors():
    import torch

    x = torch.zeros(1, 4, 4, 32)
    with pytest.raises(ValueError, match="CUDA"):
        dcn.dcn_core_forward(x, torch.zeros(1, 4, 4, 1, 9, 2), torch.zeros(1, 4, 4, 1, 9), group=1)


def test_shard_range():
    for total in (0, 1, 7, 8, 16):
        for world in (1, 2, 3, 8):
            parts = [dcn.shard_range(total, world, r) for r in range(world)]
            assert parts[0][0] == 0 and parts[-1][1] == total
            assert all(parts[i][1] == parts[i + 1][0] for i in range(world - 1))
            sizes = [hi - lo for lo, hi in parts]
            assert max(sizes) - min(sizes) <= 1


def test_roi_pool_checks(lib):
    p = B.DroiParams(2, 64, 64, 256, 10, 7, 7, 2, 0.0625, 0.1, 0)
    assert lib.deform_roi_pool_forward(ctypes.byref(p), 16, 16, 16, 0, None) == B.DCN_ERR_NULL
    assert lib.deform_roi_pool_forward(ctypes.byref(p), 8, 16, 16, 16, None) == B.DCN_ERR_ALIGN
    assert lib.deform_roi_pool_forward(ctypes.byref(p), 16, 16, 12, 16, None) == B.DCN_ERR_ALIGN
    bad = B.DroiParams(2, 64, 64, 6, 10, 7, 7, 2, 0.0625, 0.1, 1)  # 12-byte rows
    assert lib.deform_roi_pool_forward(ctypes.byref(bad), 16, 16, 16, 16, None) == B.DCN_ERR_UNSUPPORTED
    bad = B.DroiParams(2, 64, 64, 256, 10, 7, 7, 0, 0.0625, 0.1, 0)
    assert lib.deform_roi_pool_forward(ctypes.byref(bad), 16, 16, 16, 16, None) == B.DCN_ERR_SHAPE
    empty = B.DroiParams(2, 64, 64, 256, 0, 7, 7, 2, 0.0625, 0.1, 0)
    assert lib.deform_roi_pool_forward(ctypes.byref(empty), None, None, None, None, None) == B.DCN_OK


def test_proj_checks(lib):
    """dcn_core_forward_proj: unsupported configurations and bad pointers are
    refused on the host (fake, never-dereferenced pointers)."""
    p = params(G=16, C=32)  # fp16, G*C = 512
    f = lib.dcn_core_forward_proj
    assert f(ctypes.byref(p), 512, 16, 16, 16, 0, None, 16, None, 0, None) == B.DCN_ERR_NULL          # no weight
    assert f(ctypes.byref(p), 512, 16, 16, 16, 8, None, 16, None, 0, None) == B.DCN_ERR_ALIGN         # weight 8-byte
    assert f(ctypes.byref(p), 512, 16, 16, 16, 16, 3, 16, None, 0, None) == B.DCN_ERR_ALIGN           # odd bias
    assert f(ctypes.byref(p), 100, 16, 16, 16, 16, None, 16, None, 0, None) == B.DCN_ERR_UNSUPPORTED  # Cout % 8
    assert f(ctypes.byref(p), 520, 16, 16, 16, 16, None, 16, None, 0, None) == B.DCN_ERR_UNSUPPORTED  # Cout > 512
    assert f(ctypes.byref(p), 512, 16, 16, 16, 16, None, 16, None, -1, None) == B.DCN_ERR_SHAPE       # ws bytes < 0
    need = lib.dcn_core_forward_proj_workspace_bytes(ctypes.byref(p))
    assert need == 2 * 40 * 40 * 512 * 2
    assert f(ctypes.byref(p), 512, 16, 16, 16, 16, None, 16, 8, need, None) == B.DCN_ERR_ALIGN       # ws 8-byte
    for bad in (params(G=16, C=32, dtype=0),     # fp32
                params(G=3, C=32),               # G*C = 96
                params(G=32, C=32),              # G*C = 1024
                params(G=1, C=128),              # C > 64
                params(G=16, C=32, kh=7, kw=7, pad_h=3, pad_w=3)):  # 49 points
        assert f(ctypes.byref(bad), 64, 16, 16, 16, 16, None, 16, None, 0, None) == B.DCN_ERR_UNSUPPORTED
    empty = params(B=0, G=16, C=32)
    assert f(ctypes.byref(empty), 64, None, None, None, None, None, None, None, 0, None) == B.DCN_OK
    assert lib.dcn_core_forward_proj_workspace_bytes(ctypes.byref(params(H=0))) == -1


def test_selftest_limit_checked_on_host(lib):
    assert lib.dcn_selftest_bounded_wait(0, None) == B.DCN_ERR_SHAPE
    assert lib.dcn_selftest_bounded_wait(20_000_000, None) == B.DCN_ERR_SHAPE


def test_deform_conv_checks(lib):
    p = params(G=16, C=32)
    f = lib.dcn_deform_conv_forward
    assert f(ctypes.byref(p), 256, 16, 16, 16, 0, None, 16, None) == B.DCN_ERR_NULL
    assert f(ctypes.byref(p), 100, 16, 16, 16, 16, None, 16, None) == B.DCN_ERR_UNSUPPORTED
    assert f(ctypes.byref(params(G=16, C=32, dtype=0)), 64, 16, 16, 16, 16, None, 16, None) == B.DCN_ERR_UNSUPPORTED
    assert f(ctypes.byref(params(B=0, G=16, C=32)), 64, None, None, None, None, None, None, None) == B.DCN_OK
    # B*H*W = 2^31 input pixels (corner indices are 32-bit) while B*Ho*Wo = 2^29
    big = params(B=2048, H=1024, W=1024, G=16, C=32, stride_h=2, stride_w=2)
    assert f(ctypes.byref(big), 64, 16, 16, 16, 16, None, 16, None) == B.DCN_ERR_UNSUPPORTED
