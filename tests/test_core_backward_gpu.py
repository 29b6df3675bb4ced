"""GPU parity of dcn_core_backward against the fp64 oracle."""
import pytest
import torch

import oracle
import synthetic_inputs as si
from parity import assert_close_bwd

pytestmark = pytest.mark.gpu


def run_bwd(shape: si.CoreShape, inp, dev):
    import deformable_convolution_sampling_dcn_b200 as d

    x, off, m, go = (inp[k].to(dev) for k in ("x", "offset", "mask", "grad_out"))
    cfg = dict(group=shape.G, kernel=(shape.kh, shape.kw), stride=(shape.stride_h, shape.stride_w),
               pad=(shape.pad_h, shape.pad_w), dil=(shape.dil_h, shape.dil_w), offset_scale=shape.offset_scale,
               softmax=shape.softmax)
    gx, goff, gm = d.dcn_core_backward(x, off, m, go, **cfg)
    torch.cuda.synchronize()
    ref = oracle.dcn_backward(inp["x"], inp["offset"], inp["mask"], inp["grad_out"], G=shape.G, kh=shape.kh,
                              kw=shape.kw, stride=(shape.stride_h, shape.stride_w), pad=(shape.pad_h, shape.pad_w),
                              dil=(shape.dil_h, shape.dil_w), offset_scale=shape.offset_scale,
                              softmax=shape.softmax)
    ref["budget"] = oracle.dcn_grad_x_budget(inp["offset"], inp["mask"], inp["grad_out"],
                                             x_shape=tuple(inp["x"].shape), G=shape.G, kh=shape.kh, kw=shape.kw,
                                             stride=(shape.stride_h, shape.stride_w),
                                             pad=(shape.pad_h, shape.pad_w), dil=(shape.dil_h, shape.dil_w),
                                             offset_scale=shape.offset_scale, softmax=shape.softmax)
    return (gx, goff, gm), ref


# dcn_core_backward takes the staged kernel for fp32 storage with 128-byte groups
# (C = 32) and K <= 9, and the generic one otherwise; "generic" forces the
# generic kernel everywhere.
ROUTES = ["auto", "generic"]


def _route(monkeypatch, route):
    if route == "generic":
        monkeypatch.setenv("DCN_B200_FORCE_GENERIC", "1")


def check_all(got, ref, tag):
    gx, goff, gm = got
    r = [assert_close_bwd(gx, ref["grad_x"], f"{tag} grad_x", budget=ref["budget"]),
         assert_close_bwd(goff, ref["grad_offset"], f"{tag} grad_offset", atomic=False),
         assert_close_bwd(gm, ref["grad_mask"], f"{tag} grad_mask", atomic=False)]
    print(f"{tag}: worst err/bound {max(r):.3f}")


@pytest.mark.parametrize("route", ROUTES)
def test_dcnv4_p4_backward_full_size(cuda_dev, route, monkeypatch):
    _route(monkeypatch, route)
    shape, inp = si.workload_core("dcnv4_p4_bwd")
    got, ref = run_bwd(shape, inp, cuda_dev)
    check_all(got, ref, f"dcnv4_p4_bwd {route}")


SMALL = [
    # B, H, W, G, C, kh, kw, stride, pad, dil, scale, softmax, dtype
    (1, 6, 6, 2, 4, 3, 3, 1, 1, 1, 1.0, False, "f32"),
    (2, 9, 7, 3, 8, 3, 3, 2, 1, 1, 0.5, True, "f32"),
    (1, 11, 13, 2, 32, 3, 3, 1, 2, 2, 1.0, False, "f32"),
    (1, 8, 10, 1, 64, 5, 3, 1, (2, 1), 1, 0.7, True, "f32"),
    (2, 12, 9, 2, 32, 3, 3, 1, 1, 1, 1.0, False, "f16"),
    (1, 10, 10, 4, 16, 3, 3, 1, 1, 1, 1.0, True, "f16"),
    (2, 12, 9, 2, 32, 3, 3, 1, 1, 1, 1.0, False, "bf16"),
    (1, 7, 14, 2, 64, 3, 3, 2, 1, 1, 1.0, True, "bf16"),
]


def _pair(v):
    return (v, v) if isinstance(v, int) else v


@pytest.mark.parametrize("route", ROUTES)
@pytest.mark.parametrize("case", range(len(SMALL)))
def test_small_backward(case, route, cuda_dev, monkeypatch):
    _route(monkeypatch, route)
    B, H, W, G, C, kh, kw, st, pd, dl, s, sm, dt = SMALL[case]
    st, pd, dl = _pair(st), _pair(pd), _pair(dl)
    shape = si.CoreShape(B=B, H=H, W=W, G=G, C=C, kh=kh, kw=kw, stride_h=st[0], stride_w=st[1], pad_h=pd[0],
                         pad_w=pd[1], dil_h=dl[0], dil_w=dl[1], offset_scale=s, softmax=sm, dtype=dt)
    inp = si.core_inputs(shape, 200 + case, offset_std=2.0, oob_fraction=0.03, with_grad_out=True)
    got, ref = run_bwd(shape, inp, cuda_dev)
    check_all(got, ref, f"small backward {case}")


def test_autograd_function(cuda_dev):
    """DCNCoreFunction routes torch.autograd to the library's backward."""
    import deformable_convolution_sampling_dcn_b200 as d

    shape = si.CoreShape(B=1, H=9, W=9, G=2, C=32, dtype="f32")
    inp = si.core_inputs(shape, 5, with_grad_out=True)
    x, off, m = (inp[k].to(cuda_dev).requires_grad_(True) for k in ("x", "offset", "mask"))
    out = d.DCNCoreFunction.apply(x, off, m, 2)
    (out * inp["grad_out"].to(cuda_dev)).sum().backward()
    ref = oracle.dcn_backward(inp["x"], inp["offset"], inp["mask"], inp["grad_out"], G=2)
    assert_close_bwd(x.grad, ref["grad_x"], "autograd grad_x")
    assert_close_bwd(off.grad, ref["grad_offset"], "autograd grad_offset", atomic=False)
    assert_close_bwd(m.grad, ref["grad_mask"], "autograd grad_mask", atomic=False)


@pytest.mark.parametrize("route", ROUTES)
def test_dcnv3_p3_softmax_bf16_backward_full_size(cuda_dev, route, monkeypatch):
    """The DCNv3 P3 backward that bench.py times (bf16, softmax over K, 5 % far
    taps, 7.4 M taps): at full size the grad_x atomics contend and the softmax
    Jacobian runs on every (pixel, group)."""
    _route(monkeypatch, route)
    shape, inp = si.workload_core("dcnv3_p3_bwd")
    got, ref = run_bwd(shape, inp, cuda_dev)
    check_all(got, ref, f"dcnv3_p3_bwd {route}")


# Offsets with a 12-pixel spread on 40-row maps put many taps inside the map
# but beyond the staged rows (a halo of 8), which the staged kernel reads from
# global memory; several segments per plane and the softmax mode (the fp32
# cases take the staged kernel, the 16-bit ones the generic kernel); 3 % of
# the taps fully outside the map.
FAR = [
    # B, H, W, G, C, softmax, dtype
    (2, 40, 40, 2, 32, False, "f32"),
    (1, 44, 37, 3, 32, True, "f32"),
    (2, 40, 40, 2, 32, False, "f16"),
    (1, 41, 30, 2, 32, True, "bf16"),
    (1, 36, 40, 2, 64, True, "f16"),
]


@pytest.mark.parametrize("case", range(len(FAR)))
def test_far_taps_backward(case, cuda_dev):
    B, H, W, G, C, sm, dt = FAR[case]
    shape = si.CoreShape(B=B, H=H, W=W, G=G, C=C, softmax=sm, dtype=dt)
    inp = si.core_inputs(shape, 700 + case, offset_std=12.0, oob_fraction=0.03, with_grad_out=True)
    got, ref = run_bwd(shape, inp, cuda_dev)
    check_all(got, ref, f"far taps backward {case}")


def test_backward_nan_offsets(cuda_dev):
    """A NaN offset makes that point's grad_offset and grad_mask NaN (the whole
    item's grad_mask in softmax mode) and adds nothing to grad_x."""
    for sm, dt in ((False, "f32"), (True, "bf16")):
        shape = si.CoreShape(B=1, H=20, W=24, G=2, C=32, softmax=sm, dtype=dt)
        inp = si.core_inputs(shape, 77, with_grad_out=True)
        off = inp["offset"].clone()
        off[0, 3, 5, 1, 4, 0] = float("nan")
        off[0, 17, 2, 0, 0, 1] = float("nan")
        inp["offset"] = off
        got, ref = run_bwd(shape, inp, cuda_dev)
        check_all(got, ref, f"nan offsets softmax={sm}")
