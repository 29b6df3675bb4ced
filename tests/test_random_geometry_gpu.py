"""Seeded sweep over random small geometries: the forward (staged where the
shape fits it, and the generic kernel), the backward and the fused
projection against the fp64 oracle, element by element.  Each case draws
kernel size, stride, padding, dilation, group count and width, storage
type, mask mode, offset scale and a fraction of far out-of-map taps."""
import numpy as np
import pytest
import torch

import oracle
import synthetic_inputs as si
from parity import assert_close_bwd, assert_close_fwd

pytestmark = pytest.mark.gpu

N_CASES = 24


def draw(i):
    r = np.random.default_rng(1000 + i)
    dt = ["f32", "f16", "bf16"][r.integers(3)]
    es = 4 if dt == "f32" else 2
    C = int(r.choice([c for c in (4, 8, 16, 32, 64, 128) if 16 <= c * es <= 256]))
    kh, kw = int(r.integers(1, 6)), int(r.integers(1, 6))
    sh, sw = int(r.integers(1, 3)), int(r.integers(1, 3))
    dh, dw = int(r.integers(1, 3)), int(r.integers(1, 3))
    ph, pw = int(r.integers(0, 3)), int(r.integers(0, 3))
    H = int(r.integers(max(1, dh * (kh - 1) + 1 - 2 * ph), 24))
    W = int(r.integers(max(1, dw * (kw - 1) + 1 - 2 * pw), 24))
    shape = si.CoreShape(B=int(r.integers(1, 3)), H=H, W=W, G=int(r.integers(1, 5)), C=C, kh=kh, kw=kw,
                         stride_h=sh, stride_w=sw, pad_h=ph, pad_w=pw, dil_h=dh, dil_w=dw,
                         offset_scale=float(r.choice([1.0, 0.5, 0.25])), softmax=bool(r.integers(2)), dtype=dt)
    kw_in = dict(offset_std=float(r.uniform(0.5, 4.0)), oob_fraction=float(r.choice([0.0, 0.1])))
    return shape, kw_in


def geo(shape):
    return dict(kernel=(shape.kh, shape.kw), stride=(shape.stride_h, shape.stride_w), pad=(shape.pad_h, shape.pad_w),
                dil=(shape.dil_h, shape.dil_w), offset_scale=shape.offset_scale, softmax=shape.softmax)


def ogeo(shape):
    g = geo(shape)
    return dict(kh=shape.kh, kw=shape.kw, stride=g["stride"], pad=g["pad"], dil=g["dil"],
                offset_scale=shape.offset_scale, softmax=shape.softmax)


@pytest.mark.parametrize("generic", [False, True])
@pytest.mark.parametrize("i", range(N_CASES))
def test_forward(i, generic, cuda_dev, monkeypatch):
    import deformable_convolution_sampling_dcn_b200 as d

    if generic:
        monkeypatch.setenv("DCN_B200_FORCE_GENERIC", "1")
    shape, kw_in = draw(i)
    inp = si.core_inputs(shape, 2000 + i, **kw_in)
    out = d.dcn_core_forward(*(inp[k].to(cuda_dev) for k in ("x", "offset", "mask")), group=shape.G, **geo(shape))
    torch.cuda.synchronize()
    assert d._binding.take_device_error() == 0
    ref = oracle.dcn_forward(inp["x"], inp["offset"], inp["mask"], G=shape.G, **ogeo(shape))
    assert_close_fwd(out, ref, f"random forward {i} {shape}")


@pytest.mark.parametrize("i", range(N_CASES))
def test_backward(i, cuda_dev):
    import deformable_convolution_sampling_dcn_b200 as d

    shape, kw_in = draw(i)
    if shape.softmax and shape.K > 49:
        pytest.skip("softmax backward keeps at most 49 per-point gradients")
    inp = si.core_inputs(shape, 3000 + i, with_grad_out=True, **kw_in)
    gx, goff, gm = d.dcn_core_backward(*(inp[k].to(cuda_dev) for k in ("x", "offset", "mask", "grad_out")),
                                       group=shape.G, **geo(shape))
    torch.cuda.synchronize()
    ref = oracle.dcn_backward(inp["x"], inp["offset"], inp["mask"], inp["grad_out"], G=shape.G, **ogeo(shape))
    budget = oracle.dcn_grad_x_budget(inp["offset"], inp["mask"], inp["grad_out"], x_shape=tuple(inp["x"].shape),
                                      G=shape.G, **ogeo(shape))
    assert_close_bwd(gx, ref["grad_x"], f"random grad_x {i}", budget=budget)
    assert_close_bwd(goff, ref["grad_offset"], f"random grad_offset {i}", atomic=False)
    assert_close_bwd(gm, ref["grad_mask"], f"random grad_mask {i}", atomic=False)


def draw_proj(i):
    r = np.random.default_rng(5000 + i)
    dt = ["f16", "bf16"][r.integers(2)]
    C = int(r.choice([8, 16, 32, 64]))
    G = int(r.choice([g for g in range(1, 65) if (g * C) % 64 == 0 and g * C <= 512]))
    kh = kw = int(r.choice([1, 3, 5]))
    s = int(r.integers(1, 3))
    p = kh // 2
    shape = si.CoreShape(B=int(r.integers(1, 4)), H=int(r.integers(3, 30)), W=int(r.integers(3, 30)), G=G, C=C,
                         kh=kh, kw=kw, stride_h=s, stride_w=s, pad_h=p, pad_w=p, softmax=bool(r.integers(2)),
                         dtype=dt)
    cout = 8 * int(r.integers(1, 65))
    return shape, cout


@pytest.mark.parametrize("i", range(12))
def test_projection(i, cuda_dev):
    import deformable_convolution_sampling_dcn_b200 as d

    shape, cout = draw_proj(i)
    inp = si.core_inputs(shape, 6000 + i)
    inp.update(si.proj_inputs(shape.G * shape.C, cout, shape.dtype, 7000 + i))
    t = {k: v.to(cuda_dev) for k, v in inp.items()}
    out = d.dcn_core_forward_proj(t["x"], t["offset"], t["mask"], t["weight"], t["bias"], group=shape.G,
                                  **geo(shape))
    torch.cuda.synchronize()
    assert d._binding.take_device_error() == 0
    core = oracle.dcn_forward(inp["x"], inp["offset"], inp["mask"], G=shape.G, **ogeo(shape))
    assert_close_fwd(out, oracle.pointwise_projection(core, inp["weight"], inp["bias"]), f"random proj {i}")


@pytest.mark.parametrize("i", range(12))
def test_deform_conv(i, cuda_dev):
    import deformable_convolution_sampling_dcn_b200 as d

    shape, cout = draw_proj(100 + i)
    inp = si.core_inputs(shape, 9000 + i)
    inp.update(si.deform_conv_weights(shape.K, shape.G * shape.C, cout, shape.dtype, 9500 + i))
    t = {k: v.to(cuda_dev) for k, v in inp.items()}
    out = d.dcn_deform_conv_forward(t["x"], t["offset"], t["mask"], t["weight"], t["bias"], group=shape.G,
                                    **geo(shape))
    torch.cuda.synchronize()
    assert d._binding.take_device_error() == 0
    ref = oracle.deform_conv_forward(inp["x"], inp["offset"], inp["mask"], inp["weight"], inp["bias"], G=shape.G,
                                     **ogeo(shape))
    assert_close_fwd(out, ref, f"random deform conv {i}")


def draw_roi(i):
    r = np.random.default_rng(8000 + i)
    dt = ["f32", "f16", "bf16"][r.integers(3)]
    es = 4 if dt == "f32" else 2
    C = int(r.choice([c for c in (4, 8, 16, 32, 64, 128, 256, 512) if (c * es) % 16 == 0]))
    return si.RoiShape(B=int(r.integers(1, 3)), H=int(r.integers(4, 40)), W=int(r.integers(4, 40)), C=C,
                       N=int(r.integers(1, 40)), PH=int(r.integers(1, 8)), PW=int(r.integers(1, 8)),
                       S=int(r.integers(1, 4)), spatial_scale=float(r.choice([1.0, 0.5, 0.25])),
                       gamma=float(r.choice([0.1, 0.3])), dtype=dt)


@pytest.mark.parametrize("i", range(12))
def test_roi_pool(i, cuda_dev):
    import deformable_convolution_sampling_dcn_b200 as d

    rs = draw_roi(i)
    inp = si.roi_inputs(rs, 9000 + i, min_size=2.0)
    kw = dict(pooled=(rs.PH, rs.PW), sampling=rs.S, spatial_scale=rs.spatial_scale, gamma=rs.gamma)
    out = d.deform_roi_pool_forward(*(inp[k].to(cuda_dev) for k in ("x", "rois", "offset")), **kw)
    torch.cuda.synchronize()
    assert_close_fwd(out, oracle.roi_pool_forward(inp["x"], inp["rois"], inp["offset"], **kw), f"random roi {i}")


def draw_agg(i):
    r = np.random.default_rng(11000 + i)
    dt = ["f32", "f16", "bf16"][r.integers(3)]
    es = 4 if dt == "f32" else 2
    C = int(r.choice([c for c in (4, 8, 16, 32, 64) if (c * es) % 16 == 0]))
    G = int(r.choice([1, 2, 4, 8, 16]))
    if i % 2 == 0:  # every other case takes a 512/1024/2048-byte row (the all-groups kernels)
        row = int(r.choice([512, 1024, 2048]))
        G = max(1, row // (C * es))
        C = row // (G * es)
    cams = int(r.integers(1, 7))
    scales = tuple((int(r.integers(1, 20)), int(r.integers(1, 30))) for _ in range(int(r.integers(1, 5))))
    shape = si.AggShape(B=int(r.integers(1, 3)), num_cams=cams, scales=scales, num_anchors=int(r.integers(1, 60)),
                        num_pts=int(r.integers(1, 14)), G=G, C=C, dtype=dt)
    lo, hi = [(0.0, 1.0), (-0.1, 1.1), (-0.5, 1.5)][r.integers(3)]
    return shape, lo, hi


AGG_KEYS = ("feat", "spatial_shape", "scale_start_index", "sampling_location", "weights")


@pytest.mark.parametrize("i", range(16))
def test_aggregation(i, cuda_dev):
    import deformable_convolution_sampling_dcn_b200 as d

    shape, lo, hi = draw_agg(i)
    inp = si.agg_inputs(shape, 12000 + i, with_grad_out=True, loc_lo=lo, loc_hi=hi)
    t = [inp[k].to(cuda_dev) for k in AGG_KEYS]
    out = d.deform_agg_forward(*t)
    gf, gl, gw = d.deform_agg_backward(*t, inp["grad_out"].to(cuda_dev))
    torch.cuda.synchronize()
    assert_close_fwd(out, oracle.agg_forward(*(inp[k] for k in AGG_KEYS)), f"random agg forward {i}")
    ref = oracle.agg_backward(*(inp[k] for k in AGG_KEYS), inp["grad_out"])
    budget = oracle.agg_grad_feat_budget(*(inp[k] for k in AGG_KEYS), inp["grad_out"])
    assert_close_bwd(gf, ref["grad_feat"], f"random agg grad_feat {i}", budget=budget)
    assert_close_bwd(gl, ref["grad_loc"], f"random agg grad_loc {i}")
    assert_close_bwd(gw, ref["grad_weights"], f"random agg grad_weights {i}")
