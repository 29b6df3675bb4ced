"""GPU parity of dcn_core_forward_proj (the core followed by its 1x1
projection) against the fp64 oracle, element by element, on both routes: the
one fused kernel, and the core into a workspace followed by the tensor-core
GEMM."""
import numpy as np
import pytest
import torch

import oracle
import synthetic_inputs as si
from parity import assert_close_fwd

pytestmark = pytest.mark.gpu

ROUTES = ["fused", "workspace"]


def dcn():
    import deformable_convolution_sampling_dcn_b200 as d

    return d


def run(shape: si.CoreShape, inp, dev, with_bias=True, route="fused"):
    d = dcn()
    t = {k: v.to(dev) for k, v in inp.items()}
    geo = dict(kernel=(shape.kh, shape.kw), stride=(shape.stride_h, shape.stride_w), pad=(shape.pad_h, shape.pad_w),
               dil=(shape.dil_h, shape.dil_w), offset_scale=shape.offset_scale, softmax=shape.softmax)
    out = d.dcn_core_forward_proj(t["x"], t["offset"], t["mask"], t["weight"], t["bias"] if with_bias else None,
                                  group=shape.G, fused=(route == "fused"), **geo)
    torch.cuda.synchronize()
    assert d._binding.take_device_error() == 0
    core = oracle.dcn_forward(inp["x"], inp["offset"], inp["mask"], G=shape.G, kh=shape.kh, kw=shape.kw,
                              stride=geo["stride"], pad=geo["pad"], dil=geo["dil"],
                              offset_scale=shape.offset_scale, softmax=shape.softmax)
    ref = oracle.pointwise_projection(core, inp["weight"], inp["bias"] if with_bias else None)
    return out, ref, core


def case(B, H, W, G, C, cout, dtype="f16", seed=0, kh=3, kw=3, stride=1, pad=1, dil=1, softmax=False,
         oob=0.0, offset_std=3.0):
    shape = si.CoreShape(B=B, H=H, W=W, G=G, C=C, kh=kh, kw=kw, stride_h=stride, stride_w=stride, pad_h=pad,
                         pad_w=pad, dil_h=dil, dil_w=dil, softmax=softmax, dtype=dtype)
    inp = si.core_inputs(shape, seed, offset_std=offset_std, oob_fraction=oob)
    inp.update(si.proj_inputs(G * C, cout, dtype, seed + 1000))
    return shape, inp


SMALL = [
    # B, H, W, G, C, Cout, dtype, kw-args
    (2, 9, 11, 4, 16, 40, "f16", {}),                              # one K-block, Cout < 128
    (1, 7, 5, 4, 32, 136, "bf16", {}),                             # two K-blocks, a partial second M-block
    (3, 13, 17, 2, 64, 8, "f16", dict(softmax=True)),              # smallest Cout, softmax modulation
    (2, 12, 10, 8, 8, 256, "bf16", dict(kh=5, kw=5, pad=2)),       # 25 points, C = 8
    (1, 15, 19, 16, 32, 512, "f16", dict(stride=2, pad=2, dil=2, oob=0.05)),  # strided, dilated, all K-blocks
    (1, 1, 1, 2, 32, 64, "f16", {}),                               # a single output pixel
    # 20 pixels -> 2 CTAs of 10: the gather warps' first steps start in late
    # K-blocks, so each must hand over the earlier ones before waiting on a slot
    (1, 4, 5, 16, 32, 64, "f16", {}),
    (1, 3, 3, 8, 64, 24, "bf16", {}),                              # 9 pixels, C = 64
]


@pytest.mark.parametrize("route", ROUTES)
@pytest.mark.parametrize("i", range(len(SMALL)))
def test_small_cases(i, route, cuda_dev):
    B, H, W, G, C, cout, dt, kw = SMALL[i]
    shape, inp = case(B, H, W, G, C, cout, dt, seed=40 + i, **kw)
    out, ref, _ = run(shape, inp, cuda_dev, route=route)
    assert out.shape == (B, shape.Ho, shape.Wo, cout)
    assert_close_fwd(out, ref, f"proj case {i}")


@pytest.mark.parametrize("route", ROUTES)
def test_without_bias(route, cuda_dev):
    shape, inp = case(2, 8, 9, 4, 32, 128, "f16", seed=50)
    out, ref, _ = run(shape, inp, cuda_dev, with_bias=False, route=route)
    assert_close_fwd(out, ref, "proj without bias")


@pytest.mark.parametrize("route", ROUTES)
def test_many_chunks_per_cta(route, cuda_dev):
    """More pixels than 148 CTAs x 128 pixels: every CTA runs several chunks
    (fused) or tiles (GEMM), reusing its tensor memory."""
    shape, inp = case(3, 84, 90, 4, 16, 72, "bf16", seed=51)
    out, ref, _ = run(shape, inp, cuda_dev, route=route)
    assert_close_fwd(out, ref, "proj many chunks")


@pytest.mark.parametrize("route", ROUTES)
def test_rounded_core_reading(route, cuda_dev):
    """The core is rounded once to the storage type before the projection:
    the output is within the fp16 bar of both the plain definition and the
    projection of the rounded core."""
    shape, inp = case(2, 10, 12, 8, 32, 96, "f16", seed=52)
    out, ref, core = run(shape, inp, cuda_dev, route=route)
    core16 = torch.from_numpy(core).to(torch.float16).double().numpy()
    ref16 = oracle.pointwise_projection(core16, inp["weight"], inp["bias"])
    assert_close_fwd(out, ref, "proj vs definition")
    assert_close_fwd(out, ref16, "proj vs rounded core")


@pytest.mark.parametrize("route", ROUTES)
def test_nan_and_outside_positions(route, cuda_dev):
    """A NaN sampling position makes every output channel of its pixel NaN; a
    pixel whose taps all fall outside the map outputs the bias."""
    shape, inp = case(1, 6, 7, 2, 32, 64, "f16", seed=53)
    off = inp["offset"].clone()
    off[0, 1, 2, 1, 4, 0] = float("nan")
    off[0, 3, 3] = 1000.0  # every tap of every group of pixel (3, 3) far outside
    inp["offset"] = off
    out, ref, _ = run(shape, inp, cuda_dev, route=route)
    assert torch.isnan(out[0, 1, 2]).all()
    assert torch.equal(out[0, 3, 3].cpu(), inp["bias"])
    assert_close_fwd(out, ref, "proj nan/outside")


@pytest.mark.parametrize("route", ROUTES)
def test_dcnv4_p4_full_size(route, cuda_dev):
    """The DCNv4 P4 workload (B=8, 40x40, G=16, C=32, fp16) with its 512 -> 512
    projection, every output element."""
    shape, inp = si.workload_proj()
    out, ref, _ = run(shape, inp, cuda_dev, route=route)
    ratio = assert_close_fwd(out, ref, "dcnv4_p4 proj")
    print(f"dcnv4_p4 proj ({route}): worst err/bound {ratio:.3f}")


def test_workspace_holds_the_core(cuda_dev):
    """On the workspace route the workspace ends up holding exactly what
    dcn_core_forward stores (the same kernels), and the projection is the GEMM
    of it; a workspace one byte short falls back to the fused kernel."""
    d = dcn()
    shape, inp = case(2, 11, 13, 8, 32, 104, "bf16", seed=55, softmax=True)
    t = {k: v.to(cuda_dev) for k, v in inp.items()}
    core = d.dcn_core_forward(t["x"], t["offset"], t["mask"], group=shape.G, softmax=True)
    ws = torch.empty(core.numel() * 2, dtype=torch.uint8, device=cuda_dev)
    out = d.dcn_core_forward_proj(t["x"], t["offset"], t["mask"], t["weight"], t["bias"], group=shape.G,
                                  softmax=True, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(ws.view(torch.bfloat16).view(core.shape), core)
    ref = oracle.pointwise_projection(core.double().cpu().numpy(), inp["weight"], inp["bias"])
    assert_close_fwd(out, ref, "projection of the stored core")
    short = torch.zeros(core.numel() * 2 - 1, dtype=torch.uint8, device=cuda_dev)
    out2 = d.dcn_core_forward_proj(t["x"], t["offset"], t["mask"], t["weight"], t["bias"], group=shape.G,
                                   softmax=True, workspace=short)
    torch.cuda.synchronize()
    assert torch.count_nonzero(short) == 0  # untouched: the fused kernel ran
    assert_close_fwd(out2, ref, "fused fallback")


def test_rejects_unsupported(cuda_dev):
    d = dcn()
    shape, inp = case(1, 4, 4, 2, 32, 64, "f16", seed=54)
    t = {k: v.to(cuda_dev) for k, v in inp.items()}
    with pytest.raises(d.DcnError):  # Cout not a multiple of 8
        d.dcn_core_forward_proj(t["x"], t["offset"], t["mask"], t["weight"][:60].contiguous(), None, group=2)
    with pytest.raises(d.DcnError):  # fp32 storage
        d.dcn_core_forward_proj(t["x"].float(), t["offset"].float(), t["mask"].float(), t["weight"].float(), None,
                                group=2)
