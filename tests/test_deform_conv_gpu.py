"""GPU parity of dcn_deform_conv_forward (modulated deformable convolution,
a dense weight per kernel point, fused with the sampling) against the fp64
oracle, element by element."""
import numpy as np
import pytest
import torch

import oracle
import synthetic_inputs as si
from parity import assert_close_fwd

pytestmark = pytest.mark.gpu


def run(shape, inp, dev, with_bias=True):
    import deformable_convolution_sampling_dcn_b200 as d

    t = {k: v.to(dev) for k, v in inp.items()}
    g = dict(kernel=(shape.kh, shape.kw), stride=(shape.stride_h, shape.stride_w), pad=(shape.pad_h, shape.pad_w),
             dil=(shape.dil_h, shape.dil_w), offset_scale=shape.offset_scale, softmax=shape.softmax)
    out = d.dcn_deform_conv_forward(t["x"], t["offset"], t["mask"], t["weight"], t["bias"] if with_bias else None,
                                    group=shape.G, **g)
    torch.cuda.synchronize()
    assert d._binding.take_device_error() == 0
    ref = oracle.deform_conv_forward(inp["x"], inp["offset"], inp["mask"], inp["weight"],
                                     inp["bias"] if with_bias else None, G=shape.G, kh=shape.kh, kw=shape.kw,
                                     stride=g["stride"], pad=g["pad"], dil=g["dil"], offset_scale=shape.offset_scale,
                                     softmax=shape.softmax)
    return out, ref


def case(B, H, W, G, C, cout, dtype="f16", seed=0, kh=3, kw=3, stride=1, pad=1, dil=1, softmax=False,
         offset_std=2.0, oob=0.0):
    shape = si.CoreShape(B=B, H=H, W=W, G=G, C=C, kh=kh, kw=kw, stride_h=stride, stride_w=stride, pad_h=pad,
                         pad_w=pad, dil_h=dil, dil_w=dil, softmax=softmax, dtype=dtype)
    inp = si.core_inputs(shape, seed, offset_std=offset_std, oob_fraction=oob)
    inp.update(si.deform_conv_weights(shape.K, G * C, cout, dtype, seed + 500))
    return shape, inp


SMALL = [
    # B, H, W, G, C, Cout, dtype, kw-args
    (2, 9, 11, 4, 16, 40, "f16", {}),
    (1, 7, 5, 2, 32, 136, "bf16", dict(softmax=True)),
    (2, 10, 8, 1, 64, 8, "f16", dict(kh=1, kw=1, pad=0)),              # 1x1: a deformable pointwise conv
    (1, 12, 13, 8, 8, 96, "bf16", dict(kh=5, kw=5, pad=2)),            # 25 points, C = 8
    (1, 15, 19, 16, 32, 64, "f16", dict(stride=2, pad=2, dil=2, oob=0.1)),
    (1, 4, 5, 16, 32, 64, "f16", {}),                                  # 20 pixels: small chunks, 72 K-blocks
    # fewer than 11 items per K-block in a chunk: every lane computes its own tap
    (1, 3, 3, 8, 64, 64, "f16", {}),
    (1, 2, 5, 4, 64, 24, "bf16", dict(softmax=True)),
]


@pytest.mark.parametrize("i", range(len(SMALL)))
def test_small_cases(i, cuda_dev):
    B, H, W, G, C, cout, dt, kw = SMALL[i]
    shape, inp = case(B, H, W, G, C, cout, dt, seed=60 + i, **kw)
    out, ref = run(shape, inp, cuda_dev)
    assert out.shape == (B, shape.Ho, shape.Wo, cout)
    assert_close_fwd(out, ref, f"deform conv case {i}")


def test_without_bias_and_regular_conv_limit(cuda_dev):
    """Zero offsets and unit masks: the result is an ordinary convolution."""
    shape, inp = case(2, 10, 9, 2, 32, 48, "f16", seed=70)
    inp["offset"] = torch.zeros_like(inp["offset"])
    inp["mask"] = torch.ones_like(inp["mask"])
    out, ref = run(shape, inp, cuda_dev, with_bias=False)
    assert_close_fwd(out, ref, "deform conv, zero offsets")
    w = inp["weight"].double().reshape(48, 3, 3, 64).permute(0, 3, 1, 2)
    conv = torch.nn.functional.conv2d(inp["x"].double().permute(0, 3, 1, 2), w, padding=1)
    assert_close_fwd(out, conv.permute(0, 2, 3, 1).numpy(), "deform conv vs conv2d")


@pytest.mark.parametrize("B,H,W,G,C,cout,dt,softmax", [
    (4, 70, 70, 2, 32, 64, "f16", False),     # 19,600 pixels: two chunks per CTA
    (4, 100, 100, 4, 16, 32, "bf16", True),   # 40,000 pixels: three chunks per CTA
])
def test_several_chunks_per_cta(B, H, W, G, C, cout, dt, softmax, cuda_dev):
    """More than 128 pixels per CTA: the per-point work list, the weight stream and
    the accumulators are reused chunk after chunk."""
    shape, inp = case(B, H, W, G, C, cout, dt, seed=90 + B + H, softmax=softmax)
    out, ref = run(shape, inp, cuda_dev)
    assert_close_fwd(out, ref, f"deform conv {B}x{H}x{W}")


def test_dcnv2_p4_full_size(cuda_dev):
    """DCNv2-style deformable convolution at the P4 shape: B=8, 40x40, 512 input
    channels as 16 deformable groups of 32, 3x3, 256 output channels, fp16."""
    shape, inp = case(8, 40, 40, 16, 32, 256, "f16", seed=80, offset_std=3.0)
    out, ref = run(shape, inp, cuda_dev)
    ratio = assert_close_fwd(out, ref, "dcnv2 p4")
    print(f"dcnv2 p4: worst err/bound {ratio:.3f}")
