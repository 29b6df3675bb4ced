"""GPU parity of dcn_core_forward against the fp64 oracle (element by element)."""
import ctypes
import dataclasses

import numpy as np
import pytest
import torch

import oracle
import synthetic_inputs as si
from parity import assert_close_fwd

pytestmark = pytest.mark.gpu

DT = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}


def dcn():
    import deformable_convolution_sampling_dcn_b200 as d

    return d


def run_case(shape: si.CoreShape, inp, dev):
    d = dcn()
    x, off, m = (inp[k].to(dev) for k in ("x", "offset", "mask"))
    out = d.dcn_core_forward(x, off, m, group=shape.G, kernel=(shape.kh, shape.kw),
                             stride=(shape.stride_h, shape.stride_w), pad=(shape.pad_h, shape.pad_w),
                             dil=(shape.dil_h, shape.dil_w), offset_scale=shape.offset_scale,
                             softmax=shape.softmax)
    torch.cuda.synchronize()
    ref = oracle.dcn_forward(inp["x"], inp["offset"], inp["mask"], G=shape.G, kh=shape.kh, kw=shape.kw,
                             stride=(shape.stride_h, shape.stride_w), pad=(shape.pad_h, shape.pad_w),
                             dil=(shape.dil_h, shape.dil_w), offset_scale=shape.offset_scale,
                             softmax=shape.softmax)
    return out, ref


# ------------------------------------------------------------ the named workloads
@pytest.mark.parametrize("name", ["dcnv3_tiny", "dcnv4_p4", "dcnv3_p3", "dcnv3_p3_dil2"])
def test_workload_full_size(name, cuda_dev):
    shape, inp = si.workload_core(name)
    out, ref = run_case(shape, inp, cuda_dev)
    assert out.dtype == DT[shape.dtype]
    ratio = assert_close_fwd(out, ref, name)
    print(f"{name}: worst err/bound {ratio:.3f}")


# ------------------------------------------------------------ small ragged cases
SMALL = [
    # B, H, W, G, C, kh, kw, stride, pad, dil, scale, softmax, dtype
    (1, 7, 9, 3, 8, 3, 3, 1, 1, 1, 1.0, False, "f32"),
    (2, 13, 5, 2, 4, 3, 3, 2, 1, 1, 0.5, True, "f32"),
    (3, 6, 11, 1, 64, 3, 5, (1, 2), (1, 2), 1, 0.3, False, "f32"),
    (1, 1, 1, 4, 32, 3, 3, 1, 1, 1, 1.0, True, "f32"),
    (2, 9, 8, 2, 16, 3, 3, 1, 2, 2, 1.0, False, "f16"),
    (1, 17, 33, 3, 32, 5, 5, 1, 2, 1, 0.7, True, "f16"),
    (2, 5, 7, 1, 128, 1, 1, 1, 0, 1, 1.0, False, "f16"),
    (1, 12, 12, 4, 8, 3, 3, 2, 0, 1, 1.0, True, "f16"),
    (2, 10, 6, 2, 32, 3, 3, 1, 1, 1, 1.0, False, "bf16"),
    (1, 15, 15, 3, 64, 3, 3, 1, 2, 2, 0.25, True, "bf16"),
    (3, 4, 4, 5, 8, 2, 2, 1, 0, 1, 1.0, False, "bf16"),
    (1, 40, 40, 2, 32, 3, 3, 1, 1, 1, 1.0, False, "f16"),
    (1, 41, 39, 3, 32, 3, 3, 1, 1, 1, 1.0, True, "bf16"),
]


def _pair(v):
    return (v, v) if isinstance(v, int) else v


@pytest.mark.parametrize("case", range(len(SMALL)))
def test_small_ragged(case, cuda_dev):
    B, H, W, G, C, kh, kw, st, pd, dl, s, sm, dt = SMALL[case]
    st, pd, dl = _pair(st), _pair(pd), _pair(dl)
    shape = si.CoreShape(B=B, H=H, W=W, G=G, C=C, kh=kh, kw=kw, stride_h=st[0], stride_w=st[1], pad_h=pd[0],
                         pad_w=pd[1], dil_h=dl[0], dil_w=dl[1], offset_scale=s, softmax=sm, dtype=dt)
    inp = si.core_inputs(shape, 100 + case, offset_std=2.5, oob_fraction=0.05)
    out, ref = run_case(shape, inp, cuda_dev)
    assert_close_fwd(out, ref, f"small case {case}")


@pytest.mark.parametrize("name", ["dcnv3_tiny", "dcnv4_p4", "dcnv3_p3_dil2"])
def test_generic_path_full_size(name, cuda_dev, monkeypatch):
    """The generic kernel on the shapes the staged kernel normally takes."""
    monkeypatch.setenv("DCN_B200_FORCE_GENERIC", "1")
    shape, inp = si.workload_core(name)
    out, ref = run_case(shape, inp, cuda_dev)
    assert_close_fwd(out, ref, name + " generic")


@pytest.mark.parametrize("dt", ["f32", "f16", "bf16"])
def test_far_offsets_many_segments(dt, cuda_dev):
    """Offsets far beyond the staged halo (std 12 px) on a tall map: many taps
    take the direct global-memory path and every CTA walks several segments."""
    shape = si.CoreShape(B=2, H=150, W=37, G=2, C=32, dtype=dt, softmax=(dt == "bf16"))
    inp = si.core_inputs(shape, 11, offset_std=12.0, oob_fraction=0.02)
    out, ref = run_case(shape, inp, cuda_dev)
    assert_close_fwd(out, ref, "far offsets")
    d = dcn()
    assert d._binding.take_device_error() == 0


def test_strided_dilated_staged(cuda_dev):
    shape = si.CoreShape(B=3, H=61, W=45, G=3, C=16, kh=5, kw=3, stride_h=2, stride_w=3, pad_h=4, pad_w=2,
                         dil_h=2, dil_w=2, offset_scale=0.4, softmax=True, dtype="f16")
    inp = si.core_inputs(shape, 12, offset_std=3.0)
    out, ref = run_case(shape, inp, cuda_dev)
    assert_close_fwd(out, ref, "strided dilated")


def test_wide_pad_no_rows_staged(cuda_dev):
    """Padding so wide that some segments stage no input rows at all."""
    shape = si.CoreShape(B=1, H=9, W=11, G=2, C=32, kh=3, kw=3, pad_h=15, pad_w=3, dtype="f32")
    inp = si.core_inputs(shape, 13, offset_std=2.0)
    out, ref = run_case(shape, inp, cuda_dev)
    assert_close_fwd(out, ref, "wide pad")


def test_large_map(cuda_dev):
    """A 1024 x 1024 map (narrow groups): many tiles and a long grid-stride loop."""
    shape = si.CoreShape(B=1, H=1024, W=1024, G=1, C=8, dtype="f16")
    inp = si.core_inputs(shape, 7, offset_std=5.0)
    out, ref = run_case(shape, inp, cuda_dev)
    assert_close_fwd(out, ref, "large map")


# ------------------------------------------------------------ edge cases
def test_identity_exact(cuda_dev):
    """Zero offsets with a one-hot centre mask copy x bit for bit (all dtypes)."""
    d = dcn()
    for dt in (torch.float32, torch.float16, torch.bfloat16):
        x = torch.randn(2, 9, 7, 64, device=cuda_dev).to(dt)
        off = torch.zeros(2, 9, 7, 2, 9, 2, device=cuda_dev, dtype=dt)
        m = torch.zeros(2, 9, 7, 2, 9, device=cuda_dev, dtype=dt)
        m[..., 4] = 1
        out = d.dcn_core_forward(x, off, m, group=2)
        assert torch.equal(out, x)


def test_nan_and_far_offsets(cuda_dev):
    shape = si.CoreShape(B=1, H=8, W=8, G=2, C=32, dtype="f32")
    inp = si.core_inputs(shape, 3)
    inp["offset"][0, 2, 3, 1, 4, 1] = float("nan")
    inp["offset"][0, 5, 5, 0, :, 0] = float("inf")
    inp["offset"][0, 6, 6, 1, :, 1] = -1e30
    out, ref = run_case(shape, inp, cuda_dev)
    assert torch.isnan(out[0, 2, 3, 32:]).all() and not torch.isnan(out[0, 2, 3, :32]).any()
    assert_close_fwd(out, ref, "nan/far")


def test_empty_batch(cuda_dev):
    d = dcn()
    x = torch.zeros(0, 5, 5, 32, device=cuda_dev)
    off = torch.zeros(0, 5, 5, 1, 9, 2, device=cuda_dev)
    m = torch.zeros(0, 5, 5, 1, 9, device=cuda_dev)
    out = d.dcn_core_forward(x, off, m, group=1)
    assert out.shape == (0, 5, 5, 32)


def test_misaligned_pointer_rejected(cuda_dev):
    d = dcn()
    buf = torch.zeros(1 * 5 * 5 * 32 + 8, device=cuda_dev, dtype=torch.float16)
    x = buf[2:2 + 5 * 5 * 32].view(1, 5, 5, 32)  # 4-byte offset: not 16-byte aligned
    off = torch.zeros(1, 5, 5, 1, 9, 2, device=cuda_dev, dtype=torch.float16)
    m = torch.zeros(1, 5, 5, 1, 9, device=cuda_dev, dtype=torch.float16)
    with pytest.raises(d.DcnError) as e:
        d.dcn_core_forward(x, off, m, group=1)
    assert e.value.status == 4


def test_nonzero_stream(cuda_dev):
    """The call runs on torch's current stream (here a side stream)."""
    shape, inp = si.workload_core("dcnv3_tiny")
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        out, ref = run_case(shape, inp, cuda_dev)
    s.synchronize()
    assert_close_fwd(out, ref, "side stream")


def test_graph_capture_replay(cuda_dev):
    """The launch is capturable in a CUDA graph and replays to the same result."""
    d = dcn()
    shape, inp = si.workload_core("dcnv4_p4")
    x, off, m = (inp[k].to(cuda_dev) for k in ("x", "offset", "mask"))
    out = torch.empty(shape.B, shape.Ho, shape.Wo, shape.G * shape.C, device=cuda_dev, dtype=x.dtype)
    d.dcn_core_forward(x, off, m, group=shape.G, out=out)  # warm-up outside capture
    ref = out.clone()
    out.zero_()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        d.dcn_core_forward(x, off, m, group=shape.G, out=out)
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out, ref)
