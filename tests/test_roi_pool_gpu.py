"""GPU parity of deform_roi_pool_forward against the fp64 oracle."""
import pytest
import torch

import oracle
import synthetic_inputs as si
from parity import assert_close_fwd

pytestmark = pytest.mark.gpu


def run(shape: si.RoiShape, inp, dev):
    import deformable_convolution_sampling_dcn_b200 as d

    out = d.deform_roi_pool_forward(inp["x"].to(dev), inp["rois"].to(dev), inp["offset"].to(dev),
                                    pooled=(shape.PH, shape.PW), sampling=shape.S,
                                    spatial_scale=shape.spatial_scale, gamma=shape.gamma)
    torch.cuda.synchronize()
    ref = oracle.roi_pool_forward(inp["x"], inp["rois"], inp["offset"], pooled=(shape.PH, shape.PW),
                                  sampling=shape.S, spatial_scale=shape.spatial_scale, gamma=shape.gamma)
    return out, ref


def test_roi_pool_workload(cuda_dev):
    shape = si.ROI_POOL
    inp = si.roi_inputs(shape, si.SEEDS["roi_pool"])
    out, ref = run(shape, inp, cuda_dev)
    assert_close_fwd(out, ref, "roi pool")


@pytest.mark.parametrize("case", [
    # B, H, W, C, N, PH, PW, S, scale, gamma, dtype
    (1, 9, 13, 8, 5, 3, 4, 2, 0.5, 0.1, "f32"),
    (2, 20, 17, 64, 33, 7, 7, 3, 0.25, 0.3, "f16"),
    (3, 11, 11, 16, 7, 2, 5, 1, 1.0, 1.0, "bf16"),
    (1, 33, 40, 512, 9, 4, 4, 2, 0.125, 0.2, "f16"),
    (2, 15, 19, 256, 21, 3, 3, 2, 0.5, 0.2, "f32"),    # 1 KB rows: 32-byte chunks
    (1, 12, 14, 1024, 6, 2, 3, 2, 0.5, 0.1, "bf16"),   # 2 KB rows: 32-byte chunks, 2 per lane
    (1, 10, 12, 40, 5, 2, 2, 2, 1.0, 0.1, "f32"),      # 160-byte rows: a partial last chunk block
])
def test_roi_pool_small(case, cuda_dev):
    B, H, W, C, N, PH, PW, S, sc, gm, dt = case
    shape = si.RoiShape(B=B, H=H, W=W, C=C, N=N, PH=PH, PW=PW, S=S, spatial_scale=sc, gamma=gm, dtype=dt)
    inp = si.roi_inputs(shape, 500 + N, offset_std=1.5, min_size=2.0)
    out, ref = run(shape, inp, cuda_dev)
    assert_close_fwd(out, ref, f"roi small {case}")


def test_roi_bad_batch_index_reads_nothing(cuda_dev):
    """Regions whose batch index names no image (B, -1, NaN) pool to zeros, as
    the oracle defines; the others match it as usual."""
    import deformable_convolution_sampling_dcn_b200 as d

    shape = si.RoiShape(B=1, H=8, W=8, C=32, N=5, PH=2, PW=2, spatial_scale=1.0)
    inp = si.roi_inputs(shape, 9, min_size=2.0)
    inp["rois"][1, 0] = 5.0  # no such image
    inp["rois"][3, 0] = -1.0
    inp["rois"][4, 0] = float("nan")
    out = d.deform_roi_pool_forward(inp["x"].to(cuda_dev), inp["rois"].to(cuda_dev), inp["offset"].to(cuda_dev),
                                    pooled=(2, 2), spatial_scale=1.0)
    torch.cuda.synchronize()
    ref = oracle.roi_pool_forward(inp["x"], inp["rois"], inp["offset"], pooled=(2, 2), spatial_scale=1.0)
    assert (ref[[1, 3, 4]] == 0).all()
    assert_close_fwd(out, ref, "roi bad batch index")
    assert torch.count_nonzero(out[[1, 3, 4]]) == 0


def test_roi_pool_x_only_16_byte_aligned(cuda_dev):
    """An x that is 16- but not 32-byte aligned takes the 16-byte chunks."""
    import deformable_convolution_sampling_dcn_b200 as d

    shape = si.RoiShape(B=2, H=15, W=19, C=256, N=13, PH=3, PW=3, S=2, spatial_scale=0.5, gamma=0.2)
    inp = si.roi_inputs(shape, 533, offset_std=1.5, min_size=2.0)
    xs = inp["x"]
    buf = torch.empty(xs.numel() + 4, dtype=xs.dtype, device=cuda_dev)
    x = buf[4:].view(xs.shape)
    x.copy_(xs.to(cuda_dev))
    assert x.data_ptr() % 32 == 16
    out = d.deform_roi_pool_forward(x, inp["rois"].to(cuda_dev), inp["offset"].to(cuda_dev),
                                    pooled=(shape.PH, shape.PW), sampling=shape.S,
                                    spatial_scale=shape.spatial_scale, gamma=shape.gamma)
    torch.cuda.synchronize()
    ref = oracle.roi_pool_forward(inp["x"], inp["rois"], inp["offset"], pooled=(shape.PH, shape.PW),
                                  sampling=shape.S, spatial_scale=shape.spatial_scale, gamma=shape.gamma)
    assert_close_fwd(out, ref, "roi 16-byte aligned x")
