"""GPU parity of deform_agg_forward / deform_agg_backward against the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
import synthetic_inputs as si
from parity import assert_close_bwd, assert_close_fwd

pytestmark = pytest.mark.gpu


def run_fwd(inp, dev):
    import deformable_convolution_sampling_dcn_b200 as d

    keys = ("feat", "spatial_shape", "scale_start_index", "sampling_location", "weights")
    out = d.deform_agg_forward(*(inp[k].to(dev) for k in keys))
    torch.cuda.synchronize()
    assert d.lib().dcn_take_device_error() == 0
    ref = oracle.agg_forward(*(inp[k] for k in keys))
    return out, ref


def test_sparse4d_full_size_generic(cuda_dev, monkeypatch):
    """The per-group kernels on the shape the anchor-wide kernels normally take."""
    monkeypatch.setenv("DCN_B200_FORCE_GENERIC", "1")
    inp = si.agg_inputs(si.SPARSE4D, si.SEEDS["sparse4d"])
    out, ref = run_fwd(inp, cuda_dev)
    assert_close_fwd(out, ref, "sparse4d generic")


def test_sparse4d_backward_generic(cuda_dev, monkeypatch):
    monkeypatch.setenv("DCN_B200_FORCE_GENERIC", "1")
    shape = si.AggShape(B=1, num_cams=3, scales=((16, 44), (8, 22)), num_anchors=40, num_pts=5, G=8, C=32)
    inp = si.agg_inputs(shape, 77, with_grad_out=True, loc_lo=-0.05, loc_hi=1.05)
    (gf, gl, gw), ref = run_bwd(inp, cuda_dev)
    assert_close_bwd(gf, ref["grad_feat"], "grad_feat", budget=ref["budget"])
    assert_close_bwd(gw, ref["grad_weights"], "grad_weights")
    assert_close_bwd(gl, ref["grad_loc"], "grad_loc")


def test_sparse4d_full_size(cuda_dev):
    inp = si.agg_inputs(si.SPARSE4D, si.SEEDS["sparse4d"])
    out, ref = run_fwd(inp, cuda_dev)
    r = assert_close_fwd(out, ref, "sparse4d")
    print(f"sparse4d: worst err/bound {r:.3f}")


def test_feat_only_16_byte_aligned(cuda_dev):
    """A feat that is 16- but not 32-byte aligned takes the 16-byte loads."""
    import deformable_convolution_sampling_dcn_b200 as d

    shape = si.AggShape(B=2, num_cams=3, scales=((9, 13), (4, 6)), num_anchors=21, num_pts=4, G=8, C=32)
    inp = si.agg_inputs(shape, 516, loc_lo=-0.1, loc_hi=1.1)
    f = inp["feat"]
    buf = torch.empty(f.numel() + 4, dtype=f.dtype, device=cuda_dev)
    feat = buf[4:].view(f.shape)
    feat.copy_(f.to(cuda_dev))
    assert feat.data_ptr() % 32 == 16
    keys = ("spatial_shape", "scale_start_index", "sampling_location", "weights")
    out = d.deform_agg_forward(feat, *(inp[k].to(cuda_dev) for k in keys))
    torch.cuda.synchronize()
    ref = oracle.agg_forward(*(inp[k] for k in ("feat",) + keys))
    assert_close_fwd(out, ref, "16-byte aligned feat")


def test_nan_and_far_locations(cuda_dev):
    """NaN locations make their anchor's row NaN; locations far outside [0, 1]
    contribute zero."""
    shape = si.AggShape(B=2, num_cams=3, scales=((9, 13), (4, 6)), num_anchors=21, num_pts=4, G=4, C=32)
    inp = si.agg_inputs(shape, 515, loc_lo=-0.1, loc_hi=1.1)
    loc = inp["sampling_location"]
    loc[0, 3, 1, 2, 0] = float("nan")
    loc[1, 7, 0, 0, 1] = float("nan")
    loc[0, 5, 2, 1] = torch.tensor([-40.0, 3.0])
    loc[1, 11, 3, 2] = torch.tensor([float("inf"), -float("inf")])
    loc[1, 12, 0, 1] = torch.tensor([2.0e9, 0.5])
    out, ref = run_fwd(inp, cuda_dev)
    assert np.isnan(ref).sum() == 2 * shape.G * shape.C
    assert_close_fwd(out, ref, "nan/far")


SMALL = [
    # B, cams, scales, A, P, G, C, dtype, loc range
    (1, 2, ((5, 7), (3, 4)), 3, 2, 2, 8, "f32", (-0.1, 1.1)),
    (2, 3, ((7, 9), (3, 5)), 11, 3, 4, 32, "f32", (-0.1, 1.1)),      # 512-byte rows: anchor-wide
    (1, 2, ((6, 10),), 9, 4, 8, 64, "f16", (-0.1, 1.1)),             # 1024-byte rows: anchor-wide
    (1, 4, ((5, 6), (4, 3), (2, 2)), 7, 2, 16, 64, "bf16", (0.0, 1.0)),  # 2048-byte rows
    (2, 3, ((9, 13), (4, 6), (2, 3)), 17, 5, 4, 32, "f32", (0.0, 1.0)),
    (1, 6, ((16, 44), (8, 22)), 50, 13, 8, 32, "f16", (-0.05, 1.05)),
    (2, 1, ((10, 10),), 9, 3, 1, 64, "bf16", (-0.2, 1.2)),
    (1, 2, ((6, 5),), 33, 4, 3, 16, "f16", (0.0, 1.0)),
]


def small_shape(case):
    B, cams, scales, A, P, G, C, dt, lr = SMALL[case]
    return si.AggShape(B=B, num_cams=cams, scales=scales, num_anchors=A, num_pts=P, G=G, C=C, dtype=dt), lr


@pytest.mark.parametrize("case", range(len(SMALL)))
def test_small_forward(case, cuda_dev):
    shape, lr = small_shape(case)
    inp = si.agg_inputs(shape, 300 + case, loc_lo=lr[0], loc_hi=lr[1])
    out, ref = run_fwd(inp, cuda_dev)
    assert_close_fwd(out, ref, f"agg small {case}")


def run_bwd(inp, dev):
    import deformable_convolution_sampling_dcn_b200 as d

    keys = ("feat", "spatial_shape", "scale_start_index", "sampling_location", "weights", "grad_out")
    got = d.deform_agg_backward(*(inp[k].to(dev) for k in keys))
    torch.cuda.synchronize()
    assert d.lib().dcn_take_device_error() == 0
    ref = oracle.agg_backward(*(inp[k] for k in keys))
    ref["budget"] = oracle.agg_grad_feat_budget(*(inp[k] for k in keys))
    return got, ref


@pytest.mark.parametrize("case", range(len(SMALL)))
def test_small_backward(case, cuda_dev):
    shape, lr = small_shape(case)
    inp = si.agg_inputs(shape, 400 + case, loc_lo=lr[0], loc_hi=lr[1], with_grad_out=True)
    (gf, gl, gw), ref = run_bwd(inp, cuda_dev)
    assert_close_bwd(gf, ref["grad_feat"], "grad_feat", budget=ref["budget"])
    assert_close_bwd(gw, ref["grad_weights"], "grad_weights")
    # locations are fp32 in every dtype; their gradient sums fp32 atomics
    gl64 = gl.double().cpu().numpy()
    r = ref["grad_loc"]
    tol = {"f32": 1e-4, "f16": 2e-2, "bf16": 1e-1}[shape.dtype]
    rms = float(np.sqrt(np.mean(r * r)))
    assert np.all(np.abs(gl64 - r) <= tol * (np.abs(r) + rms))


def test_sparse4d_backward_full_size(cuda_dev):
    inp = si.agg_inputs(si.SPARSE4D, si.SEEDS["sparse4d"], with_grad_out=True)
    (gf, gl, gw), ref = run_bwd(inp, cuda_dev)
    assert_close_bwd(gf, ref["grad_feat"], "grad_feat", budget=ref["budget"])
    assert_close_bwd(gw, ref["grad_weights"], "grad_weights")
    assert_close_bwd(gl, ref["grad_loc"], "grad_loc")


def test_bad_table_rows_are_not_read(cuda_dev):
    """A start index that points past num_rows yields zero, not a fault."""
    import deformable_convolution_sampling_dcn_b200 as d

    shape = si.AggShape(B=1, num_cams=2, scales=((4, 4),), num_anchors=5, num_pts=2, G=1, C=8)
    inp = si.agg_inputs(shape, 9)
    bad = inp["scale_start_index"].clone()
    bad[1, 0] = 10_000  # camera 1 points far outside feat
    keys = ("feat", "spatial_shape", "scale_start_index", "sampling_location", "weights")
    args = [inp[k].to(cuda_dev) for k in keys]
    args[2] = bad.to(cuda_dev)
    out = d.deform_agg_forward(*args)
    torch.cuda.synchronize()
    # the reference: the same call with camera 1's weights zeroed and a valid table
    w = inp["weights"].clone()
    w[:, :, :, 1] = 0
    ref = oracle.agg_forward(inp["feat"], inp["spatial_shape"], inp["scale_start_index"],
                             inp["sampling_location"], w)
    assert_close_fwd(out, ref, "bad table")


def test_backward_clustered_locations(cuda_dev):
    """Units packed into a few cells of the maps (many reductions into the same
    feature rows) and a few NaN and far locations."""
    shape = si.AggShape(B=2, num_cams=3, scales=((18, 40), (9, 20), (4, 10)), num_anchors=60, num_pts=7, G=8,
                        C=32)
    inp = si.agg_inputs(shape, 812, with_grad_out=True)
    rng = np.random.default_rng(813)
    loc = inp["sampling_location"].numpy()
    centres = rng.uniform(0.1, 0.9, (5, 2))
    pick = rng.integers(0, 5, loc.shape[:-1])
    loc[:] = (centres[pick] + rng.normal(0.0, 0.01, loc.shape)).astype(np.float32)
    loc[0, 3, 2, 1] = [np.nan, 0.5]
    loc[1, 10, 0, 2] = [3.0, -2.0]
    inp["sampling_location"] = torch.from_numpy(loc)
    (gf, gl, gw), ref = run_bwd(inp, cuda_dev)
    assert np.isnan(ref["grad_loc"]).sum() == 2
    assert_close_bwd(gf, ref["grad_feat"], "grad_feat", budget=ref["budget"])
    assert_close_bwd(gw, ref["grad_weights"], "grad_weights", atomic=False)
    assert_close_bwd(gl, ref["grad_loc"], "grad_loc", atomic=False)
