"""The synthetic workloads match their stated recipes: sizes, storage types,
distributions, the share of taps placed outside the map, and the normalisation
of the aggregation weights.  The generators hold none of the method's
arithmetic; these checks keep the benchmark's inputs what the design notes say
they are."""
import numpy as np

import synthetic_inputs as si


def test_dcnv4_p4_recipe():
    shape, inp = si.workload_core("dcnv4_p4")
    assert (shape.B, shape.H, shape.W, shape.G, shape.C, shape.K) == (8, 40, 40, 16, 32, 9)
    assert inp["x"].dtype == si.DTYPES["f16"] and tuple(inp["offset"].shape) == (8, 40, 40, 16, 9, 2)
    assert shape.samples == 1_843_200 and shape.compulsory_bytes() == 37_273_600
    off, m, x = (inp[k].double().numpy() for k in ("offset", "mask", "x"))
    assert abs(off.std() - 3.0) < 0.03 and abs(off.mean()) < 0.01
    assert abs(m.std() - 1.0) < 0.01 and abs(x.std() - 1.0) < 0.01


def test_dcnv3_p3_far_taps():
    shape, inp = si.workload_core("dcnv3_p3")
    assert (shape.B, shape.H, shape.W, shape.G, shape.C) == (16, 80, 80, 8, 32) and shape.softmax
    off = inp["offset"].double().numpy()
    ho = np.arange(shape.Ho)[None, :, None, None, None]
    wo = np.arange(shape.Wo)[None, None, :, None, None]
    k = np.arange(shape.K)
    by = ho * shape.stride_h - shape.pad_h + (k // shape.kw) * shape.dil_h
    bx = wo * shape.stride_w - shape.pad_w + (k % shape.kw) * shape.dil_w
    py, px = by + off[..., 1], bx + off[..., 0]
    far = ((py <= -1) | (py >= shape.H)) & ((px <= -1) | (px >= shape.W))
    assert abs(far.mean() - 0.05) < 0.003          # 5 % placed outside on both axes
    near = np.abs(off).max(axis=-1) < 50
    assert abs(off[near].std() - 4.0) < 0.05       # the others N(0, 4^2)


def test_sparse4d_weights_normalised():
    s = si.SPARSE4D
    inp = si.agg_inputs(s, 3)
    w = inp["weights"].double().numpy()               # [B, A, P, cams, scales, G]
    assert w.shape == (1, 900, 13, 6, 4, 8)
    sums = w.sum(axis=(2, 3, 4))
    assert np.allclose(sums, 1.0, atol=1e-12)
    loc = inp["sampling_location"].numpy()
    assert loc.min() >= 0.0 and loc.max() <= 1.0
    assert s.num_rows == 89_760 and s.samples == 2_246_400
