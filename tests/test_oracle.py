"""The fp64 oracle against its pins (CPU only).

Runs every pin in oracle_pins, checks the hand-worked golden values, and
shows that the pins have teeth: each planted mistake (a swapped offset
component, a wrong padding sign, a transposed kernel-point index, a dropped
term, ...) compiled into a copy of the oracle makes at least one pin fail.
"""
import json
import os
import shutil
import subprocess

import numpy as np
import pytest

import oracle
import oracle_pins as pins

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "worked_examples.json")


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin, oracle_lib):
    pin(oracle_lib)


def test_golden_core_raw(oracle_lib):
    ex = json.load(open(GOLDEN))["core_raw"]
    x = np.array(ex["x"], dtype=np.float64).reshape(1, 2, 3, 1)
    off = np.array(ex["offset_dx_dy"], dtype=np.float64).reshape(1, 2, 3, 1, 1, 2)
    mask = np.array(ex["mask"], dtype=np.float64).reshape(1, 2, 3, 1, 1)
    out = oracle.dcn_forward(x, off, mask, G=1, kh=1, kw=1, pad=(0, 0), lib=oracle_lib)
    assert np.array_equal(out.reshape(-1), np.array(ex["expected"]).reshape(-1))


def test_golden_core_softmax(oracle_lib):
    ex = json.load(open(GOLDEN))["core_softmax"]
    x = np.array(ex["x"], dtype=np.float64).reshape(1, 1, 1, 1)
    off = np.zeros((1, 1, 1, 1, 9, 2))
    for case in ex["cases"]:
        logits = np.array(case["logits"], dtype=np.float64).reshape(1, 1, 1, 1, 9)
        out = oracle.dcn_forward(x, off, logits, G=1, softmax=True, lib=oracle_lib)
        assert abs(out.item() - case["expected"]) < 1e-14


def test_golden_aggregation(oracle_lib):
    ex = json.load(open(GOLDEN))["aggregation"]
    feat = np.array(ex["feat_rows"], dtype=np.float64).reshape(1, 6, 1)
    shape = np.array([[[2, 3]]], dtype=np.int32)
    start = np.array([[0]], dtype=np.int32)
    loc = np.array(ex["loc_uv"], dtype=np.float32).reshape(1, 1, 3, 1, 2)
    w = np.array(ex["weights"], dtype=np.float64).reshape(1, 1, 3, 1, 1, 1)
    out = oracle.agg_forward(feat, shape, start, loc, w, lib=oracle_lib)
    assert out.item() == ex["expected"]


def test_golden_deform_conv(oracle_lib):
    ex = json.load(open(GOLDEN))["deform_conv"]
    x = np.array(ex["x"], dtype=np.float64).reshape(1, 1, 3, 1)
    off = np.array(ex["offset_dx_dy"], dtype=np.float64).reshape(1, 1, 2, 1, 2, 2)
    mask = np.array(ex["mask"], dtype=np.float64).reshape(1, 1, 2, 1, 2)
    w = np.array(ex["weight_out_point"], dtype=np.float64).reshape(2, 2, 1)
    b = np.array(ex["bias"], dtype=np.float64)
    out = oracle.deform_conv_forward(x, off, mask, w, b, G=1, kh=1, kw=2, pad=(0, 0), lib=oracle_lib)
    assert np.array_equal(out.reshape(2, 2), np.array(ex["expected_out_pixel_channel"]))


def test_golden_roi_pool(oracle_lib):
    ex = json.load(open(GOLDEN))["roi_pool"]
    x = np.array(ex["x_rows"], dtype=np.float64).reshape(1, 2, 4, 1)
    rois = np.array([ex["roi"]], dtype=np.float32)
    off = np.array(ex["offset_dx_dy"], dtype=np.float32).reshape(1, 1, 1, 2)
    out = oracle.roi_pool_forward(x, rois, off, pooled=(1, 1), sampling=2, spatial_scale=1.0, gamma=0.25,
                                  lib=oracle_lib)
    assert out.item() == ex["expected"]


def test_golden_core_backward(oracle_lib):
    ex = json.load(open(GOLDEN))["core_backward"]
    x = np.array(ex["x_rows"], dtype=np.float64).reshape(1, 2, 2, 1)
    off = np.zeros((1, 2, 2, 1, 1, 2))
    off[0, 0, 0, 0, 0] = ex["offset_dx_dy_pixel00"]
    mask = np.zeros((1, 2, 2, 1, 1))
    mask[0, 0, 0, 0, 0] = ex["mask_pixel00"]
    go = np.zeros((1, 2, 2, 1))
    go[0, 0, 0, 0] = ex["grad_out_pixel00"]
    g = oracle.dcn_backward(x, off, mask, go, G=1, kh=1, kw=1, pad=(0, 0), lib=oracle_lib)
    e = ex["expected"]
    assert g["grad_mask"][0, 0, 0, 0, 0] == e["grad_mask_pixel00"]
    assert g["grad_offset"][0, 0, 0, 0, 0, 0] == e["grad_dx_pixel00"]
    assert g["grad_offset"][0, 0, 0, 0, 0, 1] == e["grad_dy_pixel00"]
    assert np.array_equal(g["grad_x"].reshape(2, 2), np.array(e["grad_x_rows"]))
    assert np.count_nonzero(g["grad_offset"]) == 2 and np.count_nonzero(g["grad_mask"]) == 1


def test_nan_position_propagates(oracle_lib):
    """A sampling position that is not a number poisons its (pixel, group)."""
    x = np.ones((1, 4, 4, 2 * 3))
    off = np.zeros((1, 4, 4, 2, 9, 2))
    off[0, 1, 2, 1, 3, 0] = np.nan
    out = oracle.dcn_forward(x, off, np.ones((1, 4, 4, 2, 9)), G=2, lib=oracle_lib)
    bad = np.isnan(out)
    assert bad[0, 1, 2, 3:6].all() and bad.sum() == 3


def test_far_offsets_contribute_nothing(oracle_lib):
    x = np.random.default_rng(0).standard_normal((1, 5, 5, 4))
    off = np.full((1, 5, 5, 1, 9, 2), 1e30)
    off[..., 1] = -np.inf
    out = oracle.dcn_forward(x, off, np.ones((1, 5, 5, 1, 9)), G=1, lib=oracle_lib)
    assert np.array_equal(out, np.zeros_like(out))


# ------------------------------------------------------------------ mutations
# (text to replace, replacement, occurrences to replace (0 = all), pins to run)
MUTATIONS = [
    ("(float)d[0], (float)bx", "(float)d[1], (float)bx", 0, pins.CORE_PINS),
    # strict support (-1 < p instead of -1 <= p) in the backward
    ("if (!(fy >= -1.0 && fy <= H - 1 && fx >= -1.0 && fx <= W - 1)) continue;",
     "if (!(fy > -1.0 && fy <= H - 1 && fx > -1.0 && fx <= W - 1)) continue;", 0, pins.BACKWARD_PINS),
    ("const int by = ho * sh - ph + i * dh;", "const int by = ho * sh + ph + i * dh;", 0, pins.CORE_PINS),
    ("const int bx = wo * sw - pw + j * dw;", "const int bx = wo * sw - pw + j;", 0, pins.CORE_PINS),
    ("const int by = ho * sh - ph + i * dh;", "const int by = ho - ph + i * dh;", 0, pins.CORE_PINS),
    ("const int k = i * kw + j;", "const int k = j * kh + i;", 1, pins.CORE_PINS),
    ("1.0 - fabs(a - b)", "1.0 - 0.5 * fabs(a - b)", 0, pins.CORE_PINS),
    ("m[k] /= s;", "m[k] /= (s + 1e-3);", 0, pins.CORE_PINS),
    ("if (qy < 0 || qy >= H) continue;", "if (qy < 0 || qy >= H - 1) continue;", 1, pins.CORE_PINS),
    ("y[c] += m[k] * Gq * xq[c];", "y[c] += Gq * xq[c];", 1, pins.CORE_PINS),
    ("return q == q_floor ? -1.0 : 1.0;", "return q == q_floor ? 1.0 : -1.0;", 0, pins.BACKWARD_PINS),
    ("gxq[c] += m[k] * gx * gy * go[c];", "gxq[c] += gx * gy * go[c];", 0, pins.BACKWARD_PINS),
    ("gl[k] = m[k] * (gm[k] - dot);", "gl[k] = m[k] * gm[k];", 0, pins.BACKWARD_PINS),
    ("gd[0] = (double)offset_scale * m[k] * dpx;", "gd[0] = m[k] * dpx;", 0, pins.BACKWARD_PINS),
    ("dpy += go[c] * gx * dgy * xq[c];", "dpy += go[c] * dgx * gy * xq[c];", 0, pins.BACKWARD_PINS),
    ("fmaf(l[0], (float)Ws, -0.5f)", "fmaf(l[0], (float)Ws, 0.0f)", 0, pins.AGG_PINS),
    ("(size_t)qy * Ws + qx;", "(size_t)qx * Hs + qy;", 1, pins.AGG_PINS),
    ("y[c] += w * Gq * f[c];", "y[c] += Gq * f[c];", 0, pins.AGG_PINS),
    ("glp[li + 0] += w * dpx * Ws;", "glp[li + 0] += w * dpx;", 0, pins.AGG_PINS),
    ("grad_feat[off + c] += w * gx * gy * go[c];", "grad_feat[off + c] += gx * gy * go[c];", 0,
     pins.AGG_PINS),
    ("const float dx = (gamma * d[0]) * rw, dy = (gamma * d[1]) * rh;",
     "const float dx = (gamma * d[1]) * rw, dy = (gamma * d[0]) * rh;", 0, pins.ROI_PINS),
    ("const float dx = (gamma * d[0]) * rw, dy = (gamma * d[1]) * rh;",
     "const float dx = (gamma * d[0]) * rw, dy = (gamma * d[1]) * rw;", 0, pins.ROI_PINS),
    ("const float bx0 = x1 + (float)j * bw, by0 = y1 + (float)i * bh;",
     "const float bx0 = x1 + (float)i * bw, by0 = y1 + (float)j * bh;", 0, pins.ROI_PINS),
    ("y[c] / (double)(S * S)", "y[c] / (double)S", 0, pins.ROI_PINS),
    ("const float px = (bx0 + ((float)sx + 0.5f) * sw) + dx;", "const float px = (bx0 + (float)sx * sw) + dx;", 0,
     pins.ROI_PINS),
    ("const float x1 = r[1] * spatial_scale, y1 = r[2] * spatial_scale;",
     "const float x1 = r[1], y1 = r[2] * spatial_scale;", 0, pins.ROI_PINS),
    ("const double *w = Wt + (size_t)o * Cin;", "const double *w = Wt + (size_t)o;", 0, pins.PROJ_PINS),
    # weight read as [Cin, Cout] (transposed; every index stays inside the array)
    ("const double *w = Wt + (size_t)o * Cin;\n            double s = bias ? bias[o] : 0.0;\n"
     "            for (int c = 0; c < Cin; ++c) s += w[c] * v[c];",
     "const double *w = Wt + (size_t)o;\n            double s = bias ? bias[o] : 0.0;\n"
     "            for (int c = 0; c < Cin; ++c) s += w[(size_t)c * Cout] * v[c];", 0, pins.PROJ_PINS),
    ("double *ck = col + (size_t)k * GC + (size_t)g * C;", "double *ck = col + (size_t)g * K * C + (size_t)k * C;",
     0, pins.DCONV_PINS),
    ("for (int c = 0; c < C; ++c) ck[c] += m[k] * Gq * xq[c];", "for (int c = 0; c < C; ++c) ck[c] += Gq * xq[c];",
     0, pins.DCONV_PINS),
    ("double acc = bias ? bias[o] : 0.0;", "double acc = 0.0;", 0, pins.DCONV_PINS),
    # the softmax flag ignored (raw modulation always)
    ("modulation(mask + item * K, K, softmax, m);", "modulation(mask + item * K, K, 0, m);", 0, pins.DCONV_PINS),
    ("double s = bias ? bias[o] : 0.0;", "double s = 0.0;", 0, pins.PROJ_PINS),
    ("double s = bias ? bias[o] : 0.0;", "double s = bias ? bias[0] : 0.0;", 0, pins.PROJ_PINS),
]


@pytest.mark.parametrize("mut", range(len(MUTATIONS)))
def test_pins_catch_planted_mistake(mut, tmp_path):
    old, new, count, pin_set = MUTATIONS[mut]
    src = open(oracle._SRC).read()
    n = src.count(old)
    assert n >= 1, f"mutation text not found: {old}"
    mutated = src.replace(old, new) if count == 0 else src.replace(old, new, count)
    csrc = tmp_path / "mutant.c"
    csrc.write_text(mutated)
    so = str(tmp_path / "libmutant.so")
    oracle.build(str(csrc), so)
    lib = oracle.load(so)
    failed = []
    for pin in pin_set:
        try:
            pin(lib)
        except AssertionError:
            failed.append(pin.__name__)
    assert failed, f"no pin caught mutation {mut}: {old!r} -> {new!r}"
