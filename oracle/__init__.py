"""fp64 CPU oracle for the deformable sampling-aggregation core.

TEST INFRASTRUCTURE ONLY. The tests, the smoke check and the benchmark's
CPU-baseline leg call it; the library's product path never imports it. It
shares no code with the CUDA library: the arithmetic lives in dcn_oracle.c,
plain C loops in fp64 that follow the page formulas (cited in that file), and
this module only builds that file with gcc and marshals numpy arrays to it.

Inputs may be torch tensors or numpy arrays in any float dtype; they are
widened to float64 exactly (fp16/bf16/fp32 values are all representable).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from typing import Dict, Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "dcn_oracle.c")
_LIB = os.path.join(_HERE, "libdcn_oracle.so")
_lock = threading.Lock()
_lib = None

CFLAGS = ["-O2", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-std=c11"]


def build(src: str = _SRC, out: str = _LIB, extra: Optional[list] = None) -> str:
    """Compile the oracle with gcc (no fast-math, no FP contraction)."""
    cmd = ["gcc", *CFLAGS, *(extra or []), src, "-o", out, "-lm"]
    subprocess.run(cmd, check=True)
    return out


def _stale() -> bool:
    return (not os.path.exists(_LIB)) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC)


def load(path: Optional[str] = None):
    """Load (building first if needed) the oracle shared library."""
    global _lib
    if path is not None:
        return _bind(ctypes.CDLL(path))
    with _lock:
        if _lib is None:
            if _stale():
                build()
            _lib = _bind(ctypes.CDLL(_LIB))
    return _lib


def _bind(lib):
    dp = ctypes.POINTER(ctypes.c_double)
    fp = ctypes.POINTER(ctypes.c_float)
    ip = ctypes.POINTER(ctypes.c_int)
    i = ctypes.c_int
    lib.oracle_set_threads.argtypes = [i]
    lib.oracle_set_threads.restype = i
    lib.oracle_dcn_forward.argtypes = [i] * 13 + [ctypes.c_float, i, dp, dp, dp, dp]
    lib.oracle_dcn_forward.restype = None
    lib.oracle_dcn_backward.argtypes = [i] * 13 + [ctypes.c_float, i, dp, dp, dp, dp, dp, dp, dp]
    lib.oracle_dcn_backward.restype = None
    lib.oracle_dcn_grad_x_budget.argtypes = [i] * 13 + [ctypes.c_float, i, dp, dp, dp, dp, dp]
    lib.oracle_dcn_grad_x_budget.restype = None
    lib.oracle_agg_grad_feat_budget.argtypes = [i] * 8 + [ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_int),
                                                          ctypes.POINTER(ctypes.c_float), dp, dp, dp, dp]
    lib.oracle_agg_grad_feat_budget.restype = None
    lib.oracle_agg_forward.argtypes = [i] * 8 + [dp, ip, ip, fp, dp, dp]
    lib.oracle_agg_forward.restype = None
    lib.oracle_agg_backward.argtypes = [i] * 8 + [dp, ip, ip, fp, dp, dp, dp, dp, dp]
    lib.oracle_agg_backward.restype = None
    lib.oracle_roi_pool_forward.argtypes = [i] * 8 + [ctypes.c_float, ctypes.c_float, dp, fp, fp, dp]
    lib.oracle_roi_pool_forward.restype = None
    lib.oracle_pointwise_projection.argtypes = [ctypes.c_longlong, i, i, dp, dp, dp, dp]
    lib.oracle_pointwise_projection.restype = None
    lib.oracle_deform_conv_forward.argtypes = [i] * 13 + [ctypes.c_float, i, i, dp, dp, dp, dp, dp, dp]
    lib.oracle_deform_conv_forward.restype = None
    return lib


def _f64(a) -> np.ndarray:
    if hasattr(a, "detach"):  # torch tensor
        a = a.detach().cpu()
        a = a.double().numpy()
    return np.ascontiguousarray(a, dtype=np.float64)


def _ptr(a: np.ndarray, ct):
    return a.ctypes.data_as(ctypes.POINTER(ct))


def set_threads(n: int) -> int:
    """Set the OpenMP thread count (n <= 0 keeps it); returns the count in use."""
    return int(load().oracle_set_threads(int(n)))


def out_hw(H, W, kh, kw, stride_h, stride_w, pad_h, pad_w, dil_h, dil_w):
    Ho = (H + 2 * pad_h - (dil_h * (kh - 1) + 1)) // stride_h + 1
    Wo = (W + 2 * pad_w - (dil_w * (kw - 1) + 1)) // stride_w + 1
    return Ho, Wo


def dcn_forward(x, offset, mask, *, G: int, kh: int = 3, kw: int = 3, stride=(1, 1), pad=(1, 1),
                dil=(1, 1), offset_scale: float = 1.0, softmax: bool = False, lib=None) -> np.ndarray:
    """out [B,Ho,Wo,G*C] in fp64 from x [B,H,W,G*C], offset [B,Ho,Wo,G,K,2], mask [B,Ho,Wo,G,K]."""
    lib = lib or load()
    x, offset, mask = _f64(x), _f64(offset), _f64(mask)
    B, H, W, GC = x.shape
    C = GC // G
    Ho, Wo = out_hw(H, W, kh, kw, *stride, *pad, *dil)
    assert offset.shape == (B, Ho, Wo, G, kh * kw, 2), offset.shape
    assert mask.shape == (B, Ho, Wo, G, kh * kw), mask.shape
    out = np.empty((B, Ho, Wo, G * C), dtype=np.float64)
    lib.oracle_dcn_forward(B, H, W, G, C, kh, kw, stride[0], stride[1], pad[0], pad[1], dil[0], dil[1],
                           float(offset_scale), int(bool(softmax)), _ptr(x, ctypes.c_double),
                           _ptr(offset, ctypes.c_double), _ptr(mask, ctypes.c_double),
                           _ptr(out, ctypes.c_double))
    return out


def pointwise_projection(v, weight, bias=None, *, lib=None) -> np.ndarray:
    """out [..., Cout] = bias + v [..., Cin] . weight[Cout, Cin]^T in fp64 (1x1 convolution with bias)."""
    lib = lib or load()
    v, weight = _f64(v), _f64(weight)
    Cout, Cin = weight.shape
    assert v.shape[-1] == Cin, (v.shape, weight.shape)
    npix = int(np.prod(v.shape[:-1]))
    b = None if bias is None else _f64(bias)
    assert b is None or b.shape == (Cout,)
    out = np.empty(v.shape[:-1] + (Cout,), dtype=np.float64)
    lib.oracle_pointwise_projection(npix, Cin, Cout, _ptr(v, ctypes.c_double), _ptr(weight, ctypes.c_double),
                                    None if b is None else _ptr(b, ctypes.c_double), _ptr(out, ctypes.c_double))
    return out


def dcn_forward_proj(x, offset, mask, weight, bias=None, *, G: int, lib=None, **core) -> np.ndarray:
    """The sampling core followed by its pointwise projection, both in fp64:
    pointwise_projection(dcn_forward(x, offset, mask, ...), weight, bias)."""
    return pointwise_projection(dcn_forward(x, offset, mask, G=G, lib=lib, **core), weight, bias, lib=lib)


def deform_conv_forward(x, offset, mask, weight, bias=None, *, G: int, kh: int = 3, kw: int = 3, stride=(1, 1),
                        pad=(1, 1), dil=(1, 1), offset_scale: float = 1.0, softmax: bool = False,
                        lib=None) -> np.ndarray:
    """out [B,Ho,Wo,Cout] in fp64: modulated deformable convolution with weight [Cout, K, G*C]."""
    lib = lib or load()
    x, offset, mask, weight = _f64(x), _f64(offset), _f64(mask), _f64(weight)
    B, H, W, GC = x.shape
    C = GC // G
    K = kh * kw
    Cout = weight.shape[0]
    assert weight.shape == (Cout, K, GC), weight.shape
    Ho, Wo = out_hw(H, W, kh, kw, *stride, *pad, *dil)
    assert offset.shape == (B, Ho, Wo, G, K, 2) and mask.shape == (B, Ho, Wo, G, K)
    b = None if bias is None else _f64(bias)
    out = np.empty((B, Ho, Wo, Cout), dtype=np.float64)
    lib.oracle_deform_conv_forward(B, H, W, G, C, kh, kw, stride[0], stride[1], pad[0], pad[1], dil[0], dil[1],
                                   float(offset_scale), int(bool(softmax)), Cout, _ptr(x, ctypes.c_double),
                                   _ptr(offset, ctypes.c_double), _ptr(mask, ctypes.c_double),
                                   _ptr(weight, ctypes.c_double), None if b is None else _ptr(b, ctypes.c_double),
                                   _ptr(out, ctypes.c_double))
    return out


def dcn_backward(x, offset, mask, grad_out, *, G: int, kh: int = 3, kw: int = 3, stride=(1, 1),
                 pad=(1, 1), dil=(1, 1), offset_scale: float = 1.0, softmax: bool = False,
                 lib=None) -> Dict[str, np.ndarray]:
    """grad_x, grad_offset, grad_mask (fp64) of <grad_out, forward(x, offset, mask)>."""
    lib = lib or load()
    x, offset, mask, go = _f64(x), _f64(offset), _f64(mask), _f64(grad_out)
    B, H, W, GC = x.shape
    C = GC // G
    Ho, Wo = out_hw(H, W, kh, kw, *stride, *pad, *dil)
    assert go.shape == (B, Ho, Wo, GC)
    gx = np.empty_like(x)
    goff = np.empty_like(offset)
    gm = np.empty_like(mask)
    lib.oracle_dcn_backward(B, H, W, G, C, kh, kw, stride[0], stride[1], pad[0], pad[1], dil[0], dil[1],
                            float(offset_scale), int(bool(softmax)), _ptr(x, ctypes.c_double),
                            _ptr(offset, ctypes.c_double), _ptr(mask, ctypes.c_double),
                            _ptr(go, ctypes.c_double), _ptr(gx, ctypes.c_double),
                            _ptr(goff, ctypes.c_double), _ptr(gm, ctypes.c_double))
    return {"grad_x": gx, "grad_offset": goff, "grad_mask": gm}


def dcn_grad_x_budget(offset, mask, grad_out, *, x_shape, G: int, kh: int = 3, kw: int = 3, stride=(1, 1),
                      pad=(1, 1), dil=(1, 1), offset_scale: float = 1.0, softmax: bool = False,
                      lib=None) -> Dict[str, np.ndarray]:
    """Per grad_x element: the absolute sum of its contributions (abs_sum,
    [B,H,W,G*C]) and their number (terms, [B,H,W,G]); see dcn_oracle.c."""
    lib = lib or load()
    offset, mask, go = _f64(offset), _f64(mask), _f64(grad_out)
    B, H, W, GC = x_shape
    C = GC // G
    abs_sum = np.empty((B, H, W, GC), dtype=np.float64)
    terms = np.empty((B, H, W, G), dtype=np.float64)
    lib.oracle_dcn_grad_x_budget(B, H, W, G, C, kh, kw, stride[0], stride[1], pad[0], pad[1], dil[0], dil[1],
                                 float(offset_scale), int(bool(softmax)), _ptr(offset, ctypes.c_double),
                                 _ptr(mask, ctypes.c_double), _ptr(go, ctypes.c_double),
                                 _ptr(abs_sum, ctypes.c_double), _ptr(terms, ctypes.c_double))
    return {"abs_sum": abs_sum, "terms": terms}


def _agg_common(feat, spatial_shape, scale_start_index, sampling_location, weights):
    feat = _f64(feat)
    ss = np.ascontiguousarray(np.asarray(spatial_shape), dtype=np.int32)
    st = np.ascontiguousarray(np.asarray(scale_start_index), dtype=np.int32)
    loc = sampling_location
    if hasattr(loc, "detach"):
        loc = loc.detach().cpu().numpy()
    loc = np.ascontiguousarray(loc, dtype=np.float32)
    w = _f64(weights)
    B, rows, GC = feat.shape
    _, A, P, cams, S, G = w.shape
    assert ss.shape == (cams, S, 2) and st.shape == (cams, S)
    assert loc.shape == (B, A, P, cams, 2)
    return feat, ss, st, loc, w, (B, cams, S, rows, A, P, G, GC // G)


def agg_forward(feat, spatial_shape, scale_start_index, sampling_location, weights, lib=None) -> np.ndarray:
    """out [B,A,G*C] (fp64) of the multi-camera multi-scale aggregation."""
    lib = lib or load()
    feat, ss, st, loc, w, dims = _agg_common(feat, spatial_shape, scale_start_index,
                                             sampling_location, weights)
    B, cams, S, rows, A, P, G, C = dims
    out = np.empty((B, A, G * C), dtype=np.float64)
    lib.oracle_agg_forward(*dims, _ptr(feat, ctypes.c_double), _ptr(ss, ctypes.c_int),
                           _ptr(st, ctypes.c_int), _ptr(loc, ctypes.c_float), _ptr(w, ctypes.c_double),
                           _ptr(out, ctypes.c_double))
    return out


def agg_backward(feat, spatial_shape, scale_start_index, sampling_location, weights, grad_out,
                 lib=None) -> Dict[str, np.ndarray]:
    """grad_feat, grad_loc, grad_weights (fp64) of <grad_out, agg_forward(...)>."""
    lib = lib or load()
    feat, ss, st, loc, w, dims = _agg_common(feat, spatial_shape, scale_start_index,
                                             sampling_location, weights)
    B, cams, S, rows, A, P, G, C = dims
    go = _f64(grad_out)
    assert go.shape == (B, A, G * C)
    gf = np.empty_like(feat)
    gl = np.empty(loc.shape, dtype=np.float64)
    gw = np.empty_like(w)
    lib.oracle_agg_backward(*dims, _ptr(feat, ctypes.c_double), _ptr(ss, ctypes.c_int),
                            _ptr(st, ctypes.c_int), _ptr(loc, ctypes.c_float), _ptr(w, ctypes.c_double),
                            _ptr(go, ctypes.c_double), _ptr(gf, ctypes.c_double),
                            _ptr(gl, ctypes.c_double), _ptr(gw, ctypes.c_double))
    return {"grad_feat": gf, "grad_loc": gl, "grad_weights": gw}


def agg_grad_feat_budget(feat, spatial_shape, scale_start_index, sampling_location, weights, grad_out,
                         lib=None) -> Dict[str, np.ndarray]:
    """Per grad_feat element: the absolute sum of its contributions (abs_sum,
    [B, rows, G*C]) and their number (terms, [B, rows, G]); see dcn_oracle.c."""
    lib = lib or load()
    feat, ss, st, loc, w, dims = _agg_common(feat, spatial_shape, scale_start_index,
                                             sampling_location, weights)
    B, cams, S, rows, A, P, G, C = dims
    go = _f64(grad_out)
    abs_sum = np.empty((B, rows, G * C), dtype=np.float64)
    terms = np.empty((B, rows, G), dtype=np.float64)
    lib.oracle_agg_grad_feat_budget(*dims, _ptr(ss, ctypes.c_int), _ptr(st, ctypes.c_int),
                                    _ptr(loc, ctypes.c_float), _ptr(w, ctypes.c_double),
                                    _ptr(go, ctypes.c_double), _ptr(abs_sum, ctypes.c_double),
                                    _ptr(terms, ctypes.c_double))
    return {"abs_sum": abs_sum, "terms": terms}


def roi_pool_forward(x, rois, offset, *, pooled=(7, 7), sampling=2, spatial_scale: float = 1.0,
                     gamma: float = 0.1, lib=None) -> np.ndarray:
    """out [N, PH, PW, C] (fp64) of deformable RoI pooling over x [B, H, W, C].

    rois [N, 5] (batch, x1, y1, x2, y2) and offset [N, PH, PW, 2] are fp32.  A
    region whose batch index lies outside [0, B) (or is NaN) pools to zeros."""
    lib = lib or load()
    x = _f64(x)
    B, H, W, C = x.shape
    r = rois.detach().cpu().numpy() if hasattr(rois, "detach") else rois
    o = offset.detach().cpu().numpy() if hasattr(offset, "detach") else offset
    r = np.ascontiguousarray(r, dtype=np.float32)
    o = np.ascontiguousarray(o, dtype=np.float32)
    N = r.shape[0]
    PH, PW = pooled
    assert r.shape == (N, 5) and o.shape == (N, PH, PW, 2)
    out = np.empty((N, PH, PW, C), dtype=np.float64)
    lib.oracle_roi_pool_forward(B, H, W, C, N, PH, PW, int(sampling), float(spatial_scale), float(gamma),
                                _ptr(x, ctypes.c_double), _ptr(r, ctypes.c_float), _ptr(o, ctypes.c_float),
                                _ptr(out, ctypes.c_double))
    return out
