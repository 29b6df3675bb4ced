"""ctypes binding of libdcn_b200.so (argument marshalling only).

Every function here checks devices, dtypes, shapes and contiguity, allocates
outputs with torch when the caller passes none, and forwards raw device
pointers plus torch's current CUDA stream to the C ABI declared in
include/dcn_b200.h.  All arithmetic runs in the library's CUDA kernels; there
is no CPU path.  If the shared library is missing the first call raises.
"""
from __future__ import annotations

import ctypes
import os
import threading
from typing import Optional, Sequence, Tuple

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libdcn_b200.so")

DCN_OK, DCN_ERR_NULL, DCN_ERR_SHAPE, DCN_ERR_UNSUPPORTED, DCN_ERR_ALIGN, DCN_ERR_CUDA = range(6)
DCN_F32, DCN_F16, DCN_BF16 = 0, 1, 2
DCN_MASK_RAW, DCN_MASK_SOFTMAX = 0, 1
_DTYPE_CODE = {torch.float32: DCN_F32, torch.float16: DCN_F16, torch.bfloat16: DCN_BF16}

# Every entry point include/dcn_b200.h declares.
EXPORTS = ("dcn_core_output_hw", "dcn_core_forward", "dcn_core_backward", "deform_agg_forward",
           "deform_agg_backward", "dcn_status_string", "dcn_last_error_detail", "dcn_abi_version",
           "dcn_take_device_error", "deform_roi_pool_forward", "dcn_core_forward_proj",
           "dcn_selftest_bounded_wait", "dcn_deform_conv_forward", "dcn_probe_rate",
           "dcn_core_forward_proj_workspace_bytes", "dcn_core_forward_proj_noalloc")
ABI_VERSION = 2


class DcnParams(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("B", "H", "W", "G", "C", "kh", "kw", "stride_h", "stride_w",
                                              "pad_h", "pad_w", "dil_h", "dil_w")] + \
               [("offset_scale", ctypes.c_float), ("mask_mode", ctypes.c_int32), ("dtype", ctypes.c_int32)]


class DaggParams(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("B", "num_cams", "num_scales", "num_rows", "num_anchors",
                                              "num_pts", "G", "C", "dtype")]


class DroiParams(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("B", "H", "W", "C", "num_rois", "pooled_h", "pooled_w",
                                              "sampling")] + \
               [("spatial_scale", ctypes.c_float), ("gamma", ctypes.c_float), ("dtype", ctypes.c_int32)]


class DcnError(RuntimeError):
    def __init__(self, status: int, detail: str):
        super().__init__(detail)
        self.status = status


_lock = threading.Lock()
_lib = None


def _declare(lib):
    vp, st = ctypes.c_void_p, ctypes.c_int
    P = ctypes.POINTER(DcnParams)
    A = ctypes.POINTER(DaggParams)
    i32p = ctypes.POINTER(ctypes.c_int32)
    lib.dcn_core_output_hw.argtypes = [P, i32p, i32p]
    lib.dcn_core_forward.argtypes = [P, vp, vp, vp, vp, vp]
    lib.dcn_core_backward.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp]
    lib.deform_agg_forward.argtypes = [A, vp, vp, vp, vp, vp, vp, vp]
    lib.deform_agg_backward.argtypes = [A, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp]
    for f in ("dcn_core_output_hw", "dcn_core_forward", "dcn_core_backward", "deform_agg_forward",
              "deform_agg_backward"):
        getattr(lib, f).restype = st
    lib.dcn_status_string.argtypes = [st]
    lib.dcn_status_string.restype = ctypes.c_char_p
    lib.dcn_last_error_detail.argtypes = []
    lib.dcn_last_error_detail.restype = ctypes.c_char_p
    lib.dcn_abi_version.argtypes = []
    lib.dcn_abi_version.restype = ctypes.c_int32
    lib.deform_roi_pool_forward.argtypes = [ctypes.POINTER(DroiParams), vp, vp, vp, vp, vp]
    lib.deform_roi_pool_forward.restype = st
    lib.dcn_core_forward_proj.argtypes = [P, ctypes.c_int32, vp, vp, vp, vp, vp, vp, vp, ctypes.c_int64, vp]
    lib.dcn_core_forward_proj.restype = st
    lib.dcn_core_forward_proj_workspace_bytes.argtypes = [P]
    lib.dcn_core_forward_proj_workspace_bytes.restype = ctypes.c_int64
    lib.dcn_core_forward_proj_noalloc.argtypes = [P, ctypes.c_int32, vp, vp, vp, vp, vp, vp, vp]
    lib.dcn_core_forward_proj_noalloc.restype = st
    lib.dcn_deform_conv_forward.argtypes = [P, ctypes.c_int32, vp, vp, vp, vp, vp, vp, vp]
    lib.dcn_deform_conv_forward.restype = st
    lib.dcn_selftest_bounded_wait.argtypes = [ctypes.c_int32, vp]
    lib.dcn_selftest_bounded_wait.restype = st
    lib.dcn_take_device_error.argtypes = []
    lib.dcn_take_device_error.restype = ctypes.c_int32
    lib.dcn_probe_rate.argtypes = [ctypes.c_int32, ctypes.c_int32, vp, ctypes.c_int64,
                                   ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_char_p), vp]
    lib.dcn_probe_rate.restype = st
    return lib


def lib(path: Optional[str] = None):
    """The loaded library (declared argtypes).  Raises if it is not built."""
    global _lib
    if path is not None:
        return _declare(ctypes.CDLL(path))
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                                   "`python -m deformable_convolution_sampling_dcn_b200.build`")
            l = _declare(ctypes.CDLL(LIB_PATH))
            if l.dcn_abi_version() != ABI_VERSION:
                raise RuntimeError("libdcn_b200.so ABI version mismatch; rebuild it")
            _lib = l
    return _lib


def check(status: int) -> None:
    if status != DCN_OK:
        L = lib()
        raise DcnError(status, f"{L.dcn_status_string(status).decode()}: {L.dcn_last_error_detail().decode()}")


def _pair(v) -> Tuple[int, int]:
    if isinstance(v, (tuple, list)):
        return int(v[0]), int(v[1])
    return int(v), int(v)


def _cuda_tensor(name, t: torch.Tensor, dtype=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device.type != "cuda":
        raise ValueError(f"{name} must be a CUDA tensor (the library has no CPU path)")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} has dtype {t.dtype}, expected {dtype}")
    return t


def _stream(t: torch.Tensor) -> int:
    return torch.cuda.current_stream(t.device).cuda_stream


def core_params(x: torch.Tensor, G: int, kernel=(3, 3), stride=(1, 1), pad=(1, 1), dil=(1, 1),
                offset_scale: float = 1.0, softmax: bool = False) -> DcnParams:
    if x.dtype not in _DTYPE_CODE:
        raise TypeError(f"unsupported dtype {x.dtype}")
    B, H, W, GC = x.shape
    if GC % G:
        raise ValueError(f"channels {GC} not divisible by G={G}")
    kh, kw = _pair(kernel)
    sh, sw = _pair(stride)
    ph, pw = _pair(pad)
    dh, dw = _pair(dil)
    return DcnParams(B, H, W, G, GC // G, kh, kw, sh, sw, ph, pw, dh, dw, float(offset_scale),
                     DCN_MASK_SOFTMAX if softmax else DCN_MASK_RAW, _DTYPE_CODE[x.dtype])


def take_device_error() -> int:
    """Read and clear the device error word (0 = no bounded wait ran out)."""
    return int(lib().dcn_take_device_error())


PROBES = ("lds128", "chunk_f32_ffma2", "ffma", "ffma2", "chunk_f16_ffma", "chunk_f16_ffma2", "chunk_bf16_ffma2",
          "chunk_f16_mixed", "ldg128_l1", "gather4", "gather8", "gather8_ffma", "alu", "ldg256_l1",
          "atoms_f32")


def probe_rate(name: str, reps: int, device=None) -> Tuple[float, str]:
    """Run one on-chip rate probe; returns (units per SM per clock, unit)."""
    dev = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
    buf = torch.zeros(65536, dtype=torch.uint8, device=dev)
    units = ctypes.c_double()
    unit = ctypes.c_char_p()
    check(lib().dcn_probe_rate(PROBES.index(name), int(reps), buf.data_ptr(), buf.numel(), ctypes.byref(units),
                               ctypes.byref(unit), torch.cuda.current_stream(dev).cuda_stream))
    torch.cuda.synchronize(dev)
    words = buf[:16].view(torch.int64).cpu().tolist()
    return units.value * words[1] / words[0], unit.value.decode()


def selftest_bounded_wait(limit_us: int = 2000, device=None) -> None:
    """Enqueue the bounded-wait self-test on the current stream (see dcn_b200.h)."""
    check(lib().dcn_selftest_bounded_wait(int(limit_us), torch.cuda.current_stream(device).cuda_stream))


def dcn_core_output_hw(p: DcnParams) -> Tuple[int, int]:
    ho, wo = ctypes.c_int32(), ctypes.c_int32()
    check(lib().dcn_core_output_hw(ctypes.byref(p), ctypes.byref(ho), ctypes.byref(wo)))
    return ho.value, wo.value


def dcn_core_forward(x: torch.Tensor, offset: torch.Tensor, mask: torch.Tensor, *, group: int,
                     kernel=(3, 3), stride=(1, 1), pad=(1, 1), dil=(1, 1), offset_scale: float = 1.0,
                     softmax: bool = False, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """out [B,Ho,Wo,G*C] = sum_k m_k bilinear(x, p_k) per (pixel, group); see dcn_b200.h."""
    _cuda_tensor("x", x)
    p = core_params(x, group, kernel, stride, pad, dil, offset_scale, softmax)
    Ho, Wo = dcn_core_output_hw(p)
    K = p.kh * p.kw
    _cuda_tensor("offset", offset, x.dtype)
    _cuda_tensor("mask", mask, x.dtype)
    if tuple(offset.shape) != (p.B, Ho, Wo, p.G, K, 2):
        raise ValueError(f"offset shape {tuple(offset.shape)} != {(p.B, Ho, Wo, p.G, K, 2)}")
    if tuple(mask.shape) != (p.B, Ho, Wo, p.G, K):
        raise ValueError(f"mask shape {tuple(mask.shape)} != {(p.B, Ho, Wo, p.G, K)}")
    if out is None:
        out = torch.empty((p.B, Ho, Wo, p.G * p.C), dtype=x.dtype, device=x.device)
    else:
        _cuda_tensor("out", out, x.dtype)
        if tuple(out.shape) != (p.B, Ho, Wo, p.G * p.C):
            raise ValueError("out has the wrong shape")
    check(lib().dcn_core_forward(ctypes.byref(p), x.data_ptr(), offset.data_ptr(), mask.data_ptr(),
                                 out.data_ptr(), _stream(x)))
    return out


def dcn_core_forward_proj(x: torch.Tensor, offset: torch.Tensor, mask: torch.Tensor, weight: torch.Tensor,
                          bias: Optional[torch.Tensor] = None, *, group: int, kernel=(3, 3), stride=(1, 1),
                          pad=(1, 1), dil=(1, 1), offset_scale: float = 1.0, softmax: bool = False,
                          out: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                          fused: bool = False) -> torch.Tensor:
    """out [B,Ho,Wo,Cout] = bias + core(x, offset, mask) . weight[Cout, G*C]^T; see dcn_b200.h.

    By default the core goes through a workspace (`workspace`, or one torch
    allocates here) and a tensor-core GEMM projects it; fused=True runs the one
    fused kernel with no workspace."""
    _cuda_tensor("x", x)
    p = core_params(x, group, kernel, stride, pad, dil, offset_scale, softmax)
    Ho, Wo = dcn_core_output_hw(p)
    K = p.kh * p.kw
    _cuda_tensor("offset", offset, x.dtype)
    _cuda_tensor("mask", mask, x.dtype)
    _cuda_tensor("weight", weight, x.dtype)
    if tuple(offset.shape) != (p.B, Ho, Wo, p.G, K, 2):
        raise ValueError(f"offset shape {tuple(offset.shape)} != {(p.B, Ho, Wo, p.G, K, 2)}")
    if tuple(mask.shape) != (p.B, Ho, Wo, p.G, K):
        raise ValueError(f"mask shape {tuple(mask.shape)} != {(p.B, Ho, Wo, p.G, K)}")
    if weight.dim() != 2 or weight.shape[1] != p.G * p.C:
        raise ValueError(f"weight shape {tuple(weight.shape)} != (Cout, {p.G * p.C})")
    cout = int(weight.shape[0])
    if bias is not None:
        _cuda_tensor("bias", bias, x.dtype)
        if tuple(bias.shape) != (cout,):
            raise ValueError(f"bias shape {tuple(bias.shape)} != ({cout},)")
    if out is None:
        out = torch.empty((p.B, Ho, Wo, cout), dtype=x.dtype, device=x.device)
    else:
        _cuda_tensor("out", out, x.dtype)
        if tuple(out.shape) != (p.B, Ho, Wo, cout):
            raise ValueError("out has the wrong shape")
    ws_ptr, ws_bytes = None, 0
    if not fused:
        need = int(lib().dcn_core_forward_proj_workspace_bytes(ctypes.byref(p)))
        if workspace is None:
            workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=x.device)
        else:
            _cuda_tensor("workspace", workspace)
        ws_ptr, ws_bytes = workspace.data_ptr(), workspace.numel() * workspace.element_size()
    check(lib().dcn_core_forward_proj(ctypes.byref(p), cout, x.data_ptr(), offset.data_ptr(), mask.data_ptr(),
                                      weight.data_ptr(), None if bias is None else bias.data_ptr(),
                                      out.data_ptr(), ws_ptr, ws_bytes, _stream(x)))
    return out


def dcn_deform_conv_forward(x: torch.Tensor, offset: torch.Tensor, mask: torch.Tensor, weight: torch.Tensor,
                            bias: Optional[torch.Tensor] = None, *, group: int, kernel=(3, 3), stride=(1, 1),
                            pad=(1, 1), dil=(1, 1), offset_scale: float = 1.0, softmax: bool = False,
                            out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """out [B,Ho,Wo,Cout] = bias + sum_k weight[:, k, :] . (m_k x(p_k)): modulated deformable convolution
    with weight [Cout, K, G*C] in one kernel; see dcn_b200.h."""
    _cuda_tensor("x", x)
    p = core_params(x, group, kernel, stride, pad, dil, offset_scale, softmax)
    Ho, Wo = dcn_core_output_hw(p)
    K = p.kh * p.kw
    _cuda_tensor("offset", offset, x.dtype)
    _cuda_tensor("mask", mask, x.dtype)
    _cuda_tensor("weight", weight, x.dtype)
    if tuple(offset.shape) != (p.B, Ho, Wo, p.G, K, 2):
        raise ValueError(f"offset shape {tuple(offset.shape)} != {(p.B, Ho, Wo, p.G, K, 2)}")
    if tuple(mask.shape) != (p.B, Ho, Wo, p.G, K):
        raise ValueError(f"mask shape {tuple(mask.shape)} != {(p.B, Ho, Wo, p.G, K)}")
    if weight.dim() != 3 or tuple(weight.shape[1:]) != (K, p.G * p.C):
        raise ValueError(f"weight shape {tuple(weight.shape)} != (Cout, {K}, {p.G * p.C})")
    cout = int(weight.shape[0])
    if bias is not None:
        _cuda_tensor("bias", bias, x.dtype)
        if tuple(bias.shape) != (cout,):
            raise ValueError(f"bias shape {tuple(bias.shape)} != ({cout},)")
    if out is None:
        out = torch.empty((p.B, Ho, Wo, cout), dtype=x.dtype, device=x.device)
    else:
        _cuda_tensor("out", out, x.dtype)
        if tuple(out.shape) != (p.B, Ho, Wo, cout):
            raise ValueError("out has the wrong shape")
    check(lib().dcn_deform_conv_forward(ctypes.byref(p), cout, x.data_ptr(), offset.data_ptr(), mask.data_ptr(),
                                        weight.data_ptr(), None if bias is None else bias.data_ptr(),
                                        out.data_ptr(), _stream(x)))
    return out


def dcn_core_backward(x, offset, mask, grad_out, *, group: int, kernel=(3, 3), stride=(1, 1), pad=(1, 1),
                      dil=(1, 1), offset_scale: float = 1.0, softmax: bool = False, grad_x=None,
                      grad_offset=None, grad_mask=None):
    """(grad_x, grad_offset, grad_mask) of <grad_out, dcn_core_forward(...)>; see dcn_b200.h."""
    _cuda_tensor("x", x)
    p = core_params(x, group, kernel, stride, pad, dil, offset_scale, softmax)
    Ho, Wo = dcn_core_output_hw(p)
    K = p.kh * p.kw
    for n, t in (("offset", offset), ("mask", mask), ("grad_out", grad_out)):
        _cuda_tensor(n, t, x.dtype)
    if tuple(offset.shape) != (p.B, Ho, Wo, p.G, K, 2) or tuple(mask.shape) != (p.B, Ho, Wo, p.G, K):
        raise ValueError("offset/mask shape mismatch")
    if tuple(grad_out.shape) != (p.B, Ho, Wo, p.G * p.C):
        raise ValueError("grad_out shape mismatch")
    grad_x = torch.empty_like(x) if grad_x is None else _cuda_tensor("grad_x", grad_x, x.dtype)
    grad_offset = torch.empty_like(offset) if grad_offset is None else _cuda_tensor("grad_offset", grad_offset, x.dtype)
    grad_mask = torch.empty_like(mask) if grad_mask is None else _cuda_tensor("grad_mask", grad_mask, x.dtype)
    if grad_x.shape != x.shape or grad_offset.shape != offset.shape or grad_mask.shape != mask.shape:
        raise ValueError("gradient buffer shape mismatch")
    check(lib().dcn_core_backward(ctypes.byref(p), x.data_ptr(), offset.data_ptr(), mask.data_ptr(),
                                  grad_out.data_ptr(), grad_x.data_ptr(), grad_offset.data_ptr(),
                                  grad_mask.data_ptr(), _stream(x)))
    return grad_x, grad_offset, grad_mask


def agg_params(feat: torch.Tensor, weights: torch.Tensor) -> DaggParams:
    if feat.dtype not in _DTYPE_CODE:
        raise TypeError(f"unsupported dtype {feat.dtype}")
    B, rows, GC = feat.shape
    Bw, A, P, cams, S, G = weights.shape
    if Bw != B or GC % G:
        raise ValueError("feat/weights shape mismatch")
    return DaggParams(B, cams, S, rows, A, P, G, GC // G, _DTYPE_CODE[feat.dtype])


def _agg_inputs(feat, spatial_shape, scale_start_index, sampling_location, weights):
    _cuda_tensor("feat", feat)
    _cuda_tensor("weights", weights, feat.dtype)
    p = agg_params(feat, weights)
    _cuda_tensor("spatial_shape", spatial_shape, torch.int32)
    _cuda_tensor("scale_start_index", scale_start_index, torch.int32)
    _cuda_tensor("sampling_location", sampling_location, torch.float32)
    if tuple(spatial_shape.shape) != (p.num_cams, p.num_scales, 2):
        raise ValueError("spatial_shape must be [cams, scales, 2]")
    if tuple(scale_start_index.shape) != (p.num_cams, p.num_scales):
        raise ValueError("scale_start_index must be [cams, scales]")
    if tuple(sampling_location.shape) != (p.B, p.num_anchors, p.num_pts, p.num_cams, 2):
        raise ValueError("sampling_location must be [B, A, P, cams, 2]")
    return p


def deform_agg_forward(feat, spatial_shape, scale_start_index, sampling_location, weights, *, out=None):
    """out [B, A, G*C]: weighted multi-camera multi-scale bilinear aggregation; see dcn_b200.h."""
    p = _agg_inputs(feat, spatial_shape, scale_start_index, sampling_location, weights)
    if out is None:
        out = torch.empty((p.B, p.num_anchors, p.G * p.C), dtype=feat.dtype, device=feat.device)
    else:
        _cuda_tensor("out", out, feat.dtype)
    check(lib().deform_agg_forward(ctypes.byref(p), feat.data_ptr(), spatial_shape.data_ptr(),
                                   scale_start_index.data_ptr(), sampling_location.data_ptr(),
                                   weights.data_ptr(), out.data_ptr(), _stream(feat)))
    return out


def deform_agg_backward(feat, spatial_shape, scale_start_index, sampling_location, weights, grad_out, *,
                        grad_feat=None, grad_loc=None, grad_weights=None):
    """(grad_feat, grad_loc, grad_weights) of <grad_out, deform_agg_forward(...)>."""
    p = _agg_inputs(feat, spatial_shape, scale_start_index, sampling_location, weights)
    _cuda_tensor("grad_out", grad_out, feat.dtype)
    grad_feat = torch.empty_like(feat) if grad_feat is None else _cuda_tensor("grad_feat", grad_feat, feat.dtype)
    grad_loc = torch.empty_like(sampling_location) if grad_loc is None else \
        _cuda_tensor("grad_loc", grad_loc, torch.float32)
    grad_weights = torch.empty_like(weights) if grad_weights is None else \
        _cuda_tensor("grad_weights", grad_weights, feat.dtype)
    check(lib().deform_agg_backward(ctypes.byref(p), feat.data_ptr(), spatial_shape.data_ptr(),
                                    scale_start_index.data_ptr(), sampling_location.data_ptr(),
                                    weights.data_ptr(), grad_out.data_ptr(), grad_feat.data_ptr(),
                                    grad_loc.data_ptr(), grad_weights.data_ptr(), _stream(feat)))
    return grad_feat, grad_loc, grad_weights


def deform_roi_pool_forward(x, rois, offset, *, pooled=(7, 7), sampling: int = 2, spatial_scale: float = 1.0,
                            gamma: float = 0.1, out=None):
    """out [N, PH, PW, C]: deformable RoI pooling of x [B, H, W, C]; see dcn_b200.h."""
    _cuda_tensor("x", x)
    if x.dtype not in _DTYPE_CODE:
        raise TypeError(f"unsupported dtype {x.dtype}")
    _cuda_tensor("rois", rois, torch.float32)
    _cuda_tensor("offset", offset, torch.float32)
    B, H, W, C = x.shape
    PH, PW = _pair(pooled)
    N = rois.shape[0]
    if tuple(rois.shape) != (N, 5) or tuple(offset.shape) != (N, PH, PW, 2):
        raise ValueError("rois must be [N, 5] and offset [N, PH, PW, 2]")
    p = DroiParams(B, H, W, C, N, PH, PW, int(sampling), float(spatial_scale), float(gamma), _DTYPE_CODE[x.dtype])
    if out is None:
        out = torch.empty((N, PH, PW, C), dtype=x.dtype, device=x.device)
    else:
        _cuda_tensor("out", out, x.dtype)
    check(lib().deform_roi_pool_forward(ctypes.byref(p), x.data_ptr(), rois.data_ptr(), offset.data_ptr(),
                                        out.data_ptr(), _stream(x)))
    return out
