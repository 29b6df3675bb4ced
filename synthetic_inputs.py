"""Seeded synthetic inputs for the deformable sampling-aggregation core.

This module is shared by the tests, the benchmark and the smoke check. It
draws random numbers and rounds them once to the storage dtype; it holds none
of the operator's arithmetic (no sampling positions, no interpolation, no
modulation). Both the fp64 oracle and the CUDA library are fed the same
tensors made here.

Every generator uses numpy's PCG64 with a fixed seed and draws in the order
x, offset, mask (or weights), grad_out. Values are returned as CPU torch
tensors in the storage dtype; an fp16/bf16 tensor holds the already-rounded
values, so both sides read bit-identical inputs.

Workload shapes stand in for the feature maps the source pages run on
(YOLO P3/P4/P5 maps at 640 input, Sparse4D's six-camera four-scale features);
the datasets behind those pages are not used.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, List, Optional, Tuple

import numpy as np
import torch

DTYPES = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}


@dataclasses.dataclass(frozen=True)
class CoreShape:
    """Shape and hyper-parameters of one deformable-core problem."""

    B: int
    H: int
    W: int
    G: int
    C: int
    kh: int = 3
    kw: int = 3
    stride_h: int = 1
    stride_w: int = 1
    pad_h: int = 1
    pad_w: int = 1
    dil_h: int = 1
    dil_w: int = 1
    offset_scale: float = 1.0
    softmax: bool = False
    dtype: str = "f32"

    @property
    def K(self) -> int:
        return self.kh * self.kw

    @property
    def Ho(self) -> int:
        return (self.H + 2 * self.pad_h - (self.dil_h * (self.kh - 1) + 1)) // self.stride_h + 1

    @property
    def Wo(self) -> int:
        return (self.W + 2 * self.pad_w - (self.dil_w * (self.kw - 1) + 1)) // self.stride_w + 1

    @property
    def samples(self) -> int:
        """Taps per call: one per (b, output pixel, group, kernel point)."""
        return self.B * self.Ho * self.Wo * self.G * self.K

    def compulsory_bytes(self, backward: bool = False) -> int:
        """x + offset + mask + out (forward) in storage bytes.

        Backward reads x, offset, mask, grad_out and writes grad_x,
        grad_offset, grad_mask.
        """
        e = torch.finfo(DTYPES[self.dtype]).bits // 8
        nx = self.B * self.H * self.W * self.G * self.C
        no = self.B * self.Ho * self.Wo * self.G * self.C
        noff = self.B * self.Ho * self.Wo * self.G * self.K * 2
        nm = self.B * self.Ho * self.Wo * self.G * self.K
        if not backward:
            return e * (nx + noff + nm + no)
        return e * (nx + noff + nm + no) + e * (nx + noff + nm)


@dataclasses.dataclass(frozen=True)
class AggShape:
    """Shape of one multi-camera multi-scale aggregation problem."""

    B: int
    num_cams: int
    scales: Tuple[Tuple[int, int], ...]  # (H_s, W_s) per scale, identical for every camera
    num_anchors: int
    num_pts: int
    G: int
    C: int
    dtype: str = "f32"

    @property
    def num_scales(self) -> int:
        return len(self.scales)

    @property
    def hw_sum(self) -> int:
        return sum(h * w for h, w in self.scales)

    @property
    def num_rows(self) -> int:
        return self.num_cams * self.hw_sum

    @property
    def samples(self) -> int:
        return self.B * self.num_anchors * self.num_pts * self.num_cams * self.num_scales * self.G

    def compulsory_bytes(self) -> int:
        e = torch.finfo(DTYPES[self.dtype]).bits // 8
        feat = self.B * self.num_rows * self.G * self.C * e
        loc = self.B * self.num_anchors * self.num_pts * self.num_cams * 2 * 4
        w = self.samples * e
        out = self.B * self.num_anchors * self.G * self.C * e
        return feat + loc + w + out


# The five workloads: a tiny DCNv3 case, the DCNv4 case at a YOLO P4 map
# (640 input, 512 channels), a high-resolution DCNv3 case at a P3 map with a
# dilated variant, the Sparse4D six-camera aggregation, and the DCNv4
# backward at the P4 shape.
DCNV3_TINY = CoreShape(B=1, H=16, W=16, G=4, C=8, softmax=True, dtype="f32")
DCNV4_P4 = CoreShape(B=8, H=40, W=40, G=16, C=32, softmax=False, dtype="f16")
DCNV3_P3 = CoreShape(B=16, H=80, W=80, G=8, C=32, softmax=True, dtype="bf16")
DCNV3_P3_DIL2 = dataclasses.replace(DCNV3_P3, pad_h=2, pad_w=2, dil_h=2, dil_w=2)
DCNV4_P4_BWD = dataclasses.replace(DCNV4_P4, dtype="f32")
SPARSE4D = AggShape(B=1, num_cams=6, scales=((64, 176), (32, 88), (16, 44), (8, 22)),
                    num_anchors=900, num_pts=13, G=8, C=32, dtype="f32")

SEEDS = {"dcnv3_tiny": 0, "dcnv4_p4": 1, "dcnv3_p3": 2, "sparse4d": 3, "dcnv4_p4_bwd": 4}


def _round(a: np.ndarray, dtype: str) -> torch.Tensor:
    """Round float64 draws once, nearest-even, to the storage dtype."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float64))
    return t.to(DTYPES[dtype]).contiguous()


def core_inputs(shape: CoreShape, seed: int, *, x_dist: str = "normal", offset_std: float = 3.0,
                mask_dist: str = "normal", oob_fraction: float = 0.0,
                with_grad_out: bool = False) -> Dict[str, torch.Tensor]:
    """Draw x [B,H,W,G*C], offset [B,Ho,Wo,G,K,2] (dx, dy), mask [B,Ho,Wo,G,K].

    x_dist: "normal" (N(0,1)) or "uniform" (U[-1,1]).
    offset_std: standard deviation of the offsets, in pixels.
    mask_dist: "normal" draws N(0,1) values; in softmax mode these are the
      logits the operator normalises, in raw mode the modulation itself.
    oob_fraction: fraction of (pixel, group, point) whose offset is replaced
      by one that lands fully outside the map on both axes: the magnitude is
      (extent of the map + the largest kernel reach + 2 + U[0,4]) pixels with
      a random sign per axis, which is out of range from every base point.
    with_grad_out: also draw grad_out [B,Ho,Wo,G*C] ~ N(0,1).
    """
    s = shape
    rng = np.random.Generator(np.random.PCG64(seed))
    nx = (s.B, s.H, s.W, s.G * s.C)
    if x_dist == "normal":
        x = rng.standard_normal(nx)
    elif x_dist == "uniform":
        x = rng.uniform(-1.0, 1.0, nx)
    else:
        raise ValueError(x_dist)
    noff = (s.B, s.Ho, s.Wo, s.G, s.K, 2)
    off = rng.standard_normal(noff) * offset_std
    if oob_fraction > 0:
        pick = rng.random(noff[:-1]) < oob_fraction
        n = int(pick.sum())
        reach_y = s.H + 2 * (s.pad_h + s.dil_h * s.kh) + 2
        reach_x = s.W + 2 * (s.pad_w + s.dil_w * s.kw) + 2
        sign = np.where(rng.random((n, 2)) < 0.5, -1.0, 1.0)
        mag = rng.uniform(0.0, 4.0, (n, 2)) + np.array([reach_x, reach_y], dtype=np.float64)
        off[pick] = sign * mag
    nm = (s.B, s.Ho, s.Wo, s.G, s.K)
    if mask_dist == "normal":
        m = rng.standard_normal(nm)
    elif mask_dist == "uniform01":
        m = rng.random(nm)
    else:
        raise ValueError(mask_dist)
    out = {"x": _round(x, s.dtype), "offset": _round(off, s.dtype), "mask": _round(m, s.dtype)}
    if with_grad_out:
        go = rng.standard_normal((s.B, s.Ho, s.Wo, s.G * s.C))
        out["grad_out"] = _round(go, s.dtype)
    return out


def workload_core(name: str) -> Tuple[CoreShape, Dict[str, torch.Tensor]]:
    """The named core workloads with their recipes."""
    if name == "dcnv3_tiny":
        return DCNV3_TINY, core_inputs(DCNV3_TINY, SEEDS[name], x_dist="uniform", offset_std=2.0)
    if name == "dcnv4_p4":
        return DCNV4_P4, core_inputs(DCNV4_P4, SEEDS[name], offset_std=3.0)
    if name == "dcnv3_p3":
        return DCNV3_P3, core_inputs(DCNV3_P3, SEEDS[name], offset_std=4.0, oob_fraction=0.05)
    if name == "dcnv3_p3_dil2":
        return DCNV3_P3_DIL2, core_inputs(DCNV3_P3_DIL2, SEEDS["dcnv3_p3"], offset_std=4.0,
                                          oob_fraction=0.05)
    if name == "dcnv4_p4_bwd":
        return DCNV4_P4_BWD, core_inputs(DCNV4_P4_BWD, SEEDS[name], offset_std=3.0,
                                         with_grad_out=True)
    if name == "dcnv3_p3_bwd":
        # the DCNv3 P3 inputs (same seed and draws) followed by grad_out ~ N(0,1)
        return DCNV3_P3, core_inputs(DCNV3_P3, SEEDS["dcnv3_p3"], offset_std=4.0, oob_fraction=0.05,
                                     with_grad_out=True)
    raise KeyError(name)


def agg_tables(shape: AggShape) -> Tuple[torch.Tensor, torch.Tensor]:
    """spatial_shape [cams, scales, 2] (H, W) and scale_start_index [cams, scales].

    Rows are laid out camera-major: each camera's maps are flattened scale
    after scale ([N, C, H, W] -> [N*H*W, C] per scale, concatenated), the
    layout of the Sparse4D feature flattening.
    """
    ss = torch.tensor([[list(hw) for hw in shape.scales]] * shape.num_cams, dtype=torch.int32)
    start = []
    row = 0
    for _cam in range(shape.num_cams):
        r = []
        for h, w in shape.scales:
            r.append(row)
            row += h * w
        start.append(r)
    return ss, torch.tensor(start, dtype=torch.int32)


def agg_inputs(shape: AggShape, seed: int, *, with_grad_out: bool = False,
               loc_lo: float = 0.0, loc_hi: float = 1.0) -> Dict[str, torch.Tensor]:
    """feat [B,rows,G*C] ~ N(0,1); loc [B,A,P,cams,2] ~ U[lo,hi]; weights
    [B,A,P,cams,scales,G] = softmax over (P, cams, scales) of N(0,1) logits
    per (anchor, group), normalised here because the caller supplies
    normalised weights to the operator."""
    s = shape
    rng = np.random.Generator(np.random.PCG64(seed))
    feat = rng.standard_normal((s.B, s.num_rows, s.G * s.C))
    loc = rng.uniform(loc_lo, loc_hi, (s.B, s.num_anchors, s.num_pts, s.num_cams, 2))
    logits = rng.standard_normal((s.B, s.num_anchors, s.num_pts, s.num_cams, s.num_scales, s.G))
    lg = np.moveaxis(logits, -1, 2).reshape(s.B, s.num_anchors, s.G, -1)
    e = np.exp(lg - lg.max(axis=-1, keepdims=True))
    w = e / e.sum(axis=-1, keepdims=True)
    w = np.moveaxis(w.reshape(s.B, s.num_anchors, s.G, s.num_pts, s.num_cams, s.num_scales), 2, -1)
    ss, start = agg_tables(s)
    out = {"feat": _round(feat, s.dtype), "spatial_shape": ss, "scale_start_index": start,
           "sampling_location": torch.from_numpy(loc.astype(np.float32)),
           "weights": _round(w, s.dtype)}
    if with_grad_out:
        out["grad_out"] = _round(rng.standard_normal((s.B, s.num_anchors, s.G * s.C)), s.dtype)
    return out



@dataclasses.dataclass(frozen=True)
class RoiShape:
    """Shape of one deformable RoI pooling problem."""

    B: int
    H: int
    W: int
    C: int
    N: int
    PH: int = 7
    PW: int = 7
    S: int = 2
    spatial_scale: float = 1.0 / 16
    gamma: float = 0.1
    dtype: str = "f32"

    @property
    def samples(self) -> int:
        return self.N * self.PH * self.PW * self.S * self.S

    def compulsory_bytes(self) -> int:
        e = torch.finfo(DTYPES[self.dtype]).bits // 8
        return (self.B * self.H * self.W * self.C * e + self.N * 5 * 4 + self.N * self.PH * self.PW * 2 * 4
                + self.N * self.PH * self.PW * self.C * e)


# Deformable RoI pooling on a stride-16 feature map of a 1024 x 1024 image:
# 512 regions, 7 x 7 bins, 2 x 2 samples per bin, 256 channels.
ROI_POOL = RoiShape(B=2, H=64, W=64, C=256, N=512)
SEEDS["roi_pool"] = 5


def roi_inputs(shape: RoiShape, seed: int, *, offset_std: float = 1.0,
               min_size: float = 16.0) -> Dict[str, torch.Tensor]:
    """x [B,H,W,C] ~ N(0,1); rois [N,5] with boxes uniform inside the image
    (W/spatial_scale x H/spatial_scale, at least min_size wide); offset
    [N,PH,PW,2] ~ N(0, offset_std) (normalised units)."""
    s = shape
    rng = np.random.Generator(np.random.PCG64(seed))
    x = rng.standard_normal((s.B, s.H, s.W, s.C))
    img_w, img_h = s.W / s.spatial_scale, s.H / s.spatial_scale
    b = rng.integers(0, s.B, s.N)
    x1 = rng.uniform(0, img_w - min_size, s.N)
    y1 = rng.uniform(0, img_h - min_size, s.N)
    x2 = np.minimum(x1 + min_size + rng.exponential(img_w / 6, s.N), img_w)
    y2 = np.minimum(y1 + min_size + rng.exponential(img_h / 6, s.N), img_h)
    rois = np.stack([b, x1, y1, x2, y2], axis=1).astype(np.float32)
    off = rng.standard_normal((s.N, s.PH, s.PW, 2)) * offset_std
    return {"x": _round(x, s.dtype), "rois": torch.from_numpy(rois),
            "offset": torch.from_numpy(off.astype(np.float32))}


# The DCNv4 module's pointwise projection after the core (a 1x1 convolution
# with bias, channels -> channels): at the P4 shape, G*C = 512 -> 512.
PROJ_COUT_P4 = 512
SEEDS["dcnv4_p4_proj"] = 6


def proj_inputs(cin: int, cout: int, dtype: str, seed: int) -> Dict[str, torch.Tensor]:
    """weight [cout, cin] ~ N(0, 1/cin) (unit-variance outputs for unit-variance
    inputs) and bias [cout] ~ N(0, 0.1^2), rounded once to the storage dtype."""
    rng = np.random.Generator(np.random.PCG64(seed))
    w = rng.standard_normal((cout, cin)) / np.sqrt(cin)
    b = rng.standard_normal(cout) * 0.1
    return {"weight": _round(w, dtype), "bias": _round(b, dtype)}


def workload_proj() -> Tuple[CoreShape, Dict[str, torch.Tensor]]:
    """DCNv4 P4 core inputs plus its 512 -> 512 projection."""
    shape, inp = workload_core("dcnv4_p4")
    inp.update(proj_inputs(shape.G * shape.C, PROJ_COUT_P4, shape.dtype, SEEDS["dcnv4_p4_proj"]))
    return shape, inp


def deform_conv_weights(K: int, cin: int, cout: int, dtype: str, seed: int) -> Dict[str, torch.Tensor]:
    """weight [cout, K, cin] ~ N(0, 1/(K*cin)) (a Conv2d weight permuted to
    point-major) and bias [cout] ~ N(0, 0.1^2), rounded once to the storage dtype."""
    rng = np.random.Generator(np.random.PCG64(seed))
    w = rng.standard_normal((cout, K, cin)) / np.sqrt(K * cin)
    b = rng.standard_normal(cout) * 0.1
    return {"weight": _round(w, dtype), "bias": _round(b, dtype)}
