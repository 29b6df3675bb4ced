"""B200 (sm_100a) modulated deformable sampling-aggregation core.

Thin Python front end of libdcn_b200.so (C ABI in include/dcn_b200.h):

    dcn_core_forward / dcn_core_backward     DCNv2/v3/v4 sampling core
    dcn_core_forward_proj                    the core fused with its 1x1 projection (DCNv4 module)
    dcn_deform_conv_forward                  modulated deformable convolution, weight per point (DCNv2)
    deform_agg_forward / deform_agg_backward Sparse4D multi-camera aggregation
    deform_roi_pool_forward                  deformable RoI pooling
    DCNCoreFunction, DeformAggFunction       autograd wrappers over the above
    shard_range                              batch split for one-process-per-GPU runs

PyTorch only allocates device memory and supplies the current stream; every
arithmetic step runs in the library's CUDA kernels.
"""
from __future__ import annotations

from typing import Tuple

import torch

from ._binding import (ABI_VERSION, EXPORTS, DaggParams, DcnError, DcnParams, DroiParams, core_params,
                       dcn_core_backward, dcn_core_forward, dcn_core_forward_proj, dcn_core_output_hw,
                       dcn_deform_conv_forward,
                       deform_agg_backward,
                       deform_agg_forward, deform_roi_pool_forward, lib)

__all__ = ["dcn_core_forward", "dcn_core_forward_proj", "dcn_deform_conv_forward", "dcn_core_backward", "dcn_core_output_hw", "deform_agg_forward",
           "deform_agg_backward", "deform_roi_pool_forward", "DroiParams", "DCNCoreFunction", "DeformAggFunction", "shard_range", "lib", "DcnError",
           "DcnParams", "DaggParams", "core_params", "EXPORTS", "ABI_VERSION"]


class DCNCoreFunction(torch.autograd.Function):
    """autograd over dcn_core_forward/backward (x, offset, mask all differentiable)."""

    @staticmethod
    def forward(ctx, x, offset, mask, group: int, kernel=(3, 3), stride=(1, 1), pad=(1, 1), dil=(1, 1),
                offset_scale: float = 1.0, softmax: bool = False):
        ctx.cfg = dict(group=group, kernel=kernel, stride=stride, pad=pad, dil=dil, offset_scale=offset_scale,
                       softmax=softmax)
        ctx.save_for_backward(x, offset, mask)
        return dcn_core_forward(x, offset, mask, **ctx.cfg)

    @staticmethod
    @torch.autograd.function.once_differentiable
    def backward(ctx, grad_out):
        x, offset, mask = ctx.saved_tensors
        gx, goff, gm = dcn_core_backward(x, offset, mask, grad_out.contiguous(), **ctx.cfg)
        return gx, goff, gm, None, None, None, None, None, None, None


class DeformAggFunction(torch.autograd.Function):
    """autograd over deform_agg_forward/backward (feat, locations, weights differentiable)."""

    @staticmethod
    def forward(ctx, feat, spatial_shape, scale_start_index, sampling_location, weights):
        ctx.save_for_backward(feat, spatial_shape, scale_start_index, sampling_location, weights)
        return deform_agg_forward(feat, spatial_shape, scale_start_index, sampling_location, weights)

    @staticmethod
    @torch.autograd.function.once_differentiable
    def backward(ctx, grad_out):
        feat, ss, st, loc, w = ctx.saved_tensors
        gf, gl, gw = deform_agg_backward(feat, ss, st, loc, w, grad_out.contiguous())
        return gf, None, None, gl, gw


def shard_range(total: int, world: int, rank: int) -> Tuple[int, int]:
    """Contiguous [lo, hi) share of `total` independent batch images for
    `rank` of `world` processes.  Images are independent in the forward and
    the backward (grad_x of image b only receives from image b), so a batch
    split needs no exchange between ranks."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("bad rank/world")
    base, extra = divmod(int(total), int(world))
    lo = rank * base + min(rank, extra)
    return lo, lo + base + (1 if rank < extra else 0)
