"""dcn_core_forward_proj_noalloc, the projection entry point for callers that
cannot allocate device memory (a plugin whose host framework owns the GPU's
memory, a loop that cannot afford cudaMalloc's device-wide synchronisation):
it runs the workspace route with the library's fixed 16 MiB scratch array.

Called through the C ABI with ctypes and compared with dcn_core_forward_proj
(the existing entry point, workspace route) on two calls in a row with
different inputs, so the second call runs on scratch that still holds the
first call's core output.  This file is collected last on purpose."""
import ctypes

import pytest
import torch

import synthetic_inputs as si
from parity import assert_close_fwd

pytestmark = pytest.mark.gpu


def _noalloc(lib, shape, t, out):
    from deformable_convolution_sampling_dcn_b200 import _binding as B

    p = B.core_params(t["x"], shape.G, (shape.kh, shape.kw), (shape.stride_h, shape.stride_w),
                      (shape.pad_h, shape.pad_w), (shape.dil_h, shape.dil_w), shape.offset_scale, shape.softmax)
    return lib.dcn_core_forward_proj_noalloc(ctypes.byref(p), int(t["weight"].shape[0]), t["x"].data_ptr(),
                                             t["offset"].data_ptr(), t["mask"].data_ptr(), t["weight"].data_ptr(),
                                             t["bias"].data_ptr(), out.data_ptr(),
                                             torch.cuda.current_stream().cuda_stream)


def test_noalloc_matches_workspace_route_twice(cuda_dev):
    import deformable_convolution_sampling_dcn_b200 as d

    lib = d._binding.lib()
    cases = []
    shape, inp = si.workload_proj()  # DCNv4 P4, 13.1 MB of core output: fits the 16 MiB scratch
    cases.append((shape, inp))
    small = si.CoreShape(B=2, H=11, W=9, G=8, C=32, softmax=True, dtype="bf16")
    inp2 = si.core_inputs(small, 77, offset_std=2.5, oob_fraction=0.03)
    inp2.update(si.proj_inputs(small.G * small.C, 136, "bf16", 78))
    cases.append((small, inp2))
    for shape, inp in cases:
        t = {k: v.to(cuda_dev) for k, v in inp.items()}
        cout = t["weight"].shape[0]
        out = torch.full((shape.B, shape.Ho, shape.Wo, cout), float("nan"), dtype=t["x"].dtype, device=cuda_dev)
        assert _noalloc(lib, shape, t, out) == 0, d._binding.lib().dcn_last_error_detail()
        ref = d.dcn_core_forward_proj(t["x"], t["offset"], t["mask"], t["weight"], t["bias"], group=shape.G,
                                      kernel=(shape.kh, shape.kw), softmax=shape.softmax)
        torch.cuda.synchronize()
        assert d._binding.take_device_error() == 0
        assert_close_fwd(out, ref.double().cpu().numpy(), "no-alloc vs workspace route")


def test_noalloc_rejects_problems_beyond_its_scratch(cuda_dev):
    """A core output larger than the fixed scratch is refused on the host with
    a detail that names both sizes; nothing is launched."""
    import deformable_convolution_sampling_dcn_b200 as d
    from deformable_convolution_sampling_dcn_b200 import _binding as B

    lib = d._binding.lib()
    big = B.DcnParams(B=16, H=40, W=40, G=16, C=32, kh=3, kw=3, stride_h=1, stride_w=1, pad_h=1, pad_w=1,
                      dil_h=1, dil_w=1, offset_scale=1.0, mask_mode=0, dtype=B.DCN_F16)  # 26.2 MB of core output
    st = lib.dcn_core_forward_proj_noalloc(ctypes.byref(big), 512, 16, 16, 16, 16, None, 16,
                                           torch.cuda.current_stream().cuda_stream)
    assert st == B.DCN_ERR_UNSUPPORTED
    detail = lib.dcn_last_error_detail().decode()
    assert "26214400" in detail and str(16 * 1024 * 1024) in detail
