"""The bounded-wait error path on the GPU, made to run out without a fault:
a wait on a barrier that nothing arrives on gives up after its limit, the
device error word reports it, and the context stays usable."""
import pytest
import torch

import oracle
import synthetic_inputs as si
from parity import assert_close_fwd

pytestmark = pytest.mark.gpu


def test_bounded_wait_runs_out_and_reports(cuda_dev):
    import deformable_convolution_sampling_dcn_b200 as d

    assert d._binding.take_device_error() == 0
    d._binding.selftest_bounded_wait(2000)  # 2 ms
    torch.cuda.synchronize()
    assert d._binding.take_device_error() == 1
    assert d._binding.take_device_error() == 0  # read clears it
    # the context is still usable: a normal call runs and matches the oracle
    shape, inp = si.workload_core("dcnv3_tiny")
    out = d.dcn_core_forward(*(inp[k].to(cuda_dev) for k in ("x", "offset", "mask")), group=shape.G, softmax=True)
    torch.cuda.synchronize()
    assert_close_fwd(out, oracle.dcn_forward(inp["x"], inp["offset"], inp["mask"], G=shape.G, softmax=True))
    assert d._binding.take_device_error() == 0


def test_selftest_rejects_bad_limit(cuda_dev):
    import deformable_convolution_sampling_dcn_b200 as d

    with pytest.raises(d.DcnError):
        d._binding.selftest_bounded_wait(0)


def test_error_word_seen_from_a_non_blocking_stream(cuda_dev):
    """A kernel that gives up on a non-blocking stream (torch's side streams are
    such) must still be reported: reading the word waits for the whole device,
    not only for the legacy default stream."""
    import deformable_convolution_sampling_dcn_b200 as d

    assert d._binding.take_device_error() == 0
    s = torch.cuda.Stream()  # created cudaStreamNonBlocking by torch
    with torch.cuda.stream(s):
        d._binding.selftest_bounded_wait(20000)  # 20 ms, no host synchronisation after it
    assert d._binding.take_device_error() == 1
    assert d._binding.take_device_error() == 0
