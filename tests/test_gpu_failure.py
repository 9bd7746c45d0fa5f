"""Device failure path, without a GPU fault: a bounded mbarrier wait that can
never complete (nothing arrives on the barrier) runs out, raises the library's
device flag, and leaves the context usable.

The kernel waits through the same bounded wait every tensor-core producer,
MMA issuer and epilogue uses; the limit is shortened to 100 ms for the test."""
import pytest
import torch

from sparse_mixture_experts_sigmoid_b200 import binding as B
from sparse_mixture_experts_sigmoid_b200 import synth
from sparse_mixture_experts_sigmoid_b200.workloads import Workload


@pytest.mark.gpu
def test_bounded_wait_runs_out_and_context_survives():
    torch.cuda.set_device(0)
    assert B.device_status() == B.MOE_OK          # start from a clear flag
    assert B.selftest_wait_timeout(100) == B.MOE_OK
    assert B.device_status() == 5                 # MOE_ERR_DEVICE_TIMEOUT
    assert B.device_status() == B.MOE_OK          # reading cleared it
    # the stream and the library still work
    w = Workload("after_timeout", T=256, d=128, E=8, h=128, k=2, seed=21)
    layer = synth.make_layer(w, "cuda")
    y = B.forward_layer(B.config_of(w), layer)
    torch.cuda.synchronize()
    assert B.device_status() == B.MOE_OK
    assert torch.isfinite(y.float()).all()


def test_selftest_rejects_bad_limits():
    assert B.lib().moe_selftest_wait_timeout(0, None) == 1
    assert B.lib().moe_selftest_wait_timeout(10001, None) == 1
