"""Failure detection on the GPU without a fault: a device wait that runs out.

Every mbarrier wait of the tcgen05 kernels is bounded (2 s); on expiry the
kernel records MOE_ERR_TIMEOUT in the caller's status word and returns.  The
test drives that wait on a barrier nothing ever arrives at, then checks that
the status says so and that the context still runs the layer correctly.
"""
import time

import pytest
import torch

import mixture_experts_layer_53_b200 as M
import workloads as W
from parity import check_forward, gpu_forward

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    from mixture_experts_layer_53_b200 import build
    build.build()
    M.library()
    assert torch.cuda.is_available()


def test_device_wait_times_out_and_the_context_survives():
    t0 = time.time()
    status = M.moe_selftest_wait_timeout()
    elapsed = time.time() - t0
    assert status == 5, f"status {status}, expected MOE_ERR_TIMEOUT"
    assert 1.5 < elapsed < 60.0, f"the wait gave up after {elapsed:.2f} s"
    wl = W.WORKLOADS["mixtral"].scaled(N=200, d_model=256, d_ff=384)
    inp = W.make_inputs(wl, "cuda")
    check_forward(wl, inp, gpu_forward(wl, inp))
