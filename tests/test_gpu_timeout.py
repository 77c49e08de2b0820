"""The bounded wait gives up: a kernel waits on an mbarrier that nothing completes, with a 5 ms
limit, through the same wait routine the pipelined kernels use. The device error word must then
read BRA_ERR_TIMEOUT (once: reading clears it), and the context must still run the forward pass."""
import pytest
import torch

import bi_level_routing_b200 as bra
from bi_level_routing_b200 import api
from bi_level_routing_b200.workloads import WORKLOADS
from parity import make

pytestmark = pytest.mark.gpu


def test_wait_times_out_and_the_context_stays_usable():
    L = api.lib()
    assert bra.check_device_error() == 0
    stream = torch.cuda.current_stream().cuda_stream
    assert L.bra_selftest_wait_timeout(5000, stream) == 0
    assert bra.check_device_error() == 5  # BRA_ERR_TIMEOUT
    assert bra.check_device_error() == 0  # read once, then cleared
    assert L.bra_selftest_wait_timeout(0, stream) == 1  # a limit of 0 is rejected
    w = WORKLOADS["stage2"].with_(B=2)
    _, (q, k, v) = make(w)
    out, idx = bra.forward(q, k, v, w.n_win, w.topk, w.heads)
    torch.cuda.synchronize()
    assert bra.check_device_error() == 0 and torch.isfinite(out.float()).all()
