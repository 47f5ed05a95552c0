"""Failure detection on the GPU without a fault: a bounded device wait is made to run
out (an mbarrier that nothing arrives at), raises PA_DEV_WAIT_TIMEOUT, and the context
stays usable for the next calls."""
import numpy as np
import pytest
import torch

from pa_testlib import TOL, max_abs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pa():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from paged_kv_cache_363_b200 import pa as _pa
    return _pa


def test_a_stalled_wait_gives_up_reports_and_leaves_the_context_usable(pa):
    assert pa.pa_device_status() == 0
    waited = pa.pa_selftest_bounded_wait()
    assert 2.0e9 <= waited < 4.0e9                      # the kernels' 2 s limit, on the device clock
    assert pa.pa_device_status() == pa.PA_DEV_WAIT_TIMEOUT
    assert pa.pa_device_status() == 0                   # reading clears it
    # the context still runs the library's kernels correctly
    from paged_kv_cache_363_b200 import runner, workloads as W
    from oracle import oracle
    from pa_testlib import oracle_decode_side
    wl = W.make_workload(1, seed=0)
    vals = W.decode_values(wl, "cpu")
    ref = oracle_decode_side(wl, vals)
    out = runner.DecodeBatch(wl, "cuda", values=vals).step()
    torch.cuda.synchronize()
    assert max_abs(out.cpu().numpy(), ref["out"]) <= TOL["f32"]
    assert pa.pa_device_status() == 0
