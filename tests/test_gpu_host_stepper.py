"""Host-fed decode steps (runner.HostStepper) against device-resident decode.

The stepper packs a step's inputs into one pinned host buffer, uploads it in one
copy, runs the batch's kernels on views of the uploaded bytes and reads the output
back; with two buffers the copies of neighbouring steps overlap the kernels.  The
kernels and their inputs are the same as those of a device-resident call, so every
output must match that call bit for bit, whatever the buffer rotation, and whether
the kernels are launched one by one or replayed from a captured CUDA graph.
"""
import numpy as np
import pytest
import torch

from paged_kv_cache_363_b200 import workloads as W
from pa_testlib import bits

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def runner():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from paged_kv_cache_363_b200 import runner as _r
    return _r


def _small(wid, seed):
    if wid == 2:
        return W.make_workload(2, seed=seed, num_seqs=12, num_blocks=2000)
    if wid == 3:
        return W.make_workload(3, seed=seed, num_seqs=40, num_blocks=4000)
    if wid == 4:
        return W.make_workload(4, seed=seed, num_prompts=4, num_blocks=800)
    return W.make_workload(wid, seed=seed)


@pytest.mark.parametrize("wid", [1, 2, 3, 4])
@pytest.mark.parametrize("depth", [1, 2, 3])
@pytest.mark.parametrize("graph", [False, True])
def test_host_fed_steps_match_device_decode(runner, wid, depth, graph):
    wl = _small(wid, seed=wid + depth)
    batch = runner.make_batch(wl, "cuda")
    st = runner.HostStepper(batch, depth=depth, graph=graph)
    assert st.h2d_bytes >= sum(getattr(batch, n).numel() * getattr(batch, n).element_size()
                               for n in ("q", "new_k", "new_v", "slot_mapping", "block_tables", "context_lens"))
    assert st.d2h_bytes == batch.out.numel() * batch.out.element_size()
    g = torch.Generator().manual_seed(100 + wid)
    qs = [torch.randn(batch.q.shape, generator=g).to(batch.q.dtype) for _ in range(2 * depth + 1)]
    last = {}                                      # buffer -> the latest step queued on it
    for k, q in enumerate(qs):
        i = k % depth
        st.host_inputs(i)["q"].copy_(q)
        assert st.submit() == i
        last[i] = k
    for i, k in last.items():
        got = st.output(i).clone()
        ref = torch.empty_like(batch.out)
        batch.q.copy_(qs[k].cuda())
        batch.append()
        batch.decode(out=ref)
        torch.cuda.synchronize()
        assert np.array_equal(bits(got), bits(ref.cpu())), "step %d (buffer %d) differs" % (k, i)
    from paged_kv_cache_363_b200 import pa
    assert pa.pa_device_status() == 0


@pytest.mark.parametrize("graph", [False, True])
def test_each_step_reads_back_its_own_output(runner, graph):
    # output of step k is read before step k + depth reuses the buffer
    wl = _small(3, seed=9)
    batch = runner.make_batch(wl, "cuda")
    depth = 2
    st = runner.HostStepper(batch, depth=depth, graph=graph)
    g = torch.Generator().manual_seed(7)
    qs = [torch.randn(batch.q.shape, generator=g).to(batch.q.dtype) for _ in range(6)]
    got = []
    for k, q in enumerate(qs):
        i = k % depth
        if k >= depth:
            got.append(st.output(i).clone())       # step k - depth, finished before the refill
        st.host_inputs(i)["q"].copy_(q)
        assert st.submit() == i
    for k in range(len(qs) - depth, len(qs)):
        got.append(st.output(k % depth).clone())
    for k, q in enumerate(qs):
        ref = torch.empty_like(batch.out)
        batch.q.copy_(q.cuda())
        batch.decode(out=ref)
        torch.cuda.synchronize()
        assert np.array_equal(bits(got[k]), bits(ref.cpu())), "step %d" % k
