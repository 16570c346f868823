"""The split-K workspace grows stream-ordered, without synchronising the device.

The regular entry points keep one split-K / stream-K workspace per (device,
stream).  When a call needs more than its stream's workspace holds, the old
buffer is released with cudaFreeAsync and a new one taken with
cudaMallocAsync, both on the call's stream.  So a growing call must return
while unrelated work on another stream is still running, and its result must
still match the oracle.
"""
import time

import numpy as np
import pytest
import torch

import oracle
import workloads
import fp8_block_scaled_bsgemm_b200 as bsg
from gpu_util import check_close, gpu_as_f64, to_device

pytestmark = pytest.mark.gpu


def _ref(p):
    ref, _ = oracle.bsgemm(p.layout, p.a, p.b, p.sa, p.sb, p.M, p.N, p.K, p.gran)
    return ref


def test_workspace_growth_does_not_wait_for_other_streams():
    torch.cuda.set_device(0)
    num_sms = torch.cuda.get_device_properties(0).multi_processor_count
    # two stream-K plans; the second needs a larger workspace than the first
    small = workloads.make_problem(64, 2048, 4096, seed=11, name="ws small")
    large = workloads.make_problem(128, 4096, 8192, seed=12, name="ws large")
    for p in (small, large):
        pl = bsg.make_plan(p.M, p.N, p.K, p.gran, p.layout, num_sms)
        assert pl["sk_ctas"] > 0 or pl["splits"] > 1, pl
    assert (bsg.scratch_bytes(bsg.make_plan(large.M, large.N, large.K, 128, "nt", num_sms)) >
            1.25 * bsg.scratch_bytes(bsg.make_plan(small.M, small.N, small.K, 128, "nt", num_sms)))
    ds, dl = to_device(small), to_device(large)
    torch.cuda.synchronize()

    blocker, s1, s2 = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    with torch.cuda.stream(blocker):
        torch.cuda._sleep(1_500_000_000)          # about a second of one SM spinning
    t0 = time.perf_counter()
    o1 = bsg.gemm(*ds, stream=s1)                # first use of s1: allocates
    o2 = bsg.gemm(*ds, stream=s2)                # first use of s2: its own workspace
    o3 = bsg.gemm(*dl, stream=s1)                # s1 grows: free + allocate, stream-ordered
    host_s = time.perf_counter() - t0
    still_running = not blocker.query()
    torch.cuda.synchronize()
    assert still_running, "a growing call waited for another stream's work"
    assert host_s < 0.5, host_s
    assert bsg.get_last_device_status() == 0
    rs, rl = _ref(small), _ref(large)
    check_close(gpu_as_f64(o1), rs, "workspace: first use of a stream")
    check_close(gpu_as_f64(o2), rs, "workspace: second stream")
    check_close(gpu_as_f64(o3), rl, "workspace: grown")
    # the grown workspace serves the small plan again, and agrees bit for bit
    o4 = bsg.gemm(*ds, stream=s1)
    torch.cuda.synchronize()
    assert torch.equal(o4.view(torch.int16), o1.view(torch.int16))


def test_release_frees_workspaces_and_later_calls_allocate_again():
    torch.cuda.set_device(0)
    p = workloads.make_problem(32, 1024, 2048, seed=13, name="ws release")
    d = to_device(p)
    s = torch.cuda.Stream()
    o1 = bsg.gemm(*d, stream=s)
    torch.cuda.synchronize()
    assert bsg.release_workspaces() == 0
    o2 = bsg.gemm(*d, stream=s)
    torch.cuda.synchronize()
    assert bsg.get_last_device_status() == 0
    check_close(gpu_as_f64(o2), _ref(p), "workspace: after release")
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16))


def test_a_captured_call_that_would_grow_the_workspace_is_refused():
    """Growing inside stream capture would hand the graph the new memory: the
    call is refused before anything is launched, and the same call made
    first outside capture then captures and replays correctly."""
    torch.cuda.set_device(0)
    p = workloads.make_problem(64, 2048, 4096, seed=14, name="ws capture")
    a, b, sa, sb = to_device(p)
    out = torch.empty((p.M, p.N), dtype=torch.bfloat16, device="cuda")
    s = torch.cuda.Stream()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with pytest.raises(bsg.BsgemmError) as e:
        with torch.cuda.graph(g, stream=s):
            bsg.gemm(a, b, sa, sb, out=out, stream=s)
    assert e.value.status == 5
    del g
    torch.cuda.synchronize()
    bsg.gemm(a, b, sa, sb, out=out, stream=s)    # grows outside capture
    torch.cuda.synchronize()
    out.zero_()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        bsg.gemm(a, b, sa, sb, out=out, stream=s)
    g.replay()
    torch.cuda.synchronize()
    assert bsg.get_last_device_status() == 0
    check_close(gpu_as_f64(out), _ref(p), "workspace: captured and replayed")
    del g
