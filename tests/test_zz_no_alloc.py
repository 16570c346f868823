"""The allocation-free entry point, checked against the regular one.

bsgemm_fp8_nt_noalloc serves callers that cannot allocate device memory:
code running inside an allocator callback, under a framework that owns all
device memory and passes the library only the tensors of the call, or in a
process that must not grow its device footprint after start-up.  Instead of
the split-K workspace the regular entry points create with cudaMalloc, it
uses a fixed scratch array inside the library.

Each case calls it twice in a row through the C ABI -- the array keeps what
the previous call left in it, so the second call shows that every call starts
from clean tile counters -- and compares both outputs with bsgemm_fp8_nt's,
within the tolerance the parity tests use.  The file is named so that pytest
collects it last.
"""
import pytest
import torch

import workloads
import fp8_block_scaled_bsgemm_b200 as bsg

from gpu_util import check_close, gpu_as_f64, to_device

pytestmark = pytest.mark.gpu

LIMIT_BYTES = 16 << 20   # BSGEMM_NOALLOC_SCRATCH_BYTES
SCRATCH_LIMIT = 7        # BSGEMM_ERR_SCRATCH_LIMIT


def _num_sms():
    return torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count


def _fixed_plan(M, N, K, g):
    """The plan the allocation-free entry point takes: the regular one (with
    128-row tiles where that one pairs CTAs) when its scratch fits the fixed
    array, otherwise the one without stream-K."""
    plan = bsg.make_plan(M, N, K, g, "nt", _num_sms())
    if plan["cta_pair"]:
        plan = bsg.make_plan(M, N, K, g, "nt", _num_sms(), {"variant": "data_parallel"})
    if bsg.scratch_bytes(plan) > LIMIT_BYTES:
        plan = bsg.make_plan(M, N, K, g, "nt", _num_sms(), {"stream_k": -1})
    return plan


def _call(fn, a, b, sa, sb, out, M, N, K, g):
    return fn(a.data_ptr(), b.data_ptr(), sa.data_ptr(), sb.data_ptr(), out.data_ptr(), M, N, K, g,
              torch.cuda.current_stream().cuda_stream)


@pytest.mark.parametrize("M,N,K,g", [(8, 7168, 7168, 128), (256, 7168, 2048, 128), (100, 1024, 4096, 64)])
def test_no_alloc_matches_regular_entry_point_twice(M, N, K, g):
    plan = _fixed_plan(M, N, K, g)
    assert 0 < bsg.scratch_bytes(plan) <= LIMIT_BYTES, plan   # the plan uses the scratch
    p = workloads.make_problem(M, N, K, g, "nt", seed=31)
    a, b, sa, sb = to_device(p)
    L = bsg.lib()
    want = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    assert _call(L.bsgemm_fp8_nt, a, b, sa, sb, want, M, N, K, g) == 0
    torch.cuda.synchronize()
    ref = gpu_as_f64(want)
    for call in (1, 2):
        got = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        assert _call(L.bsgemm_fp8_nt_noalloc, a, b, sa, sb, got, M, N, K, g) == 0
        torch.cuda.synchronize()
        check_close(gpu_as_f64(got), ref, f"allocation-free call {call}, {M}x{N}x{K} g={g}")
    assert bsg.get_last_device_status() == 0


def test_no_alloc_takes_single_cta_tiles_where_the_regular_plan_pairs():
    """Large g = 256 problems get CTA-pair tiles from the regular entry point; the
    allocation-free one has no pair kernel and takes 128-row tiles, with the same
    product and every row written."""
    M, N, K, g = 2304, 2304, 1024, 256
    if not bsg.make_plan(M, N, K, g, "nt", _num_sms())["cta_pair"]:
        pytest.skip("the regular plan does not pair CTAs on this device")
    assert _fixed_plan(M, N, K, g)["cta_pair"] == 0
    p = workloads.make_problem(M, N, K, g, "nt", seed=32)
    a, b, sa, sb = to_device(p)
    L = bsg.lib()
    want = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    assert _call(L.bsgemm_fp8_nt, a, b, sa, sb, want, M, N, K, g) == 0
    torch.cuda.synchronize()
    got = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    assert _call(L.bsgemm_fp8_nt_noalloc, a, b, sa, sb, got, M, N, K, g) == 0
    torch.cuda.synchronize()
    assert not torch.isnan(got).any()
    check_close(gpu_as_f64(got), gpu_as_f64(want), f"allocation-free call, {M}x{N}x{K} g={g}")
    assert bsg.get_last_device_status() == 0


def test_no_alloc_rejects_problems_beyond_its_scratch():
    # find a problem whose plan needs more scratch than the fixed array holds
    M, N, K, g = next((m, n, k, 128) for m, n, k in [(256, 4096, 7168), (256, 2048, 16384), (384, 4096, 8192)]
                      if bsg.scratch_bytes(_fixed_plan(m, n, k, 128)) > LIMIT_BYTES)
    a = torch.zeros((M, K), dtype=torch.uint8, device="cuda")
    b = torch.zeros((N, K), dtype=torch.uint8, device="cuda")
    sa = torch.ones((-(-M // g), -(-K // g)), dtype=torch.float32, device="cuda")
    sb = torch.ones((-(-N // g), -(-K // g)), dtype=torch.float32, device="cuda")
    out = torch.full((M, N), 3.0, dtype=torch.bfloat16, device="cuda")
    assert _call(bsg.lib().bsgemm_fp8_nt_noalloc, a, b, sa, sb, out, M, N, K, g) == SCRATCH_LIMIT
    torch.cuda.synchronize()
    assert torch.all(out == 3.0)
