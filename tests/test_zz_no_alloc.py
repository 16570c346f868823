"""The allocation-free entry point, checked against the regular one.

bsgemm_fp8_nt_noalloc serves callers that cannot allocate device memory:
code running inside an allocator callback, under a framework that owns all
device memory and passes the library only the tensors of the call, or in a
process that must not grow its device footprint after start-up.  Instead of
the split-K workspace the regular entry points allocate (cudaMallocAsync), it
uses a fixed scratch array inside the library.

Each case calls it twice in a row through the C ABI -- the array keeps what
the previous call left in it, so the second call shows that every call starts
from clean tile counters -- and compares both outputs with bsgemm_fp8_nt's,
within the tolerance the parity tests use, and with the oracle.  The file is
named so that pytest collects it last.
"""
import pytest
import torch

import oracle
import workloads
import fp8_block_scaled_bsgemm_b200 as bsg

from gpu_util import check_close, gpu_as_f64, to_device

pytestmark = pytest.mark.gpu

LIMIT_BYTES = 16 << 20   # BSGEMM_NOALLOC_SCRATCH_BYTES
MAX_TILES = 4096         # BSGEMM_NOALLOC_MAX_TILES


def _num_sms():
    return torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count


def _fits(plan):
    tiles = plan["tiles_p"] * plan["tiles_q"]
    if plan["sk_ctas"] > 0:
        counters = tiles - plan["sk_first_tile"]
    elif plan["splits"] > 1:
        counters = tiles
    else:
        counters = 0
    return bsg.scratch_bytes(plan) <= LIMIT_BYTES and counters <= MAX_TILES


def _fixed_plan(M, N, K, g):
    """The plan the allocation-free entry point takes: the regular one (with
    128-row tiles where that one pairs CTAs) when its scratch fits the fixed
    array; otherwise the same variant and tile width without stream-K, with
    the split count lowered until it fits."""
    n = _num_sms()
    plan = bsg.make_plan(M, N, K, g, "nt", n)
    if plan["cta_pair"]:
        plan = bsg.make_plan(M, N, K, g, "nt", n, {"variant": "data_parallel"})
    if not _fits(plan):
        t = {"variant": "swap_ab" if plan["swap_ab"] else "data_parallel", "bnq": plan["bnq"], "stream_k": -1}
        plan = bsg.make_plan(M, N, K, g, "nt", n, t)
        s = plan["splits"] - 1
        while not _fits(plan) and s >= 1:
            plan = bsg.make_plan(M, N, K, g, "nt", n, dict(t, splits=s))
            s -= 1
    return plan


def _call(fn, a, b, sa, sb, out, M, N, K, g):
    return fn(a.data_ptr(), b.data_ptr(), sa.data_ptr(), sb.data_ptr(), out.data_ptr(), M, N, K, g,
              torch.cuda.current_stream().cuda_stream)


# The decode shapes 128 x 7168 x 7168 and 256 x 4096 x 7168 (g = 128): their
# regular plans (128-wide stream-K tiles) need more scratch than the array
# holds, so they run with a lowered split count.  The others fit as planned.
CASES = [(8, 7168, 7168, 128), (64, 7168, 7168, 128), (100, 1024, 4096, 64),
         (128, 7168, 7168, 128), (256, 4096, 7168, 128)]


@pytest.mark.parametrize("M,N,K,g", CASES)
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
    # the oracle, on every output of the small case and on a sample of the others
    if M * N <= 200_000:
        exact, _ = oracle.bsgemm("nt", p.a, p.b, p.sa, p.sb, M, N, K, g)
        mi = ni = None
    else:
        mi, ni = workloads.sample_indices(M, N, 3000, seed=5)
        exact, _ = oracle.bsgemm_at("nt", p.a, p.b, p.sa, p.sb, M, N, K, g, mi, ni)
    for call in (1, 2):
        got = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        assert _call(L.bsgemm_fp8_nt_noalloc, a, b, sa, sb, got, M, N, K, g) == 0
        torch.cuda.synchronize()
        g64 = gpu_as_f64(got)
        check_close(g64, ref, f"allocation-free call {call} vs regular, {M}x{N}x{K} g={g}")
        check_close(g64 if mi is None else g64[mi, ni], exact,
                    f"allocation-free call {call} vs oracle, {M}x{N}x{K} g={g}")
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


def test_no_alloc_plans_stay_within_the_array():
    """Where the regular plan would overflow the fixed array, the plan the
    entry point takes instead keeps the variant and tile width and fits."""
    n = _num_sms()
    over = [(m, nn, k) for m, nn, k in [(128, 7168, 7168), (128, 7168, 16384), (256, 4096, 7168),
                                        (256, 2048, 16384), (384, 4096, 8192)]
            if not _fits(bsg.make_plan(m, nn, k, 128, "nt", n))]
    assert over, "no shape's regular plan overflows the array on this device"
    for m, nn, k in over:
        reg = bsg.make_plan(m, nn, k, 128, "nt", n)
        fixed = _fixed_plan(m, nn, k, 128)
        assert _fits(fixed) and fixed["sk_ctas"] == 0, (m, nn, k, fixed)
        assert fixed["swap_ab"] == reg["swap_ab"] and fixed["bnq"] == reg["bnq"]
