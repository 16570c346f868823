"""Grouped NT GEMM (``bsgemm_fp8_grouped_nt``): many independent products with
a shared N and K in one persistent launch (hncyxsy.com/news/191052 §2.1, the
"batch of matrices with different shapes" case). The reference is the oracle
run on each group separately, which is what the grouped call is defined as.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
import fp8_block_scaled_bsgemm_b200 as bsg

from gpu_util import check_close, gpu_as_f64

pytestmark = pytest.mark.gpu


def _grouped(ms, N, K, g, fa="e4m3", fb="e4m3", seed=0, slack=40):
    parts = [workloads.make_problem(max(m, 1), N, K, g, "nt", seed=seed + i, a_fmt=fa, b_fmt=fb)
             for i, m in enumerate(ms)]
    max_rows = sum(ms) + slack
    Kb = -(-K // g)
    a = np.zeros((max_rows, K), np.uint8)
    sa = np.full((-(-max_rows // g) + len(ms), Kb), 7.0, np.float32)   # unused rows: a visible value
    r = sr = 0
    for m, p in zip(ms, parts):
        if m:
            a[r:r + m] = p.a[:m]
            sa[sr:sr + -(-m // g)] = p.sa[:-(-m // g)]
        r += m
        sr += -(-m // g)
    b = np.stack([p.b for p in parts])
    sb = np.stack([p.sb for p in parts])
    return parts, a, sa, b, sb, max_rows


@pytest.mark.parametrize("g", [64, 128, 256])
@pytest.mark.parametrize("N", [128, 384])
def test_grouped_gemm(g, N):
    ms = [0, 1, 130, 256, 77, 300, 0, 5]
    K = 1024
    parts, a, sa, b, sb, max_rows = _grouped(ms, N, K, g, seed=40 + g)
    out = torch.full((max_rows, N), -3.0, dtype=torch.bfloat16, device="cuda")   # exact in BF16
    bsg.grouped_gemm(torch.from_numpy(a).cuda(), torch.from_numpy(b).cuda(), torch.from_numpy(sa).cuda(),
                     torch.from_numpy(sb).cuda(), torch.tensor(ms, dtype=torch.int32, device="cuda"),
                     out=out, gran=g)
    torch.cuda.synchronize()
    got = gpu_as_f64(out)
    r = 0
    for i, (m, p) in enumerate(zip(ms, parts)):
        if m:
            ref, _ = oracle.bsgemm("nt", p.a[:m], p.b, p.sa[:-(-m // g)], p.sb, m, N, K, g)
            check_close(got[r:r + m], ref, f"group {i} (M={m}) g={g} N={N}")
        r += m
    assert np.all(got[r:] == -3.0)                 # rows past the groups are untouched


def test_grouped_gemm_e5m2_and_many_groups():
    rng = np.random.default_rng(50)
    ms = rng.integers(0, 200, size=37).tolist()
    N, K, g = 256, 512, 128
    parts, a, sa, b, sb, max_rows = _grouped(ms, N, K, g, "e5m2", "e4m3", seed=60, slack=0)
    out = bsg.grouped_gemm(torch.from_numpy(a).cuda(), torch.from_numpy(b).cuda(), torch.from_numpy(sa).cuda(),
                           torch.from_numpy(sb).cuda(), torch.tensor(ms, dtype=torch.int32, device="cuda"),
                           gran=g, a_format="e5m2", b_format="e4m3")
    got = gpu_as_f64(out)
    r = 0
    for i, (m, p) in enumerate(zip(ms, parts)):
        if m:
            ref, _ = oracle.bsgemm("nt", p.a[:m], p.b, p.sa[:-(-m // g)], p.sb, m, N, K, g, "e5m2", "e4m3")
            check_close(got[r:r + m], ref, f"group {i} (M={m})")
        r += m


def test_grouped_gemm_argument_errors():
    a = torch.zeros((64, 128), dtype=torch.uint8, device="cuda")
    b = torch.zeros((2, 128, 128), dtype=torch.uint8, device="cuda")
    sa = torch.ones((3, 1), device="cuda")
    sb = torch.ones((2, 1, 1), device="cuda")
    with pytest.raises(ValueError):
        bsg.grouped_gemm(a, b, sa, sb, torch.zeros(2, dtype=torch.int64, device="cuda"))
    with pytest.raises(ValueError):
        bsg.grouped_gemm(a, b, sa, sb, torch.zeros(3, dtype=torch.int32, device="cuda"))
    gm = torch.zeros(2, dtype=torch.int32, device="cuda")
    with pytest.raises(ValueError):                  # fewer scale rows than ceil(64/128) + 2 groups
        bsg.grouped_gemm(a, b, sa[:2].contiguous(), sb, gm)
    with pytest.raises(ValueError):
        bsg.grouped_gemm(a, b, sa, sb.cpu(), gm)
    with pytest.raises(ValueError):
        bsg.grouped_gemm(a, b, sa, sb, gm.cpu())


def test_grouped_moe_workload_sampled():
    """The bench's grouped workload at full size (8192 rows over 8 experts of
    4096 x 7168, g = 128), through the same call the bench times: sampled
    outputs of every group against the oracle run on that group."""
    from gpu_util import full_rms_from_gpu
    gp = workloads.grouped_moe()
    a, b = torch.from_numpy(gp.a).cuda(), torch.from_numpy(gp.b).cuda()
    sa, sb = torch.from_numpy(gp.sa).cuda(), torch.from_numpy(gp.sb).cuda()
    out = bsg.grouped_gemm(a, b, sa, sb, torch.tensor(gp.ms, dtype=torch.int32, device="cuda"), gran=gp.gran)
    torch.cuda.synchronize()
    assert bsg.get_last_device_status() == 0
    r = 0
    for i, (m, p) in enumerate(zip(gp.ms, gp.parts)):
        if m:
            og = out[r:r + m]
            mi, ni = workloads.sample_indices(m, gp.N, 600, seed=i)
            ref, _ = oracle.bsgemm_at("nt", p.a[:m], p.b, p.sa[:-(-m // gp.gran)], p.sb, m, gp.N, gp.K,
                                      gp.gran, mi, ni)
            got = gpu_as_f64(og[torch.from_numpy(mi).cuda(), torch.from_numpy(ni).cuda()])
            check_close(got, ref, f"grouped MoE group {i} (M={m})", rms=full_rms_from_gpu(og))
        r += m
