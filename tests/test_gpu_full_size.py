"""GPU parity at the workloads' full sizes, in the launch configuration the
bench times (the library's own plan), on outputs the oracle computes one by
one: a seeded sample plus corners and tile-boundary elements.

Workloads: square 4096^3 with outlier rows; FFN up-projection 8192x14336x4096
(NT, TN and TT); small-M decode shapes M in {1,8,32,64,128}, N = K = 7168;
long-K 2048x4096x32768 at g = 64, 128, 256 with the error checked as K grows.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
import fp8_block_scaled_bsgemm_b200 as bsg

from gpu_util import check_close, full_parity, gpu_as_f64, sampled_parity

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


def test_square_4096_outliers():
    sampled_parity(workloads.square(), count=4000)


@pytest.mark.parametrize("layout", ["nt", "tn", "tt"])
def test_ffn_up_projection(layout):
    sampled_parity(workloads.ffn(layout=layout), count=2000)


@pytest.mark.parametrize("M", [1, 8, 32, 64, 128])
def test_small_m_decode(M):
    p = workloads.small_m(M)
    if M <= 8:
        full_parity(p)
    else:
        sampled_parity(p, count=3000)


@pytest.mark.parametrize("gran", [64, 128, 256])
def test_long_k_error_growth(gran):
    """Parity at growing K prefixes of the same operands (4k, 8k, 16k, 32k):
    the per-element error stays within tolerance at every length."""
    p = workloads.long_k(gran=gran)
    a = torch.from_numpy(p.a).cuda()
    b = torch.from_numpy(p.b).cuda()
    sa = torch.from_numpy(p.sa).cuda()
    sb = torch.from_numpy(p.sb).cuda()
    mi, ni = workloads.sample_indices(p.M, p.N, 600, seed=gran)
    ratios = []
    for kp in (4096, 8192, 16384, 32768):
        kbp = kp // gran
        a_k, b_k = a[:, :kp].contiguous(), b[:, :kp].contiguous()
        sa_k, sb_k = sa[:, :kbp].contiguous(), sb[:, :kbp].contiguous()
        out = bsg.gemm(a_k, b_k, sa_k, sb_k, gran=gran)
        torch.cuda.synchronize()
        ref, _ = oracle.bsgemm_at("nt", p.a[:, :kp], p.b[:, :kp], p.sa[:, :kbp], p.sb[:, :kbp],
                                  p.M, p.N, kp, gran, mi, ni)
        got = gpu_as_f64(out[torch.from_numpy(mi).cuda(), torch.from_numpy(ni).cuda()])
        ratios.append(check_close(got, ref, f"long-K g={gran} K={kp}"))
    print(f"long-K g={gran}: max err/tol at K=4k,8k,16k,32k = {[round(r, 3) for r in ratios]}")
