"""Two MMA-issuing warps: parity where their hand-offs are most fragile.

The single-CTA kernel's two issuer warps take the CTA's K-blocks in turn
(issuer x % 2 takes K-block x, counted over all of the CTA's work items).  The
hazards are at work-item boundaries, where the K-block count of a tile is odd,
and where a stage changes hands between the issuers:
- g = 64: a stage holds two K-blocks, one per issuer; an odd count leaves the
  last stage of a tile half empty;
- g = 256: a K-block is two stages, or one at the K tail;
- two TMEM buffers (256-wide tiles) give an issuer the least slack.
Each case runs at least two tiles per CTA (more tiles than 2 x 148), with
integer-valued operands and power-of-two scales, so every partial sum is exact
in FP32 and every correct plan must return the same bits.  Sampled outputs are
compared bit for bit with the oracle, and the whole output with a second plan.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
import fp8_block_scaled_bsgemm_b200 as bsg

from gpu_util import run_gpu

pytestmark = pytest.mark.gpu


def _integer_problem(M, N, K, gran, seed):
    """Values in {0, +-1, +-2} and scales in {2^-4, 2^-3, 2^-2}: |out| stays
    far below 2^16 on a 2^-8 grid, exact in the FP32 accumulator."""
    rng = np.random.default_rng(seed)
    vals = np.array([0x00, 0x38, 0x40, 0xB8, 0xC0], np.uint8)   # 0, 1, 2, -1, -2 in E4M3
    a = vals[rng.integers(0, vals.size, size=(M, K))]
    b = vals[rng.integers(0, vals.size, size=(N, K))]
    Kb = -(-K // gran)
    sa = np.exp2(rng.integers(-4, -1, size=(-(-M // gran), Kb))).astype(np.float32)
    sb = np.exp2(rng.integers(-4, -1, size=(-(-N // gran), Kb))).astype(np.float32)
    return workloads.Problem(M, N, K, gran, "nt", a, b, sa, sb, "integer-exact, many tiles")


def _tiles(plan):
    return plan["tiles_p"] * plan["tiles_q"]


# (M, N, K, g, plan under test, second plan)
CASES = [
    # g = 64, 19 K-blocks per tile, two TMEM buffers
    (2048, 4864, 1216, 64, {"variant": "data_parallel", "bnq": 256}, {"variant": "data_parallel", "bnq": 128}),
    # g = 64 with stream-K ranges (stage-aligned pieces, odd K-block tail)
    (2048, 4864, 1216, 64, {"variant": "data_parallel", "bnq": 256, "stream_k": 1},
     {"variant": "data_parallel", "bnq": 128}),
    # g = 64, four buffers
    (2048, 2432, 1216, 64, {"variant": "data_parallel", "bnq": 128}, {"variant": "data_parallel", "bnq": 256}),
    # g = 256, last K-block one stage, four stages
    (2048, 4864, 1152, 256, {"variant": "data_parallel", "bnq": 256}, {"variant": "data_parallel", "bnq": 128}),
    # g = 256 with six stages: the ring's lap holds an odd number of K-blocks
    (2048, 2432, 1152, 256, {"variant": "data_parallel", "bnq": 128}, {"variant": "data_parallel", "bnq": 256}),
    # g = 128 with a partial last K-block
    (2048, 4864, 1216, 128, {"variant": "data_parallel", "bnq": 256}, {"variant": "data_parallel", "bnq": 128}),
    # narrow swap-AB tiles, eight buffers, g = 64 and g = 256
    (192, 7168, 1216, 64, {"variant": "swap_ab", "bnq": 32}, {"variant": "swap_ab", "bnq": 64}),
    (192, 7168, 1152, 256, {"variant": "swap_ab", "bnq": 32}, {"variant": "swap_ab", "bnq": 64}),
]


@pytest.mark.parametrize("M,N,K,g,tuning,other", CASES)
def test_many_tiles_per_cta_bit_exact(M, N, K, g, tuning, other):
    n_sms = torch.cuda.get_device_properties(0).multi_processor_count
    plan = bsg.make_plan(M, N, K, g, "nt", n_sms, tuning)
    assert _tiles(plan) >= 2 * n_sms or plan["sk_ctas"] > 0, plan
    p = _integer_problem(M, N, K, g, seed=M + N + K + g)
    out = run_gpu(p, tuning)
    assert bsg.get_last_device_status() == 0
    got = out.view(torch.int16).cpu().numpy().astype(np.uint16)
    mi, ni = workloads.sample_indices(M, N, 4000, seed=g)
    ref, want = oracle.bsgemm_at("nt", p.a, p.b, p.sa, p.sb, M, N, K, g, mi, ni)
    assert np.all(ref == np.round(ref * 256) / 256)   # on the 2^-8 grid: exact in FP32
    assert np.array_equal(got[mi, ni], want), int(np.sum(got[mi, ni] != want))
    second = run_gpu(p, other).view(torch.int16).cpu().numpy().astype(np.uint16)
    assert np.array_equal(got, second), int(np.sum(got != second))
