"""Host-side checks of the seeded input generator (no GEMM arithmetic here)."""
import numpy as np
import pytest
import torch

import workloads


def _decode(codes):
    return torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()


@pytest.mark.parametrize("g", [64, 128, 256])
def test_quantize_blocks_round_trip(g):
    rng = np.random.default_rng(0)
    x = (rng.standard_normal((300, 520)) * 3).astype(np.float32)
    codes, s = workloads.quantize_blocks(x, g)
    assert codes.shape == x.shape and codes.dtype == np.uint8
    assert s.shape == (-(-300 // g), -(-520 // g)) and s.dtype == np.float32
    assert not np.any((codes & 0x7F) == 0x7F), "no NaN codes"
    deq = _decode(codes) * np.repeat(np.repeat(s.astype(np.float64), g, 0), g, 1)[:300, :520]
    # E4M3 keeps 4 significant bits: relative error <= 2^-4 for normals, plus the
    # subnormal quantum 2^-9 * scale
    err = np.abs(deq - x)
    bound = np.abs(x) * 2.0 ** -4 + np.repeat(np.repeat(s, g, 0), g, 1)[:300, :520] * 2.0 ** -9
    assert np.all(err <= bound * 1.0001)
    # every block reaches the largest code magnitude (amax maps to 448)
    mag = _decode(codes & 0x7F)
    for i in range(s.shape[0]):
        for j in range(s.shape[1]):
            assert mag[i * g:(i + 1) * g, j * g:(j + 1) * g].max() == 448.0


def test_zero_block_gets_unit_scale():
    x = np.zeros((128, 256), np.float32)
    x[:, 128:] = 1.0
    codes, s = workloads.quantize_blocks(x, 128)
    assert s[0, 0] == 1.0 and np.all(codes[:, :128] == 0)
    assert s[0, 1] == np.float32(1.0 / 448.0)


def test_saturation_clamps_to_448():
    x = np.full((1, 16), 1.0, np.float32)
    x[0, 0] = 1e30
    codes, s = workloads.quantize_blocks(x, 64)
    assert _decode(codes)[0, 0] == 448.0


def test_generator_is_deterministic_and_layouts_consistent():
    p1 = workloads.make_problem(200, 150, 384, 128, "nt", seed=3)
    p2 = workloads.make_problem(200, 150, 384, 128, "nt", seed=3)
    assert np.array_equal(p1.a, p2.a) and np.array_equal(p1.sb, p2.sb)
    for lay in ("tn", "nn", "tt"):
        q = workloads.make_problem(200, 150, 384, 128, lay, seed=3)
        assert np.array_equal(workloads.logical_a(q), p1.a)
        assert np.array_equal(workloads.logical_b(q), p1.b)


def test_outlier_rows_and_block_std():
    p = workloads.make_problem(4096, 8, 128, 128, seed=0, outlier_rows=41)
    assert p.sa.shape == (32, 1)
    q = workloads.make_problem(256, 8, 1024, 128, seed=0, block_std_log2=(-6.0, 6.0))
    ratio = q.sa.max() / q.sa.min()
    assert ratio > 2 ** 4   # per-block magnitudes spread over many octaves


def test_sample_indices_in_range():
    mi, ni = workloads.sample_indices(7, 300, 100)
    assert mi.min() >= 0 and mi.max() < 7 and ni.min() >= 0 and ni.max() < 300


def test_grouped_moe_stacks_each_group_in_place():
    """The grouped workload's stacked A rows and A scale blocks are each
    group's own, at the offsets the grouped call derives from the group sizes
    (rows R_i = sum of earlier M_i, scale rows S_i = sum of earlier ceil(M_i/g));
    a small instance keeps the test fast."""
    gp = workloads.grouped_moe(groups=5, tokens=700, N=64, K=256, gran=64)
    assert sum(gp.ms) == 700 and len(gp.ms) == 5 and gp.a.shape == (700, 256)
    assert gp.b.shape == (5, 64, 256) and gp.sb.shape == (5, 1, 4)
    assert gp.sa.shape[0] >= -(-700 // 64) + 5
    r = sr = 0
    for m, p in zip(gp.ms, gp.parts):
        nb = -(-m // 64)
        assert np.array_equal(gp.a[r:r + m], p.a[:m])
        assert np.array_equal(gp.sa[sr:sr + nb], p.sa[:nb])
        r += m
        sr += nb
    again = workloads.grouped_moe(groups=5, tokens=700, N=64, K=256, gran=64)
    assert again.ms == gp.ms and np.array_equal(again.a, gp.a) and np.array_equal(again.b, gp.b)
    assert gp.flops == 2 * 700 * 64 * 256
