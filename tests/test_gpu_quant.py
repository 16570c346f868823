"""GPU per-block FP8 quantiser (``bsgemm_quantize_fp8``) against the oracle's.

The codes are integer decisions taken in FP32 on both sides (s = amax / FMAX,
then x / s, both correctly rounded, then nearest-even with saturation), so the
bar is bit-exact codes and scales (hncyxsy.com/news/191052 §4.4, §5.2).
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
import fp8_block_scaled_bsgemm_b200 as bsg

from gpu_util import check_close, gpu_as_f64

pytestmark = pytest.mark.gpu


def _source(rows, cols, seed, scale=3.0):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((rows, cols)).astype(np.float32) * np.float32(scale)
    x[:40, :64] = 0.0                               # an all-zero region (whole block at g = 64)
    x[rows // 2, 16] = np.float32(5e3)              # an outlier
    return x


@pytest.mark.parametrize("fmt", ["e4m3", "e5m2"])
@pytest.mark.parametrize("g", [64, 128, 256])
@pytest.mark.parametrize("rows,cols", [(300, 528), (64, 64), (1, 4096)])
def test_quantiser_fp32_bit_exact(fmt, g, rows, cols):
    x = _source(rows, cols, rows + g)
    q, s = bsg.quantize(torch.from_numpy(x).cuda(), g, fmt)
    q_ref, s_ref = oracle.quantize_blocks(x, g, fmt)
    assert np.array_equal(s.cpu().numpy(), s_ref)
    assert np.array_equal(q.cpu().numpy(), q_ref)


@pytest.mark.parametrize("fmt", ["e4m3", "e5m2"])
@pytest.mark.parametrize("g", [64, 128, 256])
def test_quantiser_bf16_bit_exact(fmt, g):
    x32 = _source(200, 1040, 5)
    xb = torch.from_numpy(x32).to(torch.bfloat16)
    q, s = bsg.quantize(xb.cuda(), g, fmt)
    q_ref, s_ref = oracle.quantize_blocks(xb.float().numpy(), g, fmt)   # BF16 -> FP32 is exact
    assert np.array_equal(s.cpu().numpy(), s_ref)
    assert np.array_equal(q.cpu().numpy(), q_ref)


# BF16 block maxima: denormals (their blocks keep the division), the smallest
# normal, values around 1 and the formats' maxima, and the largest finite BF16
AMAX_BITS = [0x0001, 0x0042, 0x0080, 0x0D00, 0x1C80, 0x2F3B, 0x3A01, 0x3F80, 0x3FC0,
             0x41A5, 0x43E0, 0x4480, 0x4760, 0x5A5A, 0x6E11, 0x7F7F]


def _every_bf16_up_to(amax_bits, g):
    """Blocks of g x g BF16 values: for each amax, its value first and then
    every BF16 bit pattern of either sign with |x| <= amax, over as many
    blocks as that takes (each block starts with amax, so amax is its max)."""
    per = g * g - 1
    blocks = []
    for ab in amax_bits:
        mags = np.arange(0, ab + 1, dtype=np.uint32)
        vals = np.concatenate([mags, mags | 0x8000]).astype(np.uint16)
        for i in range(0, vals.size, per):
            chunk = vals[i:i + per]
            blk = np.full(g * g, ab, dtype=np.uint16)
            blk[1:1 + chunk.size] = chunk
            blocks.append(blk.reshape(g, g))
    return np.concatenate(blocks, axis=0)          # [blocks * g, g]


@pytest.mark.parametrize("fmt", ["e4m3", "e5m2"])
@pytest.mark.parametrize("g", [64, 128, 256])
def test_quantiser_bf16_every_value_below_amax(fmt, g):
    """The BF16 path's quotient (a corrected reciprocal product where the
    block scale allows it) against the oracle's division, for every BF16 value
    under each of several block maxima, from denormal to the largest finite."""
    u16 = _every_bf16_up_to(AMAX_BITS, g)
    xb = torch.from_numpy(u16.view(np.int16)).view(torch.bfloat16)
    q, s = bsg.quantize(xb.cuda(), g, fmt)
    q_ref, s_ref = oracle.quantize_blocks(xb.float().numpy(), g, fmt)   # BF16 -> FP32 is exact
    assert np.array_equal(s.cpu().numpy(), s_ref)
    got = q.cpu().numpy()
    assert np.array_equal(got, q_ref), int(np.sum(got != q_ref))


@pytest.mark.parametrize("src", ["fp32", "bf16"])
@pytest.mark.parametrize("g", [64, 128, 256])
def test_quantiser_large_ragged(src, g):
    """A large matrix: more blocks than the GPU holds CTAs at once (over eight
    per SM), so blocks run in several waves. The last row block and the last
    column block are ragged: 8208 columns leave a 16-column last block."""
    rows, cols = (9300 if g == 256 else 6100), 8208
    n_sms = torch.cuda.get_device_properties(0).multi_processor_count
    assert (-(-rows // g)) * (-(-cols // g)) > 8 * n_sms
    x32 = _source(rows, cols, 31 + g, scale=2.0)
    if src == "bf16":
        xt = torch.from_numpy(x32).to(torch.bfloat16)
        x_ref = xt.float().numpy()                  # BF16 -> FP32 is exact
    else:
        xt = torch.from_numpy(x32)
        x_ref = x32
    q, s = bsg.quantize(xt.cuda(), g, "e4m3")
    q_ref, s_ref = oracle.quantize_blocks(x_ref, g, "e4m3")
    assert np.array_equal(s.cpu().numpy(), s_ref)
    assert np.array_equal(q.cpu().numpy(), q_ref)


def test_quantise_then_gemm_matches_oracle_pipeline():
    """Online activations: quantise A and B on the GPU, multiply on the GPU;
    the same steps in the oracle give the reference."""
    M, N, K, g = 320, 784, 1152, 128
    rng = np.random.default_rng(9)
    a32 = rng.standard_normal((M, K)).astype(np.float32)
    b32 = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    qa, sa = bsg.quantize(torch.from_numpy(a32).cuda(), g)
    qb, sb = bsg.quantize(torch.from_numpy(b32).cuda(), g, "e5m2")
    out = bsg.gemm(qa, qb, sa, sb, layout="nt", gran=g, a_format="e4m3", b_format="e5m2")
    oqa, osa = oracle.quantize_blocks(a32, g)
    oqb, osb = oracle.quantize_blocks(b32, g, "e5m2")
    ref, _ = oracle.bsgemm("nt", oqa, oqb, osa, osb, M, N, K, g, "e4m3", "e5m2")
    check_close(gpu_as_f64(out), ref, "quantise + GEMM")


def test_quantiser_host_errors():
    x = torch.zeros((8, 40), device="cuda")
    with pytest.raises(bsg.BsgemmError) as e:
        bsg.quantize(x, 128)                          # cols % 16 != 0
    assert e.value.status == 3
    with pytest.raises(bsg.BsgemmError) as e:
        bsg.quantize(torch.zeros((8, 64), device="cuda"), 32)
    assert e.value.status == 2
