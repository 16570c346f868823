"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle.

Every case compares element by element with the tolerance in gpu_util.py;
integer-exact cases must match bit for bit. Sizes are chosen so the oracle
finishes in seconds yet the GPU path crosses several tiles and ragged tails.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
import fp8_block_scaled_bsgemm_b200 as bsg

from gpu_util import check_close, full_parity, gpu_as_f64, run_gpu, sampled_parity, to_device

pytestmark = pytest.mark.gpu


def test_library_is_native_and_device_supported():
    assert bsg.lib()._name.endswith("libbsgemm.so")
    assert torch.cuda.get_device_capability() == (10, 0)


# ---------------------------------------------------------------- the tiny config, all layouts
@pytest.mark.parametrize("layout", ["nt", "tn", "nn", "tt"])
def test_tiny_256_cubed(layout):
    full_parity(workloads.tiny(layout=layout))


# ---------------------------------------------------------------- ragged shapes, each granularity
@pytest.mark.parametrize("gran", [64, 128, 256])
@pytest.mark.parametrize("layout", ["nt", "tn", "nn", "tt"])
def test_ragged_shapes(gran, layout):
    # M, N multiples of 16 (MN-major layouts need them); neither a tile multiple
    p = workloads.make_problem(400, 336, 1040, gran, layout, seed=gran)
    full_parity(p, what=f"ragged {layout} g={gran}")


@pytest.mark.parametrize("M,N,K", [(129, 8, 16), (257, 264, 48), (130, 520, 4112), (7, 1000, 656)])
def test_odd_sizes_nt(M, N, K):
    for g in (64, 128, 256):
        full_parity(workloads.make_problem(M, N, K, g, "nt", seed=M + g), what=f"{M}x{N}x{K} g={g}")


# ---------------------------------------------------------------- every kernel variant
@pytest.mark.parametrize("variant,bnq", [("data_parallel", 128), ("data_parallel", 256),
                                         ("swap_ab", 16), ("swap_ab", 32), ("swap_ab", 64),
                                         ("swap_ab", 128)])
@pytest.mark.parametrize("splits", [1, 3, 7])
def test_forced_variants(variant, bnq, splits):
    p = workloads.make_problem(200, 392, 2048, 128, "nt", seed=splits)
    full_parity(p, tuning={"variant": variant, "bnq": bnq, "splits": splits},
                what=f"{variant} bnq={bnq} splits={splits}")


@pytest.mark.parametrize("gran", [64, 128, 256])
@pytest.mark.parametrize("layout", ["nt", "tn", "nn", "tt"])
def test_split_k_each_granularity_and_layout(gran, layout):
    p = workloads.make_problem(160, 272, 3072, gran, layout, seed=3)
    for v, bnq in (("data_parallel", 128), ("swap_ab", 64)):
        full_parity(p, tuning={"variant": v, "bnq": bnq, "splits": 5}, what=f"{layout} g={gran} {v}")


@pytest.mark.parametrize("gran", [64, 128, 256])
@pytest.mark.parametrize("layout", ["nt", "tn"])
@pytest.mark.parametrize("M,N,K", [(2048, 1536, 1040), (96, 2048, 3072)])
def test_stream_k(gran, layout, M, N, K):
    """Stream-K forced: whole tiles plus shared-out K ranges, pieces summed in K order."""
    p = workloads.make_problem(M, N, K, gran, layout, seed=gran + M)
    plan = bsg.make_plan(M, N, K, gran, layout, torch.cuda.get_device_properties(0).multi_processor_count,
                         {"stream_k": 1})
    assert plan["sk_ctas"] > 0
    full_parity(p, tuning={"stream_k": 1}, what=f"stream-K {layout} {M}x{N}x{K} g={gran}")


# ---------------------------------------------------------------- CTA pairs (cta_group::2)
@pytest.mark.parametrize("gran", [64, 128, 256])
@pytest.mark.parametrize("layout", ["nt", "tn", "nn", "tt"])
def test_cta_pair_each_granularity_and_layout(gran, layout):
    """256 x 256 tiles on CTA pairs; ragged M, N and K tails (odd CTA's rows partly past M)."""
    p = workloads.make_problem(656, 784, 1008, gran, layout, seed=11 + gran)
    full_parity(p, tuning={"variant": "cta_pair"}, what=f"pair {layout} g={gran}")


@pytest.mark.parametrize("M,N,K", [(2560, 2304, 512), (384, 4096, 2176), (130, 264, 96)])
def test_cta_pair_shapes(M, N, K):
    """More pair tiles than resident pairs (several waves), a single row of tiles, tiny."""
    p = workloads.make_problem(M, N, K, 128, "nt", seed=M)
    if M * N * K > 1 << 31:
        sampled_parity(p, count=4000, tuning={"variant": "cta_pair"}, what=f"pair {M}x{N}x{K}")
    else:
        full_parity(p, tuning={"variant": "cta_pair"}, what=f"pair {M}x{N}x{K}")


def test_cta_pair_agrees_with_single_cta():
    """Same K-block order and promotion arithmetic; the tensor core's FP32 sums
    inside a K-block round differently between the pair and the single-CTA
    instruction shapes (measured: up to 3 BF16 ulps on near-cancelling
    elements), so the two agree to the parity tolerance, not bit for bit."""
    p = workloads.make_problem(1024, 1280, 1536, 128, "nt", seed=5)
    one = gpu_as_f64(run_gpu(p, tuning={"variant": "data_parallel", "bnq": 256, "stream_k": -1}))
    two = gpu_as_f64(run_gpu(p, tuning={"variant": "cta_pair"}))
    check_close(two, one, "pair vs single CTA")


# ---------------------------------------------------------------- E5M2 operands (§2.2 second format)
@pytest.mark.parametrize("fa,fb", [("e5m2", "e4m3"), ("e4m3", "e5m2"), ("e5m2", "e5m2")])
@pytest.mark.parametrize("layout", ["nt", "tn", "nn", "tt"])
def test_e5m2_operands_each_layout(fa, fb, layout):
    p = workloads.make_problem(272, 528, 1040, 128, layout, seed=21, a_fmt=fa, b_fmt=fb)
    full_parity(p, what=f"{fa} x {fb} {layout}")


@pytest.mark.parametrize("fa,fb", [("e5m2", "e4m3"), ("e5m2", "e5m2")])
@pytest.mark.parametrize("tuning,M,gran", [
    ({"variant": "swap_ab", "bnq": 32, "splits": 3}, 24, 64),
    ({"variant": "data_parallel", "bnq": 128, "stream_k": 1}, 600, 256),
    ({"variant": "cta_pair"}, 600, 128),
])
def test_e5m2_operands_each_variant(fa, fb, tuning, M, gran):
    p = workloads.make_problem(M, 784, 1536, gran, "nt", seed=22, a_fmt=fa, b_fmt=fb)
    full_parity(p, tuning=tuning, what=f"{fa} x {fb} {tuning}")


def test_e5m2_integer_exact_bit_for_bit():
    """Small integers are exact in both formats; power-of-two scales keep every
    partial sum exact, so the GPU must equal the oracle bit for bit."""
    rng = np.random.default_rng(23)
    M, N, K, g = 192, 272, 512, 128
    vals5 = {0x00: 0, 0x3C: 1, 0x40: 2, 0x42: 3, 0x44: 4, 0xBC: -1, 0xC0: -2, 0xC2: -3, 0xC4: -4}
    vals4 = {0x00: 0, 0x38: 1, 0x40: 2, 0x44: 3, 0x48: 4, 0xB8: -1, 0xC0: -2, 0xC4: -3, 0xC8: -4}
    a = np.array(list(vals5))[rng.integers(0, 9, size=(M, K))].astype(np.uint8)
    b = np.array(list(vals4))[rng.integers(0, 9, size=(N, K))].astype(np.uint8)
    Kb = K // g
    sa = np.exp2(rng.integers(-3, 2, size=(-(-M // g), Kb))).astype(np.float32)
    sb = np.exp2(rng.integers(-3, 2, size=(-(-N // g), Kb))).astype(np.float32)
    p = workloads.Problem(M, N, K, g, "nt", a, b, sa, sb, "int e5m2 x e4m3", "e5m2", "e4m3")
    ref, bits = oracle.bsgemm("nt", a, b, sa, sb, M, N, K, g, "e5m2", "e4m3")
    got = run_gpu(p).view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.array_equal(got, bits)


def test_e5m2_binding_takes_format_from_dtype():
    p = workloads.make_problem(128, 256, 256, 128, "nt", seed=24, a_fmt="e5m2", b_fmt="e4m3")
    a, b, sa, sb = to_device(p)
    out = bsg.gemm(a.view(torch.float8_e5m2), b.view(torch.float8_e4m3fn), sa, sb, layout="nt")
    ref, _ = oracle.bsgemm("nt", p.a, p.b, p.sa, p.sb, p.M, p.N, p.K, 128, "e5m2", "e4m3")
    check_close(gpu_as_f64(out), ref, "dtype-derived formats")
    with pytest.raises(ValueError):
        bsg.gemm(a.view(torch.float8_e5m2), b, sa, sb, a_format="e4m3")


# ---------------------------------------------------------------- fused epilogue (§2.3, §6)
@pytest.mark.parametrize("activation", [None, "relu", "gelu"])
@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("tuning,M,layout", [
    (None, 400, "nt"),
    ({"variant": "swap_ab", "bnq": 64, "splits": 3}, 48, "tn"),
    ({"variant": "data_parallel", "bnq": 128, "stream_k": 1}, 640, "nn"),
    ({"variant": "cta_pair"}, 528, "tt"),
])
def test_fused_epilogue(activation, out_dtype, tuning, M, layout):
    """out = act(acc + bias[n]) stored as BF16 or FP32, against the oracle's FP64 epilogue."""
    p = workloads.make_problem(M, 784, 1280, 128, layout, seed=31)
    rng = np.random.default_rng(32)
    bias = (rng.standard_normal(784) * 0.5).astype(np.float32)
    a, b, sa, sb = to_device(p)
    out = bsg.gemm(a, b, sa, sb, layout=layout, gran=128, tuning=tuning, bias=torch.from_numpy(bias).cuda(),
                   activation=activation, out_dtype=out_dtype)
    torch.cuda.synchronize()
    ref, _ = oracle.bsgemm(layout, p.a, p.b, p.sa, p.sb, p.M, p.N, p.K, 128)
    want, bits = oracle.epilogue(ref, bias, activation)
    assert out.dtype == out_dtype
    check_close(gpu_as_f64(out), want, f"epilogue {activation} {out_dtype} {tuning}")


def test_fused_epilogue_fp32_output_without_bias_keeps_fp32_precision():
    """FP32 output: the values before BF16 rounding, so the error is the FP32
    accumulation's alone -- far inside the BF16 tolerance."""
    p = workloads.make_problem(256, 512, 1024, 128, "nt", seed=33)
    a, b, sa, sb = to_device(p)
    out = bsg.gemm(a, b, sa, sb, out_dtype=torch.float32)
    ref, _ = oracle.bsgemm("nt", p.a, p.b, p.sa, p.sb, p.M, p.N, p.K, 128)
    got = gpu_as_f64(out)
    assert np.max(np.abs(got - ref) / (np.abs(ref) + 1e-3 * np.sqrt(np.mean(ref ** 2)))) < 2.0 ** -12


def test_binding_checks_the_tensors_it_hands_to_the_library():
    """The kernels receive bare pointers, so the binding rejects a tensor on the
    host, on another device, or too small for the sizes it implies."""
    p = workloads.make_problem(128, 256, 256, 128, "nt", seed=35)
    a, b, sa, sb = to_device(p)                                   # sa, sb: [1, 2], [2, 2]
    for bad in (dict(scale_a=sa.cpu()), dict(scale_a=sa[:, :1].contiguous()),
                dict(scale_b=sb.reshape(-1)[:3].contiguous()), dict(b=b.cpu())):
        args = dict(a=a, b=b, scale_a=sa, scale_b=sb)
        args.update(bad)
        with pytest.raises(ValueError):
            bsg.gemm(args["a"], args["b"], args["scale_a"], args["scale_b"])
    with pytest.raises(ValueError):
        bsg.gemm(a, b, sa, sb, out=torch.empty((128, 256), dtype=torch.bfloat16))
    with pytest.raises(ValueError):
        bsg.gemm(a, b, sa, sb, bias=torch.zeros(256))
    x = torch.zeros((128, 256), device="cuda")
    with pytest.raises(ValueError):
        bsg.quantize(x, 128, q=torch.empty((128, 256), dtype=torch.uint8))
    with pytest.raises(ValueError):
        bsg.quantize(x, 128, scales=torch.empty((1, 1), device="cuda"))
    torch.cuda.synchronize()
    assert bsg.get_last_device_status() == 0


def test_fused_epilogue_argument_errors():
    p = workloads.make_problem(128, 256, 256, 128, "nt", seed=34)
    a, b, sa, sb = to_device(p)
    with pytest.raises(ValueError):
        bsg.gemm(a, b, sa, sb, activation="tanh")
    with pytest.raises(ValueError):
        bsg.gemm(a, b, sa, sb, bias=torch.zeros(255, device="cuda"))


# ---------------------------------------------------------------- small M (decode-style)
@pytest.mark.parametrize("M", [1, 8, 32, 64, 128])
def test_small_m_reduced_k(M):
    p = workloads.make_problem(M, 7168, 1024, 128, "nt", seed=M)
    full_parity(p, what=f"small-M {M}")


# ---------------------------------------------------------------- exactness and invariants
def _integer_problem(M, N, K, gran, layout, seed):
    """Values |v| <= 2 and power-of-two scales: every partial sum and every
    scaled accumulation is exact in FP32, so GPU and oracle round the same
    exact value to BF16."""
    rng = np.random.default_rng(seed)
    vals = np.array([0x00, 0x38, 0x40, 0xB8, 0xC0], np.uint8)   # 0, 1, 2, -1, -2
    a = vals[rng.integers(0, vals.size, size=(M, K))]
    b = vals[rng.integers(0, vals.size, size=(N, K))]
    Kb = -(-K // gran)
    sa = np.exp2(rng.integers(-4, -1, size=(-(-M // gran), Kb))).astype(np.float32)
    sb = np.exp2(rng.integers(-4, -1, size=(-(-N // gran), Kb))).astype(np.float32)
    p = workloads.Problem(M, N, K, gran, "nt", a, b, sa, sb, "integer-exact")
    return workloads.relayout(p, layout)


@pytest.mark.parametrize("layout", ["nt", "tn", "nn", "tt"])
@pytest.mark.parametrize("tuning", [None, {"variant": "swap_ab", "bnq": 32, "splits": 2},
                                    {"variant": "data_parallel", "bnq": 256, "splits": 3},
                                    {"variant": "data_parallel", "bnq": 128, "stream_k": 1},
                                    {"variant": "cta_pair"}])
def test_integer_exact_bit_for_bit(layout, tuning):
    p = _integer_problem(272, 304, 1024, 128, layout, seed=5)
    ref, want = oracle.bsgemm(p.layout, p.a, p.b, p.sa, p.sb, p.M, p.N, p.K, p.gran)
    # |ref| < 256 on a 2^-8 grid: 16 significant bits, exact in the FP32 accumulator
    assert np.all(np.abs(ref) < 256) and np.all(ref == np.round(ref * 256) / 256)
    out = run_gpu(p, tuning)
    got = out.view(torch.int16).cpu().numpy().astype(np.uint16)
    assert np.array_equal(got, want)


def test_power_of_two_scale_is_exact_on_gpu():
    p = workloads.make_problem(256, 512, 1024, 128, "nt", seed=7)
    out1 = run_gpu(p)
    p2 = workloads.Problem(p.M, p.N, p.K, p.gran, p.layout, p.a, p.b, p.sa * np.float32(4.0), p.sb)
    out2 = run_gpu(p2)
    assert torch.equal(out2.float(), out1.float() * 4.0)


def test_single_block_scale_lands_on_its_block():
    # one K-block of one row block scaled by 2^10: only rows of that block change
    p = workloads.make_problem(384, 256, 768, 128, "nt", seed=8)
    base = gpu_as_f64(run_gpu(p))
    sa = p.sa.copy()
    sa[1, 2] *= np.float32(1024.0)
    p2 = workloads.Problem(p.M, p.N, p.K, p.gran, p.layout, p.a, p.b, sa, p.sb)
    got = gpu_as_f64(run_gpu(p2))
    assert np.array_equal(got[:128], base[:128]) and np.array_equal(got[256:], base[256:])
    ref, _ = oracle.bsgemm("nt", p2.a, p2.b, p2.sa, p2.sb, p.M, p.N, p.K, p.gran)
    check_close(got, ref, "scaled block")


def test_layouts_agree_bit_for_bit():
    p = workloads.make_problem(256, 384, 1536, 128, "nt", seed=10)
    outs = [run_gpu(workloads.relayout(p, lay)) for lay in ("nt", "tn", "nn", "tt")]
    for o in outs[1:]:
        assert torch.equal(o, outs[0])


@pytest.mark.parametrize("tuning", [None, {"variant": "swap_ab", "bnq": 16, "splits": 6},
                                    {"variant": "data_parallel", "bnq": 128, "stream_k": 1},
                                    {"variant": "cta_pair"}])
def test_deterministic_repeats(tuning):
    p = workloads.make_problem(64, 2048, 4096, 128, "nt", seed=11)
    a, b, sa, sb = to_device(p)
    first = bsg.gemm(a, b, sa, sb, gran=128, tuning=tuning)
    for _ in range(20):
        again = bsg.gemm(a, b, sa, sb, gran=128, tuning=tuning)
        assert torch.equal(again, first)


def test_poisoned_output_is_fully_written():
    p = workloads.make_problem(136, 264, 512, 64, "nt", seed=12)
    a, b, sa, sb = to_device(p)
    out = torch.full((p.M, p.N), float("nan"), dtype=torch.bfloat16, device="cuda")
    bsg.gemm(a, b, sa, sb, out=out, gran=64)
    torch.cuda.synchronize()
    assert not torch.isnan(out).any()


# ---------------------------------------------------------------- errors and the bounded wait
def test_host_side_errors_leave_output_untouched():
    p = workloads.tiny()
    a, b, sa, sb = to_device(p)
    out = torch.full((256, 256), 7.0, dtype=torch.bfloat16, device="cuda")
    A, B, SA, SB, O = a.data_ptr(), b.data_ptr(), sa.data_ptr(), sb.data_ptr(), out.data_ptr()
    cases = [
        ((A, B, SA, SB, O, 256, 256, 256, 96), 2),       # unsupported granularity
        ((0, B, SA, SB, O, 256, 256, 256, 128), 1),      # null pointer
        ((A, B, SA, SB, O, 0, 256, 256, 128), 1),        # empty M
        ((A + 1, B, SA, SB, O, 256, 256, 256, 128), 3),  # misaligned base
        ((A, B, SA, SB, O, 256, 256, 200, 128), 3),      # K % 16 != 0
        ((A, B, SA, SB, O, 256, 250, 256, 128), 3),      # N % 8 != 0
    ]
    L = bsg.lib()
    for args, want in cases:
        assert L.bsgemm_fp8_nt(*args, None) == want, args
    torch.cuda.synchronize()
    assert torch.all(out == 7.0)


def test_bounded_wait_times_out_and_context_survives():
    assert bsg.get_last_device_status() == 0
    assert bsg.diag_wait_timeout(2_000_000) == 0          # 2 ms limit
    assert bsg.get_last_device_status() == 6              # BSGEMM_ERR_DEVICE_TIMEOUT
    assert bsg.get_last_device_status() == 0              # cleared
    full_parity(workloads.tiny(), what="after a timed-out wait")
