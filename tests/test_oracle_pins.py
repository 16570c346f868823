"""Pins for the CPU oracle: checks against things other than the oracle itself.

The oracle (``oracle/bsgemm_oracle.c``) restates the block-scaled FP8 GEMM of
hncyxsy.com/news/191052 (§2.2 block scaling + FP32 accumulation, §3.2
segment-wise accumulation, §4.2 API and layouts, §5.2 dequantise by
multiplying). These tests pin it to:
  - torch's own float8_e4m3fn decode (a library routine) and hand values;
  - an independent exact-integer BF16 rounding written here, and torch's
    FP32 -> BF16 rounding on FP32-representable inputs;
  - hand-worked cases in tests/golden/hand_cases.json;
  - closed forms (all-ones blocks give K * sA * sB);
  - power-of-two scale invariants (doubling one block's scale adds exactly
    that block's contribution once more);
  - an exact-rational brute force (Python Fractions, no block grouping);
  - layout and operand-swap equivalences.
"""
import json
import math
import os
import random
import struct
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_cases.json")


# --------------------------------------------------------------------------- E4M3
def test_e4m3_table_matches_torch_decode():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = oracle.e4m3_table()
    nan = np.isnan(ref)
    assert list(np.nonzero(nan)[0]) == [0x7F, 0xFF]
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])
    # 0x80 (-0) decodes to a zero; the sign of a zero term cannot change a sum
    assert got[0x80] == 0.0


@pytest.mark.parametrize("code,value", [
    (0x38, 1.0), (0x30, 0.5), (0x40, 2.0), (0x44, 3.0), (0x4A, 5.0), (0xB8, -1.0),
    (0x7E, 448.0), (0xFE, -448.0), (0x01, 2.0 ** -9), (0x07, 7 * 2.0 ** -9),
    (0x08, 2.0 ** -6), (0x77, 240.0), (0x00, 0.0),
])
def test_e4m3_hand_values(code, value):
    assert oracle.e4m3_value(code) == value


# --------------------------------------------------------------------------- BF16
def _bf16_rne_exact(x: float) -> int:
    """Independent FP64 -> BF16 rounding on exact rationals (ties to even)."""
    if math.isnan(x):
        return 0x7FC0
    sign = 0x8000 if math.copysign(1.0, x) < 0 else 0
    f = abs(Fraction(x))
    if f == 0:
        return sign
    # find e with 2^e <= f < 2^(e+1)
    e = f.numerator.bit_length() - f.denominator.bit_length()
    if Fraction(2) ** e > f:
        e -= 1
    e = max(e, -126)                     # subnormals share the 2^-126 quantum grid
    quantum = Fraction(2) ** (e - 7)
    q, rem = divmod(f, quantum)
    q = int(q)
    if rem * 2 > quantum or (rem * 2 == quantum and q % 2 == 1):
        q += 1
    val = q * quantum
    if val > Fraction(255) * Fraction(2) ** 120:
        return sign | 0x7F80
    bits = struct.unpack("<I", struct.pack("<f", float(val)))[0]
    return sign | ((bits >> 16) & 0x7FFF)


@pytest.mark.parametrize("x,bits", [
    (1.0, 0x3F80), (-2.0, 0xC000), (257.0, 0x4380), (259.0, 0x4382),
    (257.0 + 2.0 ** -20, 0x4381),          # one rounding from FP64, not two
    (1.0 + 2.0 ** -8, 0x3F80),             # tie -> even
    (1.0 + 3 * 2.0 ** -8, 0x3F82),         # tie -> even (up)
    (2.0 ** -133, 0x0001),                 # smallest BF16 subnormal
    (2.0 ** -134, 0x0000),                 # tie with zero -> even (zero)
    (3 * 2.0 ** -135, 0x0001),
    (255.0 * 2.0 ** 120, 0x7F7F),          # largest finite
    ((255.5) * 2.0 ** 120, 0x7F80),        # tie above the largest finite rounds to Inf
    (float("inf"), 0x7F80), (-float("inf"), 0xFF80), (-0.0, 0x8000),
])
def test_bf16_rne_hand(x, bits):
    assert oracle.bf16_rne(x) == bits


def test_bf16_rne_matches_exact_rounding_on_random_doubles():
    rnd = random.Random(1234)
    for _ in range(20000):
        mant = rnd.getrandbits(53) | (1 << 52)
        x = math.ldexp(mant, rnd.randint(-190, 80)) * rnd.choice((-1, 1))
        assert oracle.bf16_rne(x) == _bf16_rne_exact(x), x
    # values on and next to BF16 midpoints
    for _ in range(5000):
        b = rnd.randint(1, 0x7F7E)
        lo = struct.unpack("<f", struct.pack("<I", b << 16))[0]
        hi = struct.unpack("<f", struct.pack("<I", (b + 1) << 16))[0]
        mid = (Fraction(lo) + Fraction(hi)) / 2
        for x in (float(mid), math.nextafter(float(mid), 0.0), math.nextafter(float(mid), 1e300)):
            assert oracle.bf16_rne(x) == _bf16_rne_exact(x), x


def test_bf16_rne_matches_torch_on_float32_inputs():
    # torch rounds FP32 -> BF16 to nearest even; on FP32-representable inputs a
    # single rounding from FP64 must agree with it bit for bit.
    g = torch.Generator().manual_seed(5)
    x = (torch.randn(20000, generator=g, dtype=torch.float32)
         * torch.exp2(torch.randint(-40, 40, (20000,), generator=g).float()))
    want = x.to(torch.bfloat16).view(torch.int16).numpy().astype(np.uint16)
    got = np.array([oracle.bf16_rne(float(v)) for v in x.numpy()], dtype=np.uint16)
    assert np.array_equal(got, want)


# --------------------------------------------------------------------------- golden
def _rows(spec, K):
    out = []
    for row in spec:
        codes = []
        for code, count in row:
            codes += [int(code, 16)] * count
        assert len(codes) == K
        out.append(codes)
    return np.array(out, dtype=np.uint8)


def test_golden_hand_cases():
    data = json.load(open(GOLDEN))
    assert data["cases"]
    for case in data["cases"]:
        M, N, K, g = case["M"], case["N"], case["K"], case["gran"]
        a = _rows(case["a_rows"], K)
        b = _rows(case["b_rows"], K)
        sa = np.array(case["sa"], dtype=np.float32)
        sb = np.array(case["sb"], dtype=np.float32)
        ref, out = oracle.bsgemm("nt", a, b, sa, sb, M, N, K, g)
        assert np.array_equal(ref, np.array(case["ref"], dtype=np.float64)), case["name"]
        want = np.array([[int(v, 16) for v in r] for r in case["out_bf16"]], dtype=np.uint16)
        assert np.array_equal(out, want), case["name"]


# --------------------------------------------------------------------------- closed forms
@pytest.mark.parametrize("M,N,K,g", [(130, 70, 300, 64), (130, 257, 300, 128), (300, 20, 520, 256),
                                     (1, 1, 16, 128)])
def test_closed_form_all_ones(M, N, K, g):
    """All codes 1.0 (0x38): out[m,n] = sum_kb len(kb) * sA[m/g,kb] * sB[n/g,kb]."""
    Kb = -(-K // g)
    rng = np.random.default_rng(3)
    sa = np.exp2(rng.integers(-4, 5, size=(-(-M // g), Kb))).astype(np.float32)
    sb = np.exp2(rng.integers(-4, 5, size=(-(-N // g), Kb))).astype(np.float32)
    a = np.full((M, K), 0x38, np.uint8)
    b = np.full((N, K), 0x38, np.uint8)
    ref, _ = oracle.bsgemm("nt", a, b, sa, sb, M, N, K, g)
    lens = np.array([min(K, (kb + 1) * g) - kb * g for kb in range(Kb)], dtype=np.float64)
    for m in range(0, M, max(1, M // 7)):
        for n in range(0, N, max(1, N // 7)):
            want = float(np.sum(lens * sa[m // g].astype(np.float64) * sb[n // g].astype(np.float64)))
            assert ref[m, n] == want
    # uniform scales: K * s_a * s_b exactly
    ref2, _ = oracle.bsgemm("nt", a, b, np.full_like(sa, 0.75), np.full_like(sb, 3.0), M, N, K, g)
    assert np.all(ref2 == K * 0.75 * 3.0)


def _small_int_problem(M, N, K, g, seed):
    """Codes whose values are small integers (|v| <= 4), power-of-two scales:
    every FP64 operation in the oracle is then exact."""
    rng = np.random.default_rng(seed)
    small = np.array([0x00, 0x38, 0x40, 0x44, 0x48, 0xB8, 0xC0, 0xC4, 0xC8], dtype=np.uint8)
    a = small[rng.integers(0, small.size, size=(M, K))]
    b = small[rng.integers(0, small.size, size=(N, K))]
    Kb = -(-K // g)
    sa = np.exp2(rng.integers(-3, 4, size=(-(-M // g), Kb))).astype(np.float32)
    sb = np.exp2(rng.integers(-3, 4, size=(-(-N // g), Kb))).astype(np.float32)
    return a, b, sa, sb


@pytest.mark.parametrize("g", [64, 128, 256])
def test_power_of_two_scale_doubles_one_block(g):
    M, N, K = 3 * g // 2 + 5, g + 9, 3 * g + 32
    a, b, sa, sb = _small_int_problem(M, N, K, g, seed=g)
    ref, _ = oracle.bsgemm("nt", a, b, sa, sb, M, N, K, g)
    i, kb = sa.shape[0] - 1, 1
    sa2 = sa.copy()
    sa2[i, kb] *= 2
    ref2, _ = oracle.bsgemm("nt", a, b, sa2, sb, M, N, K, g)
    only = np.zeros_like(sa)
    only[i, kb] = sa[i, kb]
    blk, _ = oracle.bsgemm("nt", a, b, only, sb, M, N, K, g)
    # rows outside m-block i are unchanged; rows inside gain exactly the block's term
    assert np.array_equal(ref2 - ref, blk)
    assert np.all(blk[: i * g] == 0)
    assert np.any(blk[i * g:] != 0)


def test_global_power_of_two_scaling_is_exact():
    M, N, K, g = 140, 90, 384, 128
    p = workloads.make_problem(M, N, K, g, seed=11)
    ref, out = oracle.bsgemm("nt", p.a, p.b, p.sa, p.sb, M, N, K, g)
    ref2, out2 = oracle.bsgemm("nt", p.a, p.b, p.sa * np.float32(8.0), p.sb, M, N, K, g)
    assert np.array_equal(ref2, ref * 8.0)
    # BF16 of 8x is the same mantissa with exponent + 3 (no under/overflow here)
    nz = (out & 0x7FFF) != 0
    assert np.array_equal(out2[nz].astype(np.int32) - out[nz].astype(np.int32),
                          np.full(nz.sum(), 3 << 7))


def test_negating_a_negates_result():
    p = workloads.make_problem(70, 50, 256, 64, seed=2)
    ref, _ = oracle.bsgemm("nt", p.a, p.b, p.sa, p.sb, 70, 50, 256, 64)
    ref_n, _ = oracle.bsgemm("nt", p.a ^ np.uint8(0x80), p.b, p.sa, p.sb, 70, 50, 256, 64)
    assert np.array_equal(ref_n, -ref)


# --------------------------------------------------------------------------- brute force
def _exact(a, b, sa, sb, g, m, n):
    """Exact rational out[m,n]: per-element dequantisation, no block grouping."""
    dec = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn)
    dec = dec.to(torch.float64).tolist()
    total = Fraction(0)
    K = a.shape[1]
    for k in range(K):
        xa = Fraction(dec[a[m, k]]) * Fraction(float(sa[m // g, k // g]))
        xb = Fraction(dec[b[n, k]]) * Fraction(float(sb[n // g, k // g]))
        total += xa * xb
    return total


@pytest.mark.parametrize("M,N,K,g,seed", [
    (5, 4, 200, 64, 0),      # Kb = 4, partial last K block
    (130, 3, 320, 64, 1),    # Mb = 3, Kb = 5: a transposed scale index reads other blocks
    (3, 300, 384, 128, 2),   # Nb = 3, Kb = 3, ragged N block
    (4, 2, 768, 256, 3),     # Kb = 3 with g = 256
    (2, 140, 80, 64, 4),     # K smaller than two blocks, partial second block
])
def test_brute_force_exact_rational(M, N, K, g, seed):
    rng = np.random.default_rng(seed)
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    a = codes[rng.integers(0, codes.size, size=(M, K))]
    b = codes[rng.integers(0, codes.size, size=(N, K))]
    Kb = -(-K // g)
    # distinct, non-power-of-two scales so that a transposed or shifted index shows
    sa = rng.uniform(0.01, 3.0, size=(-(-M // g), Kb)).astype(np.float32)
    sb = rng.uniform(0.01, 3.0, size=(-(-N // g), Kb)).astype(np.float32)
    ref, out = oracle.bsgemm("nt", a, b, sa, sb, M, N, K, g)
    picks = [(m, n) for m in range(M) for n in range(N)]
    random.Random(seed).shuffle(picks)
    for m, n in picks[:60]:
        ex = _exact(a, b, sa, sb, g, m, n)
        # bound: Kb FP64 roundings of terms of size <= |term|
        bound = 0
        for kb in range(Kb):
            blk = sum(abs(Fraction(oracle.e4m3_value(a[m, k])) * Fraction(oracle.e4m3_value(b[n, k])))
                      for k in range(kb * g, min(K, (kb + 1) * g)))
            bound += blk * Fraction(float(sa[m // g, kb])) * Fraction(float(sb[n // g, kb]))
        tol = bound * Fraction(Kb + 1) * Fraction(2) ** -52
        assert abs(Fraction(ref[m, n]) - ex) <= tol, (m, n)
        # the BF16 output is the rounding of the exact value unless that value
        # sits within the FP64 error of a rounding boundary
        lo, hi = float(ex - tol), float(ex + tol)
        if _bf16_rne_exact(lo) == _bf16_rne_exact(hi):
            assert out[m, n] == _bf16_rne_exact(float(ex)), (m, n)


# --------------------------------------------------------------------------- layouts
@pytest.mark.parametrize("layout", ["tn", "nn", "tt"])
def test_layouts_give_identical_results(layout):
    p = workloads.make_problem(150, 70, 320, 64, "nt", seed=9)
    ref, out = oracle.bsgemm("nt", p.a, p.b, p.sa, p.sb, p.M, p.N, p.K, p.gran)
    q = workloads.relayout(p, layout)
    assert q.a.shape == ((p.K, p.M) if layout[0] == "t" else (p.M, p.K))
    assert q.b.shape == ((p.K, p.N) if layout[1] == "n" else (p.N, p.K))
    ref2, out2 = oracle.bsgemm(layout, q.a, q.b, q.sa, q.sb, p.M, p.N, p.K, p.gran)
    assert np.array_equal(ref, ref2) and np.array_equal(out, out2)


def test_swapping_operands_transposes_result():
    p = workloads.make_problem(90, 140, 256, 128, seed=4)
    ref, _ = oracle.bsgemm("nt", p.a, p.b, p.sa, p.sb, 90, 140, 256, 128)
    refT, _ = oracle.bsgemm("nt", p.b, p.a, p.sb, p.sa, 140, 90, 256, 128)
    assert np.array_equal(ref, refT.T)


def test_sampled_equals_full():
    p = workloads.make_problem(200, 300, 384, 128, seed=6)
    ref, out = oracle.bsgemm("nt", p.a, p.b, p.sa, p.sb, 200, 300, 384, 128)
    mi, ni = workloads.sample_indices(200, 300, 500, seed=1)
    r2, o2 = oracle.bsgemm_at("nt", p.a, p.b, p.sa, p.sb, 200, 300, 384, 128, mi, ni)
    assert np.array_equal(r2, ref[mi, ni]) and np.array_equal(o2, out[mi, ni])


def test_nan_code_is_reported():
    a = np.full((1, 16), 0x38, np.uint8)
    a[0, 3] = 0x7F
    b = np.full((1, 16), 0x38, np.uint8)
    with pytest.raises(RuntimeError):
        oracle.bsgemm("nt", a, b, np.ones((1, 1), np.float32), np.ones((1, 1), np.float32), 1, 1, 16, 128)


# --------------------------------------------------------------------------- E5M2 (second format, §2.2)
def test_e5m2_table_matches_torch_decode():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e5m2).to(torch.float64).numpy()
    got = oracle.fp8_table("e5m2")
    nan = np.isnan(ref)
    assert sorted(np.nonzero(nan)[0].tolist()) == [0x7D, 0x7E, 0x7F, 0xFD, 0xFE, 0xFF]
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])          # includes +-Inf at 0x7C / 0xFC


@pytest.mark.parametrize("code,value", [
    (0x3C, 1.0), (0x38, 0.5), (0x40, 2.0), (0x42, 3.0), (0x45, 5.0), (0xBC, -1.0),
    (0x7B, 57344.0), (0xFB, -57344.0), (0x01, 2.0 ** -16), (0x03, 3 * 2.0 ** -16),
    (0x04, 2.0 ** -14), (0x7C, math.inf), (0x00, 0.0),
])
def test_e5m2_hand_values(code, value):
    assert oracle.fp8_value("e5m2", code) == value


def test_e4m3_entry_equals_format_entry():
    assert all(oracle.fp8_value("e4m3", c) == oracle.e4m3_value(c) or
               (math.isnan(oracle.e4m3_value(c)) and math.isnan(oracle.fp8_value("e4m3", c)))
               for c in range(256))


def _dec_fmt(fmt):
    dt = torch.float8_e5m2 if fmt == "e5m2" else torch.float8_e4m3fn
    return torch.arange(256, dtype=torch.int32).to(torch.uint8).view(dt).to(torch.float64).tolist()


def _finite_codes(fmt):
    t = _dec_fmt(fmt)
    return np.array([c for c in range(256) if math.isfinite(t[c])], dtype=np.uint8)


@pytest.mark.parametrize("fa,fb", [("e5m2", "e4m3"), ("e4m3", "e5m2"), ("e5m2", "e5m2")])
@pytest.mark.parametrize("M,N,K,g,seed", [(4, 3, 320, 64, 10), (3, 130, 256, 128, 11)])
def test_brute_force_exact_rational_mixed_formats(fa, fb, M, N, K, g, seed):
    """Exact rationals, per-element dequantisation, every finite code of each format."""
    rng = np.random.default_rng(seed)
    a = _finite_codes(fa)[rng.integers(0, _finite_codes(fa).size, size=(M, K))]
    b = _finite_codes(fb)[rng.integers(0, _finite_codes(fb).size, size=(N, K))]
    Kb = -(-K // g)
    sa = rng.uniform(0.01, 3.0, size=(-(-M // g), Kb)).astype(np.float32)
    sb = rng.uniform(0.01, 3.0, size=(-(-N // g), Kb)).astype(np.float32)
    ref, out = oracle.bsgemm("nt", a, b, sa, sb, M, N, K, g, a_fmt=fa, b_fmt=fb)
    da, db = _dec_fmt(fa), _dec_fmt(fb)
    for m in range(M):
        for n in range(N if N < 8 else 8):
            ex = Fraction(0)
            bound = Fraction(0)
            for k in range(K):
                t = Fraction(da[a[m, k]]) * Fraction(db[b[n, k]]) * \
                    Fraction(float(sa[m // g, k // g])) * Fraction(float(sb[n // g, k // g]))
                ex += t
                bound += abs(t)
            # block sums may need one more FP64 rounding with E5M2 operands
            tol = bound * Fraction(2 * Kb + 2) * Fraction(2) ** -52
            assert abs(Fraction(ref[m, n]) - ex) <= tol, (fa, fb, m, n)
            lo, hi = float(ex - tol), float(ex + tol)
            if _bf16_rne_exact(lo) == _bf16_rne_exact(hi):
                assert out[m, n] == _bf16_rne_exact(float(ex)), (m, n)


def test_e5m2_closed_form_all_ones():
    # 0x3C is 1.0 in E5M2, 0x38 is 1.0 in E4M3: out = K * sA * sB per block
    M, N, K, g = 3, 5, 384, 128
    a = np.full((M, K), 0x3C, np.uint8)
    b = np.full((N, K), 0x38, np.uint8)
    sa = np.full((1, 3), 0.5, np.float32)
    sb = np.array([[2.0, 4.0, 8.0]], np.float32)
    ref, _ = oracle.bsgemm("nt", a, b, sa, sb, M, N, K, g, a_fmt="e5m2", b_fmt="e4m3")
    assert np.all(ref == 128 * 0.5 * (2.0 + 4.0 + 8.0))


def test_e5m2_nonfinite_codes_are_reported():
    a = np.full((1, 16), 0x3C, np.uint8)
    b = np.full((1, 16), 0x3C, np.uint8)
    for bad in (0x7C, 0xFC, 0x7E):
        a2 = a.copy(); a2[0, 5] = bad
        with pytest.raises(RuntimeError):
            oracle.bsgemm("nt", a2, b, np.ones((1, 1), np.float32), np.ones((1, 1), np.float32),
                          1, 1, 16, 128, a_fmt="e5m2", b_fmt="e5m2")


def test_workload_quantiser_e5m2_round_trip():
    """The caller-side E5M2 quantiser: codes decode to values within E5M2 rounding of x / s."""
    rng = np.random.default_rng(3)
    x = rng.standard_normal((130, 200)).astype(np.float32)
    q, s = workloads.quantize_blocks(x, 64, "e5m2")
    dec = np.array(_dec_fmt("e5m2"))[q]
    scale = np.repeat(np.repeat(s, 64, axis=0), 64, axis=1)[:130, :200].astype(np.float64)
    back = dec * scale
    # E5M2 keeps 3 significant bits: relative rounding error <= 2^-3 for normal values
    assert np.all(np.abs(back - x) <= 2.0 ** -3 * np.abs(x) + scale * 2.0 ** -16)
    assert np.isclose(np.max(np.abs(dec)), 57344.0)


# --------------------------------------------------------------------------- quantiser (§4.4, §5.2)
@pytest.mark.parametrize("fmt,tdtype,fmax", [("e4m3", torch.float8_e4m3fn, 448.0),
                                             ("e5m2", torch.float8_e5m2, 57344.0)])
def test_fp8_encode_matches_torch_saturating_cast(fmt, tdtype, fmax):
    """torch's float32 -> float8 cast rounds to nearest even; clamping first
    makes it saturating, which is what the oracle's encoder must equal."""
    rng = np.random.default_rng(7)
    mags = rng.choice([1e-7, 1e-5, 1e-3, 0.1, 1.0, 30.0, 300.0, 3e4], size=8000).astype(np.float32)
    v = np.concatenate([rng.standard_normal(8000).astype(np.float32) * mags,
                        np.array([0.0, -0.0, fmax, -fmax, 2 * fmax, -3 * fmax], np.float32)])
    ours = np.array([oracle.fp8_encode(fmt, x) for x in v], np.uint8)
    ref = torch.from_numpy(np.clip(v, -fmax, fmax)).to(tdtype).view(torch.uint8).numpy()
    assert np.array_equal(ours, ref)


@pytest.mark.parametrize("fmt,v,code", [
    ("e4m3", 1.0625, 0x38), ("e4m3", 1.1875, 0x3A), ("e4m3", 3 * 2.0 ** -10, 0x02),  # ties -> even
    ("e4m3", 2.0 ** -10, 0x00), ("e4m3", -2.0 ** -11, 0x80), ("e4m3", 464.0, 0x7E),   # underflow, saturation
    ("e5m2", 1.125, 0x3C), ("e5m2", 1.375, 0x3E), ("e5m2", 61440.0, 0x7B), ("e5m2", -1e9, 0xFB),
])
def test_fp8_encode_hand_values(fmt, v, code):
    assert oracle.fp8_encode(fmt, v) == code


@pytest.mark.parametrize("fmt", ["e4m3", "e5m2"])
@pytest.mark.parametrize("rows,cols,g", [(130, 208, 64), (257, 384, 128), (96, 512, 256)])
def test_oracle_quantiser_matches_torch_quantiser(fmt, rows, cols, g):
    """The C quantiser against the torch one in workloads (amax, FP32 divide,
    clamp, cast): two independent restatements, bit for bit."""
    rng = np.random.default_rng(rows + cols)
    x = rng.standard_normal((rows, cols)).astype(np.float32) * np.float32(3.0)
    x[: min(g, rows), :g] = 0.0                      # an all-zero block -> scale 1
    x[-1, -5:] = np.float32(1e4)                     # a block dominated by outliers
    q1, s1 = oracle.quantize_blocks(x, g, fmt)
    q2, s2 = workloads.quantize_blocks(x, g, fmt)
    assert s1[0, 0] == 1.0
    assert np.array_equal(s1, s2) and np.array_equal(q1, q2)


def test_oracle_quantiser_round_trip_error():
    x = np.random.default_rng(2).standard_normal((128, 256)).astype(np.float32)
    q, s = oracle.quantize_blocks(x, 128, "e4m3")
    back = oracle.e4m3_table()[q] * np.repeat(np.repeat(s, 128, 0), 128, 1)
    # E4M3 keeps 4 significant bits: relative error <= 2^-4 above the subnormal range
    assert np.all(np.abs(back - x) <= 2.0 ** -4 * np.abs(x) + np.repeat(np.repeat(s, 128, 0), 128, 1) * 2.0 ** -9)


# --------------------------------------------------------------------------- fused epilogue (§2.3, §6)
def test_epilogue_hand_values():
    ref = np.array([[-2.0, -0.5, 0.0, 0.5, 1.0, 3.0]])
    bias = np.array([0.0, 0.0, 0.0, 0.25, -1.0, 0.0], np.float32)
    v, _ = oracle.epilogue(ref, bias, "relu")
    assert v.tolist() == [[0.0, 0.0, 0.0, 0.75, 0.0, 3.0]]
    v, _ = oracle.epilogue(ref, None, "gelu")
    want = [0.5 * x * (1.0 + math.erf(x / math.sqrt(2.0))) for x in ref[0]]
    assert np.allclose(v[0], want, rtol=0, atol=1e-15)
    assert abs(v[0, 4] - 0.8413447460685429) < 1e-15          # GELU(1) = Phi(1)
    v, bits = oracle.epilogue(ref, bias, None)
    assert np.array_equal(v, ref + bias.astype(np.float64))
    assert bits[0, 4] == oracle.bf16_rne(0.0)


def test_epilogue_all_zero_operands_give_act_of_bias():
    """A = 0: the product is exactly 0, so the output is act(bias) per column."""
    M, N, K, g = 3, 16, 128, 128
    a = np.zeros((M, K), np.uint8)
    b = np.full((N, K), 0x38, np.uint8)
    ref, _ = oracle.bsgemm("nt", a, b, np.ones((1, 1), np.float32), np.ones((1, 1), np.float32), M, N, K, g)
    bias = np.linspace(-2, 2, N).astype(np.float32)
    for act in (None, "relu", "gelu"):
        v, _ = oracle.epilogue(ref, bias, act)
        x = bias.astype(np.float64)
        want = x if act is None else (np.maximum(x, 0) if act == "relu" else
                                      0.5 * x * (1 + np.array([math.erf(t / math.sqrt(2)) for t in x])))
        assert np.allclose(v, np.broadcast_to(want, (M, N)), rtol=0, atol=1e-15)
