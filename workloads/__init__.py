"""Seeded synthetic inputs for block-scaled FP8 GEMM.

This module is shared by the tests, the bench and the smoke check. It holds
none of the GEMM's arithmetic: it only draws FP32 matrices with the
distributions of the workloads below and prepares them the way a caller of
the library would (hncyxsy.com/news/191052 §4.4: quantisation happens outside
the GEMM library, with a granularity that must match the GEMM's).

Caller-side preparation, per g x g block of each operand:
  scale = amax / FMAX      (FMAX is the format's largest finite value: 448
                            for E4M3, 57344 for E5M2; a block whose amax is 0
                            gets scale 1.0)
  code  = FP8(clamp(x / scale, -FMAX, FMAX))   (round to nearest even)
The cast uses torch's ``float8_e4m3fn`` / ``float8_e5m2`` conversion; the
clamp makes it saturating. The scale tensors are row-major FP32
[ceil(rows/g), ceil(K/g)].

Workloads (synthetic stand-ins for the transformer projection / FFN GEMMs
the pages centre on; no dataset is involved):
  tiny     256^3, A ~ N(0,1), B ~ N(0,0.02)
  square   4096^3, as tiny but 1% of A's rows (41 rows, seeded permutation)
           multiplied by 50 before quantisation
  ffn      M=8192, N=14336, K=4096, A ~ Student-t(4), B ~ N(0,0.02)
  small_m  M in {1,8,32,64,128}, N=K=7168, A ~ N(0,1), B ~ N(0,0.02)
  long_k   M=2048, N=4096, K=32768, A ~ N(0,1) times a per-128x128-block
           std drawn as 2^U(-6,6), B ~ N(0,0.02)
Seeds: numpy PCG64 with ``seed`` for A and ``seed + 1`` for B (and
``seed + 2`` for any extra draw such as outlier rows or block stds).
"""
from __future__ import annotations

import dataclasses

import numpy as np
import torch

E4M3_MAX = 448.0
E5M2_MAX = 57344.0
FORMATS = {"e4m3": (E4M3_MAX, torch.float8_e4m3fn), "e5m2": (E5M2_MAX, torch.float8_e5m2)}

LAYOUTS = ("nt", "tn", "nn", "tt")


@dataclasses.dataclass
class Problem:
    """One GEMM's inputs, stored as the layout says, plus its logical shape."""
    M: int
    N: int
    K: int
    gran: int
    layout: str
    a: np.ndarray   # uint8 FP8 codes; [M,K] for layouts n?, [K,M] for t?
    b: np.ndarray   # uint8 FP8 codes; [N,K] for ?t, [K,N] for ?n
    sa: np.ndarray  # float32 [ceil(M/g), ceil(K/g)]
    sb: np.ndarray  # float32 [ceil(N/g), ceil(K/g)]
    name: str = ""
    a_fmt: str = "e4m3"
    b_fmt: str = "e4m3"

    @property
    def flops(self) -> int:
        return 2 * self.M * self.N * self.K


def quantize_blocks(x: np.ndarray, gran: int, fmt: str = "e4m3"):
    """Caller-side per-block FP8 quantisation of a logical [R, K] FP32 matrix.

    Returns (codes uint8 [R, K], scales float32 [ceil(R/g), ceil(K/g)]).
    """
    fmax, tdtype = FORMATS[fmt]
    x = np.ascontiguousarray(x, dtype=np.float32)
    R, K = x.shape
    Rb, Kb = -(-R // gran), -(-K // gran)
    t = torch.from_numpy(x)
    pad = torch.zeros((Rb * gran, Kb * gran), dtype=torch.float32)
    pad[:R, :K] = t
    blocks = pad.view(Rb, gran, Kb, gran)
    amax = blocks.abs().amax(dim=(1, 3))
    scale = torch.where(amax > 0, amax / fmax, torch.ones_like(amax))
    q = (blocks / scale[:, None, :, None]).clamp(-fmax, fmax)
    codes = q.view(Rb * gran, Kb * gran)[:R, :K].to(tdtype)
    return codes.view(torch.uint8).numpy().copy(), scale.numpy().astype(np.float32)


def store(codes_rk: np.ndarray, transposed: bool) -> np.ndarray:
    """Lay a logical [R, K] code matrix out as [R, K] or, transposed, [K, R]."""
    return np.ascontiguousarray(codes_rk.T if transposed else codes_rk)


def a_is_transposed(layout: str) -> bool:
    """First layout letter is A: 'n' -> stored [M,K], 't' -> stored [K,M]."""
    return layout[0] == "t"


def b_is_transposed(layout: str) -> bool:
    """Second letter is B: 't' -> stored [N,K] (the native NT form), 'n' -> [K,N]."""
    return layout[1] == "n"


def make_problem(M, N, K, gran=128, layout="nt", seed=0, a_dist="normal", b_std=0.02,
                 outlier_rows=0, outlier_mult=50.0, block_std_log2=None, name="",
                 a_fmt="e4m3", b_fmt="e4m3"):
    """Draw A [M,K] and B [N,K] in FP32, quantise per block, store per layout."""
    if layout not in LAYOUTS:
        raise ValueError(f"layout must be one of {LAYOUTS}")
    ra = np.random.Generator(np.random.PCG64(seed))
    rb = np.random.Generator(np.random.PCG64(seed + 1))
    rx = np.random.Generator(np.random.PCG64(seed + 2))
    if a_dist == "normal":
        a32 = ra.standard_normal((M, K), dtype=np.float32)
    elif a_dist == "student_t4":
        a32 = ra.standard_t(4.0, size=(M, K)).astype(np.float32)
    elif a_dist == "ones":
        a32 = np.ones((M, K), dtype=np.float32)
    else:
        raise ValueError(a_dist)
    if outlier_rows:
        rows = rx.permutation(M)[:outlier_rows]
        a32[rows] *= np.float32(outlier_mult)
    if block_std_log2 is not None:
        lo, hi = block_std_log2
        bm, bk = -(-M // 128), -(-K // 128)
        std = np.exp2(rx.uniform(lo, hi, size=(bm, bk))).astype(np.float32)
        a32 *= np.repeat(np.repeat(std, 128, axis=0), 128, axis=1)[:M, :K]
    b32 = (rb.standard_normal((N, K), dtype=np.float32) * np.float32(b_std))
    qa, sa = quantize_blocks(a32, gran, a_fmt)
    qb, sb = quantize_blocks(b32, gran, b_fmt)
    return Problem(M, N, K, gran, layout, store(qa, a_is_transposed(layout)),
                   store(qb, b_is_transposed(layout)), sa, sb, name, a_fmt, b_fmt)


def tiny(seed=0, layout="nt", gran=128):
    return make_problem(256, 256, 256, gran, layout, seed, name="tiny 256^3")


def square(seed=0, layout="nt", gran=128):
    return make_problem(4096, 4096, 4096, gran, layout, seed, outlier_rows=41,
                        name="square 4096^3, 41 outlier rows x50")


def ffn(seed=0, layout="nt", gran=128):
    return make_problem(8192, 14336, 4096, gran, layout, seed, a_dist="student_t4",
                        name="ffn up-projection 8192x14336x4096, A ~ t(4)")


def small_m(M, seed=0, layout="nt", gran=128):
    if M not in (1, 8, 32, 64, 128):
        raise ValueError("small-M sweep uses M in {1, 8, 32, 64, 128}")
    return make_problem(M, 7168, 7168, gran, layout, seed, name=f"small-M {M}x7168x7168")


def long_k(gran=128, seed=0, layout="nt"):
    return make_problem(2048, 4096, 32768, gran, layout, seed, block_std_log2=(-6.0, 6.0),
                        name=f"long-K 2048x4096x32768 g={gran}")


@dataclasses.dataclass
class GroupedProblem:
    """Inputs of one grouped NT call: group i multiplies its M_i rows of A by
    its own B_i; A's rows and A's scale blocks are stacked group after group."""
    ms: list            # rows per group
    N: int
    K: int
    gran: int
    a: np.ndarray       # uint8 [sum M_i, K]
    sa: np.ndarray      # float32 [sum ceil(M_i/g) + len(ms), Kb] (group i's blocks from row S_i)
    b: np.ndarray       # uint8 [G, N, K]
    sb: np.ndarray      # float32 [G, ceil(N/g), Kb]
    parts: list         # each group's own Problem (its A rows and scales, its B)
    name: str = ""

    @property
    def flops(self) -> int:
        return 2 * sum(self.ms) * self.N * self.K


def grouped_moe(seed=0, groups=8, tokens=8192, N=4096, K=7168, gran=128):
    """A mixture-of-experts up-projection: `tokens` rows routed to `groups`
    experts in seeded, uneven shares (Dirichlet(1) proportions, multinomial
    counts), each expert with its own [N, K] weights."""
    rng = np.random.Generator(np.random.PCG64(seed + 1000))
    ms = [int(m) for m in rng.multinomial(tokens, rng.dirichlet(np.ones(groups)))]
    parts = [make_problem(max(m, 1), N, K, gran, "nt", seed + 10 * i) for i, m in enumerate(ms)]
    kb = -(-K // gran)
    a = np.zeros((tokens, K), np.uint8)
    sa = np.ones((-(-tokens // gran) + groups, kb), np.float32)
    r = sr = 0
    for m, p in zip(ms, parts):
        if m:
            a[r:r + m] = p.a[:m]
            sa[sr:sr + -(-m // gran)] = p.sa[:-(-m // gran)]
        r += m
        sr += -(-m // gran)
    b = np.stack([p.b for p in parts])
    sb = np.stack([p.sb for p in parts])
    return GroupedProblem(ms, N, K, gran, a, sa, b, sb, parts,
                          f"grouped MoE up-projection: {tokens} rows over {groups} experts, "
                          f"N={N}, K={K}, g={gran}")


def logical_a(p: Problem) -> np.ndarray:
    """A's codes as the logical [M, K] matrix, whatever the storage layout."""
    return np.ascontiguousarray(p.a.T) if a_is_transposed(p.layout) else p.a


def logical_b(p: Problem) -> np.ndarray:
    """B's codes as the logical [N, K] matrix, whatever the storage layout."""
    return np.ascontiguousarray(p.b.T) if b_is_transposed(p.layout) else p.b


def relayout(p: Problem, layout: str) -> Problem:
    """The same logical problem stored in another layout."""
    return Problem(p.M, p.N, p.K, p.gran, layout,
                   store(logical_a(p), a_is_transposed(layout)),
                   store(logical_b(p), b_is_transposed(layout)), p.sa, p.sb, p.name, p.a_fmt, p.b_fmt)


def sample_indices(M, N, count, seed=0, include_corners=True):
    """Seeded output positions for sampled parity checks at large sizes.

    Always includes the four corners and the last row/column of each
    128-tile boundary region, so ragged tails are sampled."""
    r = np.random.Generator(np.random.PCG64(seed + 7))
    mi = r.integers(0, M, size=count, dtype=np.int64)
    ni = r.integers(0, N, size=count, dtype=np.int64)
    if include_corners:
        cm = np.array([0, 0, M - 1, M - 1, M // 2, min(M - 1, 127), min(M - 1, 128)], dtype=np.int64)
        cn = np.array([0, N - 1, 0, N - 1, N // 2, min(N - 1, 255), min(N - 1, 256)], dtype=np.int64)
        mi = np.concatenate([cm, mi])
        ni = np.concatenate([cn, ni])
    return mi, ni
