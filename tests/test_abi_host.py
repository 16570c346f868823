"""The C ABI library, checked without a GPU: it loads, exports every symbol
include/bsgemm.h declares, and its host-only plan logic behaves."""
import ctypes
import glob
import os
import re

import pytest

import fp8_block_scaled_bsgemm_b200 as bsg
from fp8_block_scaled_bsgemm_b200 import build as bsg_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _header_functions():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names |= set(re.findall(r"\b(bsgemm_\w+)\s*\(", text))
    return names


def test_library_exports_every_declared_symbol():
    L = bsg.lib()
    declared = _header_functions()
    assert declared, "no declarations found"
    missing = [n for n in sorted(declared) if not hasattr(L, n)]
    assert not missing, missing
    assert set(bsg.EXPORTS) <= declared


def test_status_strings_and_version():
    for s in range(7):
        assert bsg.status_string(s)
    assert bsg.lib().bsgemm_version() >= 100


@pytest.mark.parametrize("M,N,K,gran,want_swap", [
    (4096, 4096, 4096, 128, 0), (1, 7168, 7168, 128, 1), (64, 7168, 7168, 128, 1), (128, 7168, 7168, 128, 0),
    (8192, 14336, 4096, 128, 0), (2048, 4096, 32768, 64, 0), (7, 1000, 656, 256, 1)])
def test_plan_is_consistent(M, N, K, gran, want_swap):
    pl = bsg.make_plan(M, N, K, gran, "nt", 148)
    assert pl["swap_ab"] == want_swap
    P, Q = (N, M) if pl["swap_ab"] else (M, N)
    assert pl["tiles_p"] == -(-P // 128) and pl["tiles_q"] == -(-Q // pl["bnq"])
    Kb = -(-K // gran)
    assert pl["splits"] * pl["kb_per_split"] >= Kb > (pl["splits"] - 1) * pl["kb_per_split"]
    if gran == 64:
        assert pl["kb_per_split"] % 2 == 0 or pl["splits"] == 1
    tiles = pl["tiles_p"] * pl["tiles_q"]
    U = -(-Kb // (2 if gran == 64 else 1))
    assert pl["sk_units_per_tile"] == U
    assert 1 <= pl["grid"] <= 148
    if pl["sk_ctas"] > 0:
        # whole tiles in full waves, then the rest shared out by stream-K
        assert pl["splits"] == 1 and pl["sk_first_tile"] % 148 == 0
        assert pl["sk_units"] == (tiles - pl["sk_first_tile"]) * U
        assert 1 <= pl["sk_ctas"] <= min(148, pl["sk_units"])
        assert pl["grid"] == min(148, max(pl["sk_first_tile"], pl["sk_ctas"]))
    else:
        assert pl["grid"] == min(148, tiles * pl["splits"])


def test_plan_fills_the_machine_for_small_m():
    pl = bsg.make_plan(1, 7168, 7168, 128, "nt", 148)
    assert max(pl["tiles_p"] * pl["splits"], pl["sk_ctas"]) >= 100


def test_plan_uses_stream_k_for_a_ragged_last_wave():
    # long K, single-CTA tiles: 256 tiles = 1 wave + 108, whose units are shared out
    dp = {"variant": "data_parallel"}
    pl = bsg.make_plan(2048, 4096, 32768, 128, "nt", 148, dp)
    assert pl["sk_first_tile"] == 148 and pl["sk_ctas"] == 148
    assert bsg.make_plan(2048, 4096, 32768, 64, "nt", 148)["sk_ctas"] == 148
    assert bsg.make_plan(2048, 4096, 32768, 128, "nt", 148, {"stream_k": -1})["sk_ctas"] == 0
    assert bsg.make_plan(2048, 4096, 32768, 128, "nt", 148, {"splits": 2})["sk_ctas"] == 0
    # short K (32 K-blocks): whole tiles unless forced
    assert bsg.make_plan(4096, 4096, 4096, 128, "nt", 148)["sk_ctas"] == 0
    forced = bsg.make_plan(4096, 4096, 4096, 128, "nt", 148, {"stream_k": 1})
    assert forced["sk_first_tile"] == 444 and forced["sk_ctas"] == 148
    # fewer tiles than SMs: stream-K, whatever the tile width; split-K when
    # stream-K is turned off
    assert bsg.make_plan(128, 7168, 7168, 128, "nt", 148)["sk_ctas"] == 148
    assert bsg.make_plan(16, 7168, 7168, 128, "nt", 148)["sk_ctas"] == 148
    assert bsg.make_plan(1, 7168, 7168, 128, "nt", 148)["sk_ctas"] == 148
    small = bsg.make_plan(16, 7168, 7168, 128, "nt", 148, {"stream_k": -1})
    assert small["sk_ctas"] == 0 and small["splits"] > 1
    # an exact number of full waves needs no stream-K
    assert bsg.make_plan(128 * 148, 256, 1024, 128, "nt", 148, {"stream_k": 1})["sk_ctas"] == 0


def test_plan_for_cta_pairs():
    pl = bsg.make_plan(4096, 4096, 4096, 128, "nt", 148, {"variant": "cta_pair"})
    assert pl["cta_pair"] == 1 and pl["bnq"] == 256 and pl["splits"] == 1 and pl["sk_ctas"] == 0
    assert (pl["tiles_p"], pl["tiles_q"]) == (16, 16) and pl["grid"] == 148
    small = bsg.make_plan(300, 200, 64, 64, "tn", 148, {"variant": "cta_pair"})
    assert (small["tiles_p"], small["tiles_q"], small["grid"]) == (2, 1, 4)
    for bad in ({"variant": "cta_pair", "bnq": 128}, {"variant": "cta_pair", "splits": 2},
                {"variant": "cta_pair", "stream_k": 1}):
        with pytest.raises(bsg.BsgemmError):
            bsg.make_plan(4096, 4096, 4096, 128, "nt", 148, bad)
    assert bsg.make_plan(4096, 4096, 4096, 128, "nt", 148)["cta_pair"] == 0
    # the heuristic takes CTA pairs at g = 256, and at g = 128 for long K, with a
    # full wave of 256 x 256 tiles
    assert bsg.make_plan(2048, 4096, 32768, 256, "nt", 148)["cta_pair"] == 1
    assert bsg.make_plan(2048, 4096, 32768, 128, "nt", 148)["cta_pair"] == 1
    assert bsg.make_plan(2048, 4096, 32768, 64, "nt", 148)["cta_pair"] == 0
    assert bsg.make_plan(8192, 14336, 4096, 128, "nt", 148)["cta_pair"] == 0
    assert bsg.make_plan(512, 512, 4096, 256, "nt", 148)["cta_pair"] == 0          # 4 pair tiles
    assert bsg.make_plan(2048, 4096, 32768, 256, "nt", 148, {"stream_k": -1})["cta_pair"] == 0


def _sk_partition(tiles_sk, U, G):
    """Mirror of the kernel's stream-K walk (sk_start, sk_owner, piece slots)."""
    R = tiles_sk * U
    q, r = divmod(R, G)
    start = lambda c: c * q + min(c, r)
    owner = lambda u: u // (q + 1) if u < r * (q + 1) else r + (u - r * (q + 1)) // q
    assert start(G) == R and all(owner(u) == max(c for c in range(G) if start(c) <= u) for u in range(R))
    pieces = {}
    for c in range(G):
        u, ue = start(c), start(c + 1)
        while u < ue:
            t = u // U
            t0 = t * U
            se = min(ue, t0 + U)
            slot = 2 * c + (0 if start(c) // U == t else 1)
            pieces.setdefault(t, []).append((c, u - t0, se - t0, slot, owner(t0), owner(t0 + U - 1)))
            u = se
    return pieces, start


@pytest.mark.parametrize("tiles_sk,U,G", [(68, 32, 148), (56, 56, 148), (108, 256, 148), (1, 2, 1),
                                          (3, 5, 7), (32, 32, 148), (5, 3, 4), (16, 64, 148)])
def test_stream_k_partition_covers_each_tile_once_in_k_order(tiles_sk, U, G):
    pieces, start = _sk_partition(tiles_sk, U, G)
    assert sorted(pieces) == list(range(tiles_sk))
    used = set()
    for t, ps in pieces.items():
        # contiguous cover of [0, U) by CTAs in increasing order
        assert ps[0][1] == 0 and ps[-1][2] == U
        for a, b in zip(ps, ps[1:]):
            assert a[2] == b[1] and b[0] == a[0] + 1
        first, last = ps[0][4], ps[0][5]
        assert [p[0] for p in ps] == list(range(first, last + 1))
        if len(ps) > 1:
            for j, p in enumerate(ps):
                # the slot the reducer computes for piece j is the one the piece wrote
                c = first + j
                assert p[3] == 2 * c + (0 if start(c) // U == t else 1)
                assert p[3] not in used
                used.add(p[3])
            # The reducer is piece 0's CTA, and piece 0 is the last segment of
            # its CTA's range; every later piece is the first segment of its
            # CTA's range.  So a reducer waits only on pieces their CTAs reach
            # before any wait of their own: no cycle of waits.
            c0 = ps[0][0]
            assert ps[0][1] == 0 and start(c0 + 1) == t * U + ps[0][2]
            for p in ps[1:]:
                assert start(p[0]) == t * U + p[1]


def test_plan_rejects_bad_tuning():
    with pytest.raises(bsg.BsgemmError):
        bsg.make_plan(256, 256, 256, 128, "nt", 148, {"variant": "data_parallel", "bnq": 64})
    with pytest.raises(bsg.BsgemmError):
        bsg.make_plan(256, 256, 256, 96, "nt", 148)


def test_argument_errors_are_reported_before_touching_a_device():
    L = bsg.lib()
    # null pointers and bad sizes are rejected on the host, no CUDA call made
    assert L.bsgemm_fp8_nt(None, None, None, None, None, 1, 1, 1, 128, None) == 1
    assert L.bsgemm_fp8_tn(16, 16, 16, 16, 16, 1, 16, 16, 128, None) == 3   # M % 16 for A stored [K,M]
    assert L.bsgemm_fp8_nt(16, 16, 16, 16, 16, 16, 16, 16, 100, None) == 2


def test_register_split_kernels_have_the_planned_launch_registers():
    """setmaxnreg in the widest tiles needs exactly 168 launch registers; the
    host also checks this before launching, this catches it at build time."""
    bsg_build.build()
    logs = glob.glob(os.path.join(ROOT, "_build", "bsgemm_inst_g*.log"))
    assert len(logs) == 12
    seen = pairs = 0
    for log in logs:
        cur = None
        for ln in open(log):
            m = re.search(r"Compiling entry function '_ZN3bsg13bsgemm_kernelILi(\d+)E", ln)
            if m:
                cur = int(m.group(1))
                continue
            if "Compiling entry function '_ZN3bsg18bsgemm_pair_kernel" in ln:
                cur = -1   # CTA-pair tiles: always the 256-wide register split
                continue
            if cur is not None and "Used" in ln:
                regs = int(re.search(r"Used (\d+) registers", ln).group(1))
                if cur in (256, -1):
                    assert regs == 168, (log, ln)
                    seen += cur == 256
                    pairs += cur == -1
                assert regs <= 168
                cur = None
    # 12 (granularity, layout) units x {split, no split}, plus the grouped
    # instance in each of the 3 NT units; one CTA-pair kernel per unit
    assert seen == 24 + 3
    assert pairs == 12
    # the allocation-free unit instantiates its own split kernels: one
    # 256-wide instance per granularity, under the same rule
    wide = 0
    cur = None
    for ln in open(os.path.join(ROOT, "_build", "bsgemm_noalloc.o.log")):
        m = re.search(r"Compiling entry function '_ZN3bsg13bsgemm_kernelILi(\d+)E", ln)
        if m:
            cur = int(m.group(1))
            continue
        if cur is not None and "Used" in ln:
            regs = int(re.search(r"Used (\d+) registers", ln).group(1))
            assert regs == 168 if cur == 256 else regs <= 168, ln
            wide += cur == 256
            cur = None
    assert wide == 3


def test_new_entry_points_reject_bad_arguments_on_the_host():
    """Formats, epilogue options, quantiser and grouped arguments are checked
    before any CUDA call (no device is touched here)."""
    L = bsg.lib()
    A = 256  # a 16-byte aligned stand-in address; nothing is dereferenced
    # unknown FP8 format
    assert L.bsgemm_fp8_gemm_fmt(0, 2, 0, A, A, A, A, A, 16, 16, 16, 128, None, None) == 1
    assert L.bsgemm_fp8_gemm_fmt(0, 0, -1, A, A, A, A, A, 16, 16, 16, 128, None, None) == 1
    # epilogue: unknown activation, unknown output type, misaligned bias
    epi = bsg.Epilogue(None, 7, 0)
    assert L.bsgemm_fp8_gemm_fused(0, 0, 0, A, A, A, A, ctypes.byref(epi), A, 16, 16, 16, 128, None, None) == 1
    epi = bsg.Epilogue(None, 1, 5)
    assert L.bsgemm_fp8_gemm_fused(0, 0, 0, A, A, A, A, ctypes.byref(epi), A, 16, 16, 16, 128, None, None) == 1
    epi = bsg.Epilogue(A + 2, 0, 0)
    assert L.bsgemm_fp8_gemm_fused(0, 0, 0, A, A, A, A, ctypes.byref(epi), A, 16, 16, 16, 128, None, None) == 3
    # quantiser: null pointer, bad source type, bad gran, cols % 16, misaligned source
    assert L.bsgemm_quantize_fp8(0, 0, None, 16, 16, 128, A, A, None) == 1
    assert L.bsgemm_quantize_fp8(3, 0, A, 16, 16, 128, A, A, None) == 1
    assert L.bsgemm_quantize_fp8(0, 0, A, 16, 16, 96, A, A, None) == 2
    assert L.bsgemm_quantize_fp8(0, 0, A, 16, 40, 128, A, A, None) == 3
    assert L.bsgemm_quantize_fp8(1, 1, A + 8, 16, 32, 128, A, A, None) == 3
    # grouped: no groups, no rows, misaligned group sizes, K % 16
    assert L.bsgemm_fp8_grouped_nt(0, 0, A, A, A, A, A, A, 0, 64, 128, 128, 128, None) == 1
    assert L.bsgemm_fp8_grouped_nt(0, 0, A, A, A, A, A, A, 2, 0, 128, 128, 128, None) == 1
    assert L.bsgemm_fp8_grouped_nt(0, 0, A, A, A, A, A, A + 2, 2, 64, 128, 128, 128, None) == 3
    assert L.bsgemm_fp8_grouped_nt(0, 0, A, A, A, A, A, A, 2, 64, 128, 40, 128, None) == 3


def test_binding_rejects_host_tensors_before_calling_the_library():
    """The binding hands bare pointers to the kernels: a host tensor is refused
    in Python, with nothing passed to the library."""
    import torch
    a = torch.zeros((128, 256), dtype=torch.uint8)
    s = torch.ones((1, 2))
    with pytest.raises(ValueError):
        bsg.gemm(a, a, s, s)
    with pytest.raises(ValueError):
        bsg.quantize(torch.zeros((128, 256)), 128)
    with pytest.raises(ValueError):
        bsg.grouped_gemm(a, a.reshape(1, 128, 256), torch.ones((2, 2)), s,
                         torch.zeros(1, dtype=torch.int32))


def test_plan_rejects_sizes_past_its_32_bit_counts():
    """Tile and work-item counts are 32-bit in the launch; a size or forced
    split count that would overflow them is refused, not truncated."""
    for M, N, K in ((1 << 31, 256, 256), (256, (1 << 30) + 8, 256), (256, 256, 1 << 31)):
        with pytest.raises(bsg.BsgemmError) as e:
            bsg.make_plan(M, N, K, 128, "nt", 148)
        assert e.value.status == 1
    with pytest.raises(bsg.BsgemmError):          # 2^45 tiles of 128 x 256
        bsg.make_plan(1 << 30, 1 << 30, 128, 128, "nt", 148)
    # 2^20 tiles x 2^14 forced K splits = 2^34 work items
    with pytest.raises(bsg.BsgemmError):
        bsg.make_plan(1 << 20, 1 << 15, 1 << 20, 64, "nt", 148, {"splits": 1 << 14})
    # the largest sizes themselves still plan
    pl = bsg.make_plan(1 << 30, 256, 1 << 30, 128, "nt", 148, {"variant": "data_parallel"})
    assert pl["tiles_p"] == (1 << 23) and pl["tiles_q"] == 1 and pl["splits"] == 1
    pl = bsg.make_plan(1 << 30, 256, 1 << 30, 128, "nt", 148)     # long K: CTA pairs
    assert pl["cta_pair"] == 1 and pl["tiles_p"] == (1 << 22) and pl["tiles_q"] == 1


def test_allocation_free_plan_never_pairs_ctas():
    """bsgemm_fp8_nt_noalloc launches single-CTA tiles only. Where the regular
    plan pairs CTAs (large g = 256 problems) it re-plans with the data-parallel
    variant named, which keeps the regular stream-K choice and has no pairs."""
    pl = bsg.make_plan(2304, 2304, 1024, 256, "nt", 148)
    assert pl["cta_pair"] == 1 and (pl["tiles_p"], pl["tiles_q"]) == (9, 9)
    dp = bsg.make_plan(2304, 2304, 1024, 256, "nt", 148, {"variant": "data_parallel"})
    assert dp["cta_pair"] == 0 and dp["swap_ab"] == 0 and dp["bnq"] == 256
    assert (dp["tiles_p"], dp["tiles_q"]) == (18, 9)
    # the fallback plan without stream-K never pairs either
    assert bsg.make_plan(2304, 2304, 1024, 256, "nt", 148, {"stream_k": -1})["cta_pair"] == 0


def _cdiv(a, b):
    return -(-a // b)


def _grouped_walk(ms, tiles_q, grid, gran):
    """Mirror of the grouped kernel's work cursor (work_begin / group_seek /
    work_next with GROUPED): per CTA, the (group, tp, tq, g_row, g_srow, g_m)
    of each tile it takes."""
    BM = 128
    items = []
    for cta in range(grid):
        wi, g, g_first, g_row, g_srow = cta, 0, 0, 0, 0
        g_m = max(0, ms[0])
        g_tiles = _cdiv(g_m, BM) * tiles_q
        while True:
            alive = True
            while wi >= g_first + g_tiles:
                g_first += g_tiles
                g_row += g_m
                g_srow += _cdiv(g_m, gran)
                g += 1
                if g >= len(ms):
                    alive = False
                    break
                g_m = max(0, ms[g])
                g_tiles = _cdiv(g_m, BM) * tiles_q
            if not alive:
                break
            lt = wi - g_first
            tiles_p = _cdiv(g_m, BM)
            items.append((cta, g, lt % tiles_p, lt // tiles_p, g_row, g_srow, g_m))
            wi += grid
    return items


@pytest.mark.parametrize("seed", range(6))
def test_grouped_cursor_covers_each_tile_once_inside_its_group(seed):
    import random
    rng = random.Random(seed)
    for _ in range(25):
        G = rng.randint(1, 12)
        ms = [rng.choice([0, 0, 1, 5, 127, 128, 129, 300, 513]) for _ in range(G)]
        gran = rng.choice([64, 128, 256])
        bnq = rng.choice([128, 256])
        N = rng.choice([128, 256, 384, 1000])
        tiles_q = _cdiv(N, bnq)
        max_rows = sum(ms) + rng.choice([0, 1, 40])
        grid = rng.choice([1, 3, 148])
        items = _grouped_walk(ms, tiles_q, grid, gran)
        want = {(g, tp, tq) for g, m in enumerate(ms) for tp in range(_cdiv(m, 128)) for tq in range(tiles_q)}
        got = [(g, tp, tq) for _, g, tp, tq, _, _, _ in items]
        assert len(got) == len(set(got)) and set(got) == want, (ms, grid)
        Pb = _cdiv(max_rows, gran) + G          # scale_a rows the call documents
        for _, g, tp, tq, g_row, g_srow, g_m in items:
            assert g_row == sum(ms[:g]) and g_m == ms[g]
            assert g_srow == sum(_cdiv(m, gran) for m in ms[:g])
            # each promotion warp's scale row (clamped as the kernel does) is one of
            # the group's own rows, inside the documented scale_a bound
            last = max(0, (g_m - 1) // gran)
            for quad in range(4):
                pb = g_srow + min((tp * 128 + quad * 32) // gran, last)
                pb = min(pb, Pb - 1)
                assert g_srow <= pb <= g_srow + _cdiv(g_m, gran) - 1 <= Pb - 1
            # rows stored: the tile's rows that lie in the group, all below max_rows
            lo, hi = g_row + tp * 128, g_row + min(g_m, tp * 128 + 128)
            assert g_row <= lo < hi <= g_row + g_m <= max_rows


def test_automatic_plan_works_for_any_sm_count():
    """The heuristic only pairs CTAs where pairs can run (two SMs or more); the
    plan for one SM is a plain single-CTA plan."""
    for sms in (1, 2, 3, 148):
        for M, N, K, g in ((4096, 4096, 4096, 256), (1, 7168, 7168, 128), (300, 200, 64, 64)):
            pl = bsg.make_plan(M, N, K, g, "nt", sms)
            assert 1 <= pl["grid"] <= sms
            assert pl["cta_pair"] == 0 or sms >= 2


def _tile_coords(tiles_p, tiles_q, group_p, tile):
    """Mirror of the kernels' grouped raster (tile_coords)."""
    per_group = group_p * tiles_q
    grp = tile // per_group
    first_p = grp * group_p
    rows = min(tiles_p - first_p, group_p)
    local = tile - grp * per_group
    return first_p + local % rows, local // rows


@pytest.mark.parametrize("group_p", [1, 8, 16])
def test_raster_maps_work_items_onto_the_tile_grid_one_to_one(group_p):
    """Every tile index in [0, tiles) names a distinct tile of the grid (the
    last, shorter group of rows included), and the tiles a group's CTAs take
    together share their B (Q-side) tile column."""
    import random
    rng = random.Random(group_p)
    for _ in range(200):
        tp_n, tq_n = rng.randint(1, 70), rng.randint(1, 70)
        seen = [_tile_coords(tp_n, tq_n, group_p, t) for t in range(tp_n * tq_n)]
        assert sorted(seen) == [(a, b) for a in range(tp_n) for b in range(tq_n)]
        per_group = group_p * tq_n
        for t in range(tp_n * tq_n - 1):
            (a0, b0), (a1, b1) = seen[t], seen[t + 1]
            if t // per_group == (t + 1) // per_group and a1 == a0 + 1:
                assert b1 == b0              # next row of the same group: same B column


@pytest.mark.parametrize("M,N,K,want_bnq", [
    (4096, 4096, 4096, 256), (8192, 14336, 4096, 256),      # many tiles: 256 wide
    (128, 7168, 7168, 128), (256, 4096, 7168, 128),          # few tiles, 128-wide ones fit one wave
    (384, 7168, 7168, 256), (512, 7168, 7168, 256),          # 128-wide tiles would spill past a wave
    (768, 7168, 7168, 128), (1280, 4096, 2048, 128),         # whole tiles: 3 waves of 128 beat 2 of 256
    (2048, 4096, 32768, 256),                                 # long K: stream-K evens the waves at 256
    (96, 100, 4096, 128)])                                    # N <= 128
def test_data_parallel_width(M, N, K, want_bnq):
    pl = bsg.make_plan(M, N, K, 128, "nt", 148, {"variant": "data_parallel"})
    assert pl["bnq"] == want_bnq, pl
