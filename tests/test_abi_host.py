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
    (4096, 4096, 4096, 128, 0), (1, 7168, 7168, 128, 1), (128, 7168, 7168, 128, 1),
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
    assert 1 <= pl["grid"] <= 148
    assert pl["grid"] == min(148, pl["tiles_p"] * pl["tiles_q"] * pl["splits"])


def test_plan_fills_the_machine_for_small_m():
    pl = bsg.make_plan(1, 7168, 7168, 128, "nt", 148)
    assert pl["tiles_p"] * pl["splits"] >= 100


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
    seen = 0
    for log in logs:
        cur = None
        for ln in open(log):
            m = re.search(r"Compiling entry function '_ZN3bsg13bsgemm_kernelILi(\d+)E", ln)
            if m:
                cur = int(m.group(1))
                continue
            if cur is not None and "Used" in ln:
                regs = int(re.search(r"Used (\d+) registers", ln).group(1))
                if cur == 256:
                    assert regs == 168, (log, ln)
                    seen += 1
                assert regs <= 168
                cur = None
    assert seen == 24   # 12 (granularity, layout) units x {split, no split}
