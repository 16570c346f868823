"""The quantiser's fast quotient for BF16 input, checked for every input.

``tests/quant_division_model.c`` runs the quotient steps of
``csrc/bsgemm_quant.cu`` (Markstein's correction of x * RN(1/s)) in IEEE
single precision. It covers every BF16 block amax and every BF16 x with
|x| <= amax, for both FP8 formats, about 1.9e9 pairs, and compares with the
correctly rounded x / s that the pages' quantiser divides by
(hncyxsy.com/news/191052 §5.2: quantisation divides by the scale). The GPU
tests then check the kernel itself against the oracle, bit for bit.
"""
import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))


def test_fast_quotient_matches_division_for_every_bf16_input(tmp_path):
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    exe = str(tmp_path / "quant_division_model")
    flags = ["-O2", "-ffp-contract=off", "-std=c99"]
    omp = subprocess.run([cc, *flags, "-fopenmp", os.path.join(HERE, "quant_division_model.c"), "-o", exe, "-lm"],
                         capture_output=True, text=True)
    if omp.returncode != 0:   # no OpenMP runtime: one thread
        subprocess.run([cc, *flags, os.path.join(HERE, "quant_division_model.c"), "-o", exe, "-lm"],
                       check=True, capture_output=True, text=True)
    run = subprocess.run([exe], capture_output=True, text=True, timeout=900)
    assert run.returncode == 0, run.stdout + run.stderr
    lines = [l for l in run.stdout.splitlines() if "pairs" in l]
    assert len(lines) == 2 and all(", 0 differ" in l for l in lines), run.stdout
