"""Mutation check of the oracle's pins (CPU only; not collected by pytest).

Each entry below plants one plausible mistake in a scratch copy of
``oracle/bsgemm_oracle.c`` -- a transposed index, a dropped term, a wrong sign,
bias or rounding rule -- and runs ``tests/test_oracle_pins.py`` against that
copy. The pins are doing their job when every mutant makes them fail.

    python tests/oracle_mutants.py            # all mutants, about 4 minutes
    python tests/oracle_mutants.py -k quant   # the ones whose name contains "quant"

The scratch copies live in the repository's git-ignored ``_build/`` folder and
are removed afterwards. Exit status 0 means every mutant was caught.
"""
from __future__ import annotations

import argparse
import os
import shutil
import subprocess
import sys
import tempfile

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# (name, text in bsgemm_oracle.c, replacement)
MUTANTS = [
    # ---- the block-scaled product
    ("transposed sA index", "sa[(m / g) * Kb + kb]", "sa[kb * ((M + g - 1) / g) + (m / g)]"),
    ("sB uses m block", "sb[(n / g) * Kb + kb]", "sb[(m % ((N + g - 1) / g)) * Kb + kb]"),
    ("drop last partial block", "int64_t k1 = k0 + g < K ? k0 + g : K;",
     "int64_t k1 = k0 + g < K ? k0 + g : k0;"),
    ("divide instead of multiply", "acc += ldexp((double)blocksum, -shift) * scale;",
     "acc += ldexp((double)blocksum, -shift) / scale;"),
    ("quantum off by one", "acc += ldexp((double)blocksum, -shift) * scale;",
     "acc += ldexp((double)blocksum, -shift + 1) * scale;"),
    ("TN A index", "return a[k * M + m];", "return a[m * K + k];"),
    ("NN B index", "return b[k * N + n];", "return b[n * K + k];"),
    ("BF16 via FP32", "if (fabs(x) < ldexp(1.0, -126)) {",
     "x = (double)(float)x; if (fabs(x) < ldexp(1.0, -126)) {"),
    # ---- E4M3 / E5M2 decode
    ("E4M3 subnormal", "mag = m;", "mag = m << 1;"),
    ("E4M3 exponent bias", "mag = (int64_t)(8 + m) << (e - 1);", "mag = (int64_t)(8 + m) << e;"),
    ("E4M3 sign dropped", "*units = s ? -mag : mag;", "*units = mag;"),
    ("E5M2 exponent bias", "mag = (int64_t)(4 + m) << (e - 1);", "mag = (int64_t)(4 + m) << e;"),
    ("E5M2 field split", "int e = (code >> 2) & 0x1F;", "int e = (code >> 3) & 0xF;"),
    # ---- encoder and quantiser
    ("encode ties to odd", "(err == best_err && (c & 1) == 0)", "(err == best_err && (c & 1) == 1)"),
    ("encode ties to the larger", "(err == best_err && (c & 1) == 0)", "(err == best_err)"),
    ("encode drops the sign", "best |= 0x80;", "best |= 0x00;"),
    ("quantise multiplies", "oracle_fp8_encode(fmt, x[r * cols + c] / s);",
     "oracle_fp8_encode(fmt, x[r * cols + c] * s);"),
    ("scale inverted", "s = amax > 0.0f ? amax / fmax : 1.0f;", "s = amax > 0.0f ? fmax / amax : 1.0f;"),
    ("scale by a rounded reciprocal", "s = amax > 0.0f ? amax / fmax : 1.0f;",
     "s = amax > 0.0f ? (float)((double)amax * (1.0 / 448.0)) : 1.0f;"),
    ("zero block scale", "s = amax > 0.0f ? amax / fmax : 1.0f;", "s = amax > 0.0f ? amax / fmax : 0.5f;"),
    ("scales transposed", "scales[rb * Cb + cb] = s;", "scales[cb * Rb + rb] = s;"),
    ("amax without abs", "float a = fabsf(x[r * cols + c]);", "float a = x[r * cols + c];"),
    ("partial block short a column", "int64_t c0 = cb * g, c1 = c0 + g < cols ? c0 + g : cols;",
     "int64_t c0 = cb * g, c1 = c0 + g < cols ? c0 + g : cols - 1;"),
    # ---- epilogue
    ("bias by row", "(bias ? (double)bias[n] : 0.0)", "(bias ? (double)bias[m % N] : 0.0)"),
    ("bias dropped", "(bias ? (double)bias[n] : 0.0)", "0.0"),
    ("ReLU flipped", "v = v > 0.0 ? v : 0.0;", "v = v < 0.0 ? v : 0.0;"),
    ("GELU tanh form", "v = 0.5 * v * (1.0 + erf(v / sqrt(2.0)));",
     "v = 0.5 * v * (1.0 + tanh(0.7978845608028654 * (v + 0.044715 * v * v * v)));"),
    ("GELU erf argument", "v = 0.5 * v * (1.0 + erf(v / sqrt(2.0)));",
     "v = 0.5 * v * (1.0 + erf(v * sqrt(2.0)));"),
]


def run_one(scratch: str, name: str, old: str, new: str) -> str:
    """'caught', 'survived' or 'stale' (the text to mutate is not in the oracle)."""
    work = os.path.join(scratch, "m")
    if os.path.isdir(work):
        shutil.rmtree(work)
    os.makedirs(work)
    for d in ("oracle", "workloads", "tests"):
        shutil.copytree(os.path.join(ROOT, d), os.path.join(work, d),
                        ignore=shutil.ignore_patterns("*.so", "__pycache__"))
    shutil.copy(os.path.join(ROOT, "pytest.ini"), work)
    src = os.path.join(work, "oracle", "bsgemm_oracle.c")
    text = open(src).read()
    if old not in text:
        return "stale"
    open(src, "w").write(text.replace(old, new, 1))
    r = subprocess.run([sys.executable, "-m", "pytest", "tests/test_oracle_pins.py", "-q", "-x",
                        "-p", "no:cacheprovider"], cwd=work, capture_output=True, text=True)
    return "caught" if r.returncode != 0 else "survived"


def main(argv=None) -> int:
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("-k", default="", help="run only mutants whose name contains this text")
    args = ap.parse_args(argv)
    base = os.path.join(ROOT, "_build")
    os.makedirs(base, exist_ok=True)
    scratch = tempfile.mkdtemp(prefix="oracle_mutants_", dir=base)
    bad = 0
    try:
        for name, old, new in MUTANTS:
            if args.k not in name:
                continue
            verdict = run_one(scratch, name, old, new)
            bad += verdict != "caught"
            print(f"{verdict:9s} {name}", flush=True)
    finally:
        shutil.rmtree(scratch, ignore_errors=True)
    print("all mutants caught" if not bad else f"{bad} mutant(s) not caught")
    return 1 if bad else 0


if __name__ == "__main__":
    sys.exit(main())
