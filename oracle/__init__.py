"""Plain CPU oracle for block-scaled FP8 GEMM (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
leg (and its ``--impl reference`` arm) may import this package.  The product
path (``fp8_block_scaled_bsgemm_b200``) never imports it and shares no code
with it: the arithmetic lives in ``bsgemm_oracle.c``; this module only
compiles that file with the host C compiler and marshals numpy arrays.

What the oracle computes is stated in the header of ``bsgemm_oracle.c``
(hncyxsy.com/news/191052, §2.2 block scaling, §3.1 granularity, §3.2
segment-wise FP32 accumulation, §4.2 API and layouts, §5.2 scale direction).

Parity pins: ``tests/test_oracle_pins.py`` and ``tests/golden/``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "bsgemm_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

LAYOUTS = {"nt": 0, "tn": 1, "nn": 2, "tt": 3}
FORMATS = {"e4m3": 0, "e5m2": 1}


def build(force: bool = False) -> str:
    """Compile ``bsgemm_oracle.c`` into ``liboracle.so`` (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-Wall", "-Wextra",
               "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            p = ctypes.c_void_p
            i64 = ctypes.c_int64
            lib.oracle_e4m3_value.restype = ctypes.c_double
            lib.oracle_e4m3_value.argtypes = [ctypes.c_uint8]
            lib.oracle_bf16_rne.restype = ctypes.c_uint16
            lib.oracle_bf16_rne.argtypes = [ctypes.c_double]
            lib.oracle_bsgemm.restype = ctypes.c_int
            lib.oracle_bsgemm.argtypes = [ctypes.c_int, p, p, p, p, i64, i64, i64, i64, p, p]
            lib.oracle_bsgemm_at.restype = ctypes.c_int
            lib.oracle_bsgemm_at.argtypes = [ctypes.c_int, p, p, p, p, i64, i64, i64, i64, i64,
                                             p, p, p, p]
            lib.oracle_fp8_value.restype = ctypes.c_double
            lib.oracle_fp8_value.argtypes = [ctypes.c_int, ctypes.c_uint8]
            i32 = ctypes.c_int
            lib.oracle_bsgemm_fmt.restype = ctypes.c_int
            lib.oracle_bsgemm_fmt.argtypes = [i32, i32, i32, p, p, p, p, i64, i64, i64, i64, p, p]
            lib.oracle_bsgemm_at_fmt.restype = ctypes.c_int
            lib.oracle_bsgemm_at_fmt.argtypes = [i32, i32, i32, p, p, p, p, i64, i64, i64, i64, i64,
                                                 p, p, p, p]
            lib.oracle_fp8_encode.restype = ctypes.c_uint8
            lib.oracle_fp8_encode.argtypes = [i32, ctypes.c_float]
            lib.oracle_quantize_blocks.restype = ctypes.c_int
            lib.oracle_quantize_blocks.argtypes = [i32, p, i64, i64, i64, p, p]
            lib.oracle_epilogue.restype = ctypes.c_int
            lib.oracle_epilogue.argtypes = [p, i64, i64, p, i32, p, p]
            lib.oracle_num_threads.restype = ctypes.c_int
            lib.oracle_num_threads.argtypes = []
            _lib = lib
    return _lib


def _ptr(x: np.ndarray):
    return x.ctypes.data_as(ctypes.c_void_p)


def e4m3_value(code: int) -> float:
    """Exact value of one E4M3 code (NaN for 0x7F / 0xFF)."""
    return _load().oracle_e4m3_value(int(code))


def e4m3_table() -> np.ndarray:
    """All 256 E4M3 codes decoded to float64."""
    return np.array([e4m3_value(c) for c in range(256)], dtype=np.float64)


def fp8_value(fmt: str, code: int) -> float:
    """Exact value of one code of format ``fmt`` ("e4m3" or "e5m2")."""
    return _load().oracle_fp8_value(FORMATS[fmt], int(code))


def fp8_table(fmt: str) -> np.ndarray:
    """All 256 codes of ``fmt`` decoded to float64 (E5M2: +-Inf and NaN codes included)."""
    return np.array([fp8_value(fmt, c) for c in range(256)], dtype=np.float64)


def bf16_rne(x: float) -> int:
    """BF16 bit pattern of ``x`` rounded once, to nearest-even, from FP64."""
    return int(_load().oracle_bf16_rne(float(x)))


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def _check_inputs(layout, a, b, sa, sb, M, N, K, gran):
    if layout not in LAYOUTS:
        raise ValueError(f"layout must be one of {sorted(LAYOUTS)}")
    a = np.ascontiguousarray(a, dtype=np.uint8)
    b = np.ascontiguousarray(b, dtype=np.uint8)
    sa = np.ascontiguousarray(sa, dtype=np.float32)
    sb = np.ascontiguousarray(sb, dtype=np.float32)
    kb = -(-K // gran)
    if a.size != M * K or b.size != N * K:
        raise ValueError("operand sizes do not match M, N, K")
    if sa.size != -(-M // gran) * kb or sb.size != -(-N // gran) * kb:
        raise ValueError("scale sizes do not match the granularity")
    return a, b, sa, sb


def bsgemm(layout: str, a, b, sa, sb, M: int, N: int, K: int, gran: int, a_fmt="e4m3", b_fmt="e4m3"):
    """Full oracle product. Returns (ref float64 [M,N], out bf16 bits uint16 [M,N])."""
    a, b, sa, sb = _check_inputs(layout, a, b, sa, sb, M, N, K, gran)
    ref = np.empty((M, N), dtype=np.float64)
    out = np.empty((M, N), dtype=np.uint16)
    rc = _load().oracle_bsgemm_fmt(LAYOUTS[layout], FORMATS[a_fmt], FORMATS[b_fmt], _ptr(a), _ptr(b),
                                   _ptr(sa), _ptr(sb), M, N, K, gran, _ptr(ref), _ptr(out))
    if rc != 0:
        raise RuntimeError(f"oracle_bsgemm failed with code {rc}")
    return ref, out


def bsgemm_at(layout: str, a, b, sa, sb, M: int, N: int, K: int, gran: int, mi, ni,
              a_fmt="e4m3", b_fmt="e4m3"):
    """Oracle outputs at (mi[i], ni[i]) only. Returns (ref float64, out uint16)."""
    a, b, sa, sb = _check_inputs(layout, a, b, sa, sb, M, N, K, gran)
    mi = np.ascontiguousarray(mi, dtype=np.int64)
    ni = np.ascontiguousarray(ni, dtype=np.int64)
    if mi.shape != ni.shape:
        raise ValueError("mi and ni must have the same shape")
    ref = np.empty(mi.shape, dtype=np.float64)
    out = np.empty(mi.shape, dtype=np.uint16)
    rc = _load().oracle_bsgemm_at_fmt(LAYOUTS[layout], FORMATS[a_fmt], FORMATS[b_fmt], _ptr(a), _ptr(b),
                                      _ptr(sa), _ptr(sb), M, N, K, gran, mi.size, _ptr(mi), _ptr(ni),
                                      _ptr(ref), _ptr(out))
    if rc != 0:
        raise RuntimeError(f"oracle_bsgemm_at failed with code {rc}")
    return ref, out


def fp8_encode(fmt: str, v: float) -> int:
    """Nearest code of ``fmt`` to the FP32 value ``v``: ties to an even mantissa, saturating."""
    return int(_load().oracle_fp8_encode(FORMATS[fmt], float(np.float32(v))))


def quantize_blocks(x, gran: int, fmt: str = "e4m3"):
    """Per-block FP8 quantisation of a row-major FP32 [rows, cols] matrix.

    Returns (codes uint8 [rows, cols], scales float32 [ceil(rows/g), ceil(cols/g)]):
    s = amax / FMAX per block (1 for an all-zero block), code = nearest(x / s)
    with both divisions in FP32."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    rows, cols = x.shape
    q = np.empty((rows, cols), dtype=np.uint8)
    s = np.empty((-(-rows // gran), -(-cols // gran)), dtype=np.float32)
    rc = _load().oracle_quantize_blocks(FORMATS[fmt], _ptr(x), rows, cols, gran, _ptr(q), _ptr(s))
    if rc != 0:
        raise RuntimeError(f"oracle_quantize_blocks failed with code {rc}")
    return q, s


ACTIVATIONS = {None: 0, "none": 0, "relu": 1, "gelu": 2}


def epilogue(ref, bias=None, activation=None):
    """act(ref + bias[n]) in FP64 on an FP64 [M,N] product. Returns (value float64, bf16 bits uint16)."""
    ref = np.ascontiguousarray(ref, dtype=np.float64)
    M, N = ref.shape
    b = None if bias is None else np.ascontiguousarray(bias, dtype=np.float32)
    if b is not None and b.size != N:
        raise ValueError("bias must have N elements")
    v = np.empty((M, N), dtype=np.float64)
    out = np.empty((M, N), dtype=np.uint16)
    rc = _load().oracle_epilogue(_ptr(ref), M, N, None if b is None else _ptr(b), ACTIVATIONS[activation],
                                 _ptr(v), _ptr(out))
    if rc != 0:
        raise RuntimeError(f"oracle_epilogue failed with code {rc}")
    return v, out
