"""Python binding of the B200 block-scaled FP8 GEMM C ABI (``include/bsgemm.h``).

Argument marshalling only: every step of the GEMM runs in ``libbsgemm.so``'s
CUDA kernels.  PyTorch supplies device memory and streams.  There is no CPU
path: if the library is missing (and cannot be built here) every call raises.

    out = bsgemm_fp8_nt(a, b, scale_a, scale_b)          # a [M,K], b [N,K]
    out = gemm(a, b, scale_a, scale_b, layout="tn")      # a [K,M], b [K,N]

Operation (hncyxsy.com/news/191052 §2.2, §3.2, §4.2):
out[m,n] = bf16(sum_kb sA[m/g][kb] * sB[n/g][kb] * sum_{k in kb} A[m,k] B[n,k]).
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libbsgemm.so")

LAYOUTS = {"nt": 0, "tn": 1, "nn": 2, "tt": 3}
FORMATS = {"e4m3": 0, "e5m2": 1}
VARIANTS = {"auto": 0, "data_parallel": 1, "swap_ab": 2, "cta_pair": 3}
STATUS = {0: "ok", 1: "invalid argument", 2: "unsupported granularity", 3: "misaligned",
          4: "unsupported device", 5: "CUDA error", 6: "device wait timeout",
          7: "needs more scratch than the allocation-free entry point holds"}

_lock = threading.Lock()
_lib = None


class BsgemmError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        super().__init__(f"{what}: {STATUS.get(status, 'unknown')} (status {status})")


class Tuning(ctypes.Structure):
    _fields_ = [("variant", ctypes.c_int), ("bnq", ctypes.c_int), ("splits", ctypes.c_int),
                ("stream_k", ctypes.c_int)]


class Epilogue(ctypes.Structure):
    _fields_ = [("bias", ctypes.c_void_p), ("activation", ctypes.c_int), ("out_dtype", ctypes.c_int)]


ACTIVATIONS = {None: 0, "none": 0, "relu": 1, "gelu": 2}


class Plan(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in ("layout", "gran", "swap_ab", "bnq", "tiles_p", "tiles_q",
                                            "splits", "kb_per_split", "grid", "group_p", "kernels",
                                            "sk_first_tile", "sk_units_per_tile", "sk_ctas", "sk_units",
                                            "cta_pair", "grouped")]

    def as_dict(self):
        return {n: getattr(self, n) for n, _ in self._fields_}


EXPORTS = ("bsgemm_fp8_nt", "bsgemm_fp8_tn", "bsgemm_fp8_nn", "bsgemm_fp8_tt", "bsgemm_fp8_gemm_ex",
           "bsgemm_fp8_gemm_fmt", "bsgemm_fp8_gemm_fused", "bsgemm_fp8_grouped_nt",
           "bsgemm_make_plan", "bsgemm_status_string", "bsgemm_get_last_device_status",
           "bsgemm_last_device_status_detail", "bsgemm_diag_wait_timeout", "bsgemm_version",
           "bsgemm_fp8_nt_noalloc", "bsgemm_quantize_fp8", "bsgemm_release_workspaces")


def lib():
    """Load ``libbsgemm.so`` (building it first if it is missing and nvcc exists)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                from . import build as _build
                _build.build()
            L = ctypes.CDLL(LIB_PATH)
            p, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
            gemm_args = [p, p, p, p, p, i64, i64, i64, i32, p]
            for name in ("bsgemm_fp8_nt", "bsgemm_fp8_tn", "bsgemm_fp8_nn", "bsgemm_fp8_tt",
                         "bsgemm_fp8_nt_noalloc", "bsgemm_quantize_fp8", "bsgemm_release_workspaces"):
                getattr(L, name).argtypes = gemm_args
                getattr(L, name).restype = i32
            L.bsgemm_fp8_gemm_ex.argtypes = [i32, p, p, p, p, p, i64, i64, i64, i32,
                                             ctypes.POINTER(Tuning), p]
            L.bsgemm_fp8_gemm_ex.restype = i32
            L.bsgemm_fp8_gemm_fmt.argtypes = [i32, i32, i32, p, p, p, p, p, i64, i64, i64, i32,
                                              ctypes.POINTER(Tuning), p]
            L.bsgemm_fp8_gemm_fmt.restype = i32
            L.bsgemm_fp8_gemm_fused.argtypes = [i32, i32, i32, p, p, p, p, ctypes.POINTER(Epilogue), p,
                                                i64, i64, i64, i32, ctypes.POINTER(Tuning), p]
            L.bsgemm_fp8_gemm_fused.restype = i32
            L.bsgemm_fp8_grouped_nt.argtypes = [i32, i32, p, p, p, p, p, p, i32, i64, i64, i64, i32, p]
            L.bsgemm_fp8_grouped_nt.restype = i32
            L.bsgemm_make_plan.argtypes = [i32, i64, i64, i64, i32, i32, ctypes.POINTER(Tuning),
                                           ctypes.POINTER(Plan)]
            L.bsgemm_make_plan.restype = i32
            L.bsgemm_status_string.argtypes = [i32]
            L.bsgemm_status_string.restype = ctypes.c_char_p
            L.bsgemm_get_last_device_status.argtypes = [p]
            L.bsgemm_get_last_device_status.restype = i32
            L.bsgemm_last_device_status_detail.argtypes = []
            L.bsgemm_last_device_status_detail.restype = i32
            L.bsgemm_diag_wait_timeout.argtypes = [ctypes.c_ulonglong, p]
            L.bsgemm_diag_wait_timeout.restype = i32
            L.bsgemm_quantize_fp8.argtypes = [i32, i32, p, i64, i64, i32, p, p, p]
            L.bsgemm_quantize_fp8.restype = i32
            L.bsgemm_release_workspaces.argtypes = []
            L.bsgemm_release_workspaces.restype = i32
            L.bsgemm_version.argtypes = []
            L.bsgemm_version.restype = i32
            _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().bsgemm_status_string(int(status)).decode()


def _stream_handle(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream) if hasattr(stream, "cuda_stream") else int(stream)


def _tuning(tuning):
    if tuning is None:
        return None
    if isinstance(tuning, Tuning):
        return ctypes.byref(tuning)
    t = Tuning(VARIANTS[tuning.get("variant", "auto")], int(tuning.get("bnq", 0)),
               int(tuning.get("splits", 0)), int(tuning.get("stream_k", 0)))
    return ctypes.byref(t)


def _as_bytes(x: torch.Tensor, name: str, device=None) -> torch.Tensor:
    if x.dtype not in (torch.float8_e4m3fn, torch.float8_e5m2, torch.uint8):
        raise TypeError(f"{name} must be float8_e4m3fn, float8_e5m2 or uint8 codes, got {x.dtype}")
    if not x.is_cuda or not x.is_contiguous():
        raise ValueError(f"{name} must be a contiguous CUDA tensor")
    if device is not None and x.device != device:
        raise ValueError(f"{name} is on {x.device}, the first operand on {device}")
    return x


def _device_tensor(t, name: str, dtype, device, numel=None, min_numel=None):
    """Check a tensor whose data pointer goes to the library: the kernels get
    only the pointer, so its type, placement and size are checked here."""
    if not isinstance(t, torch.Tensor) or t.dtype != dtype or not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous {dtype} CUDA tensor")
    if t.device != device:
        raise ValueError(f"{name} is on {t.device}, the first operand on {device}")
    if numel is not None and t.numel() != numel:
        raise ValueError(f"{name} must have {numel} elements, got {t.numel()}")
    if min_numel is not None and t.numel() < min_numel:
        raise ValueError(f"{name} must have at least {min_numel} elements, got {t.numel()}")
    return t


def _blocks(n: int, gran) -> int:
    return -(-int(n) // int(gran))


_GRANS = (64, 128, 256)   # other values go to the library, which rejects them


def shapes(layout: str, a: torch.Tensor, b: torch.Tensor):
    """(M, N, K) from the stored shapes of a and b for a layout."""
    if a.dim() != 2 or b.dim() != 2:
        raise ValueError("a and b must be 2-D")
    M, Ka = (a.shape[1], a.shape[0]) if layout[0] == "t" else (a.shape[0], a.shape[1])
    N, Kb = (b.shape[0], b.shape[1]) if layout[1] == "t" else (b.shape[1], b.shape[0])
    if Ka != Kb:
        raise ValueError(f"K mismatch: {Ka} vs {Kb}")
    return int(M), int(N), int(Ka)


def _format(x: torch.Tensor, given, name: str) -> int:
    """FP8 format of an operand: from its dtype, or ``given`` for uint8 codes."""
    from_dtype = {torch.float8_e4m3fn: "e4m3", torch.float8_e5m2: "e5m2"}.get(x.dtype)
    fmt = given if given is not None else (from_dtype or "e4m3")
    if fmt not in FORMATS:
        raise ValueError(f"{name}: format must be one of {sorted(FORMATS)}")
    if from_dtype is not None and fmt != from_dtype:
        raise ValueError(f"{name}: dtype {x.dtype} does not match format {fmt}")
    return FORMATS[fmt]


def gemm(a, b, scale_a, scale_b, out=None, layout="nt", gran=128, tuning=None, stream=None,
         a_format=None, b_format=None, bias=None, activation=None, out_dtype=torch.bfloat16):
    """out[M,N] of the block-scaled FP8 GEMM; see ``include/bsgemm.h``.

    ``a_format`` / ``b_format``: "e4m3" or "e5m2"; taken from the tensor's
    dtype when it is a float8 type, E4M3 for uint8 codes unless given.
    Fused epilogue: out = activation(acc + bias[n]) with ``bias`` an FP32 [N]
    CUDA tensor or None, ``activation`` None / "relu" / "gelu" (erf form), and
    ``out_dtype`` torch.bfloat16 or torch.float32."""
    if layout not in LAYOUTS:
        raise ValueError(f"layout must be one of {sorted(LAYOUTS)}")
    fa = _format(a, a_format, "a")
    fb = _format(b, b_format, "b")
    a = _as_bytes(a, "a")
    dev = a.device
    b = _as_bytes(b, "b", dev)
    M, N, K = shapes(layout, a, b)
    ok_g = gran in _GRANS
    _device_tensor(scale_a, "scale_a", torch.float32, dev,
                   _blocks(M, gran) * _blocks(K, gran) if ok_g else None)
    _device_tensor(scale_b, "scale_b", torch.float32, dev,
                   _blocks(N, gran) * _blocks(K, gran) if ok_g else None)
    if out_dtype not in (torch.bfloat16, torch.float32):
        raise ValueError("out_dtype must be torch.bfloat16 or torch.float32")
    if activation not in ACTIVATIONS:
        raise ValueError(f"activation must be one of {sorted(k for k in ACTIVATIONS if k)}")
    if bias is not None:
        _device_tensor(bias, "bias", torch.float32, dev, N)
    if out is None:
        out = torch.empty((M, N), dtype=out_dtype, device=dev)
    _device_tensor(out, "out", out_dtype, dev)
    if tuple(out.shape) != (M, N):
        raise ValueError(f"out must be a {out_dtype} [M, N] = [{M}, {N}] tensor, got {tuple(out.shape)}")
    epi = None
    if bias is not None or ACTIVATIONS[activation] or out_dtype == torch.float32:
        epi = ctypes.byref(Epilogue(bias.data_ptr() if bias is not None else None, ACTIVATIONS[activation],
                                    1 if out_dtype == torch.float32 else 0))
    with torch.cuda.device(dev):
        st = lib().bsgemm_fp8_gemm_fused(LAYOUTS[layout], fa, fb, a.data_ptr(), b.data_ptr(),
                                         scale_a.data_ptr(), scale_b.data_ptr(), epi, out.data_ptr(), M,
                                         N, K, int(gran), _tuning(tuning), _stream_handle(stream))
    if st != 0:
        raise BsgemmError(st, f"bsgemm {layout} M={M} N={N} K={K} g={gran}")
    return out


def bsgemm_fp8_nt(a, b, scale_a, scale_b, out=None, gran=128, stream=None):
    return gemm(a, b, scale_a, scale_b, out, "nt", gran, None, stream)


def bsgemm_fp8_tn(a, b, scale_a, scale_b, out=None, gran=128, stream=None):
    return gemm(a, b, scale_a, scale_b, out, "tn", gran, None, stream)


def bsgemm_fp8_nn(a, b, scale_a, scale_b, out=None, gran=128, stream=None):
    return gemm(a, b, scale_a, scale_b, out, "nn", gran, None, stream)


def bsgemm_fp8_tt(a, b, scale_a, scale_b, out=None, gran=128, stream=None):
    return gemm(a, b, scale_a, scale_b, out, "tt", gran, None, stream)


def quantize(x: torch.Tensor, gran: int = 128, fmt: str = "e4m3", q=None, scales=None, stream=None):
    """Per-block FP8 quantisation of a row-major FP32/BF16 CUDA matrix [rows, cols].

    Returns (q uint8 [rows, cols], scales float32 [ceil(rows/g), ceil(cols/g)]):
    the GEMM's operand and scale tensors. See ``bsgemm_quantize_fp8``."""
    if x.dim() != 2 or not x.is_cuda or not x.is_contiguous():
        raise ValueError("x must be a contiguous 2-D CUDA tensor")
    src = {torch.float32: 0, torch.bfloat16: 1}.get(x.dtype)
    if src is None:
        raise TypeError(f"x must be float32 or bfloat16, got {x.dtype}")
    if fmt not in FORMATS:
        raise ValueError(f"fmt must be one of {sorted(FORMATS)}")
    rows, cols = x.shape
    dev = x.device
    if q is None:
        q = torch.empty((rows, cols), dtype=torch.uint8, device=dev)
    _device_tensor(q, "q", torch.uint8, dev, rows * cols)
    ok_g = gran in _GRANS
    if scales is None:
        scales = torch.empty((_blocks(rows, gran), _blocks(cols, gran)) if ok_g else (1,),
                             dtype=torch.float32, device=dev)
    _device_tensor(scales, "scales", torch.float32, dev,
                   _blocks(rows, gran) * _blocks(cols, gran) if ok_g else None)
    with torch.cuda.device(dev):
        st = lib().bsgemm_quantize_fp8(src, FORMATS[fmt], x.data_ptr(), rows, cols, int(gran), q.data_ptr(),
                                       scales.data_ptr(), _stream_handle(stream))
    if st != 0:
        raise BsgemmError(st, f"bsgemm_quantize_fp8 {rows}x{cols} g={gran}")
    return q, scales


def grouped_gemm(a, b, scale_a, scale_b, group_m, out=None, gran=128, a_format=None, b_format=None,
                 stream=None):
    """Grouped NT GEMM: group i multiplies rows R_i .. R_i + M_i - 1 of ``a`` [max_rows, K]
    by ``b[i]`` ([num_groups, N, K]); ``group_m`` is an int32 CUDA tensor of the M_i.
    See ``bsgemm_fp8_grouped_nt`` for the scale layouts."""
    fa = _format(a, a_format, "a")
    fb = _format(b, b_format, "b")
    a = _as_bytes(a, "a")
    dev = a.device
    b = _as_bytes(b, "b", dev)
    if a.dim() != 2 or b.dim() != 3 or a.shape[1] != b.shape[2]:
        raise ValueError("a must be [max_rows, K] and b [num_groups, N, K]")
    max_rows, K = a.shape
    G, N = b.shape[0], b.shape[1]
    _device_tensor(group_m, "group_m (one int32 entry per group)", torch.int32, dev, G)
    if gran in _GRANS:
        kb = _blocks(K, gran)
        _device_tensor(scale_a, "scale_a", torch.float32, dev,
                       min_numel=(_blocks(max_rows, gran) + G) * kb)
        _device_tensor(scale_b, "scale_b", torch.float32, dev, G * _blocks(N, gran) * kb)
    else:
        _device_tensor(scale_a, "scale_a", torch.float32, dev)
        _device_tensor(scale_b, "scale_b", torch.float32, dev)
    if out is None:
        out = torch.empty((max_rows, N), dtype=torch.bfloat16, device=dev)
    _device_tensor(out, "out", torch.bfloat16, dev)
    if tuple(out.shape) != (max_rows, N):
        raise ValueError(f"out must be a bfloat16 [max_rows, N] = [{max_rows}, {N}] tensor")
    with torch.cuda.device(dev):
        st = lib().bsgemm_fp8_grouped_nt(fa, fb, a.data_ptr(), b.data_ptr(), scale_a.data_ptr(),
                                         scale_b.data_ptr(), out.data_ptr(), group_m.data_ptr(), G,
                                         max_rows, N, K, int(gran), _stream_handle(stream))
    if st != 0:
        raise BsgemmError(st, f"bsgemm grouped G={G} max_rows={max_rows} N={N} K={K} g={gran}")
    return out


def scratch_bytes(plan: dict) -> int:
    """Split-K / stream-K workspace bytes (FP32 partial tiles) a plan uses."""
    tile = plan["bnq"] * 128 * 4
    if plan["sk_ctas"] > 0:
        return 2 * plan["sk_ctas"] * tile
    if plan["splits"] > 1:
        return plan["tiles_p"] * plan["tiles_q"] * plan["splits"] * tile
    return 0


def make_plan(M, N, K, gran=128, layout="nt", num_sms=148, tuning=None) -> dict:
    pl = Plan()
    st = lib().bsgemm_make_plan(LAYOUTS[layout], M, N, K, gran, num_sms, _tuning(tuning), ctypes.byref(pl))
    if st != 0:
        raise BsgemmError(st, "bsgemm_make_plan")
    return pl.as_dict()


def get_last_device_status(stream=None) -> int:
    return int(lib().bsgemm_get_last_device_status(_stream_handle(stream)))


def release_workspaces() -> int:
    """Free the library's split-K workspaces on the current device (waits for the device)."""
    return int(lib().bsgemm_release_workspaces())


def diag_wait_timeout(timeout_ns: int, stream=None) -> int:
    return int(lib().bsgemm_diag_wait_timeout(int(timeout_ns), _stream_handle(stream)))
