"""Helpers shared by the GPU parity tests (not a test module).

Tolerance (per element, the parity bar for this GEMM):
    |gpu - ref| <= 2^-7 * |ref| + 2^-8 * rms(ref)
where ref is the oracle's FP64 value before BF16 rounding and rms is taken
over the whole output matrix.  2^-7 is one BF16 rounding (2^-8) plus the same
again for FP32 accumulation of per-block partials; the rms term absorbs
cancellation in elements whose exact value is near zero.

Where the whole output is checked, rms comes from ref itself.  Where only a
sample of outputs is checked (full-size problems), the oracle has only the
sampled ref values, so rms over the whole matrix comes from the GPU output
instead, lowered by 2^-6.  When every element meets the bound,
rms(gpu - ref) <= 2^-7 rms(ref) + 2^-8 rms(ref), so
rms(gpu) <= rms(ref) (1 + 3 * 2^-8) < rms(ref) / (1 - 2^-6), and the bound
built on rms(gpu) (1 - 2^-6) is tighter than the exact one.  (An output far
off in unsampled elements could raise rms(gpu); those elements are not
checked by a sampled test in any case.)
"""
import numpy as np
import torch

import oracle
import workloads
import fp8_block_scaled_bsgemm_b200 as bsg


def to_device(p: workloads.Problem, device="cuda"):
    a = torch.from_numpy(p.a).to(device)
    b = torch.from_numpy(p.b).to(device)
    sa = torch.from_numpy(p.sa).to(device)
    sb = torch.from_numpy(p.sb).to(device)
    return a, b, sa, sb


def run_gpu(p: workloads.Problem, tuning=None, out=None):
    a, b, sa, sb = to_device(p)
    out = bsg.gemm(a, b, sa, sb, out=out, layout=p.layout, gran=p.gran, tuning=tuning,
                   a_format=p.a_fmt, b_format=p.b_fmt)
    torch.cuda.synchronize()
    return out


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def gpu_as_f64(out: torch.Tensor) -> np.ndarray:
    return out.float().cpu().numpy().astype(np.float64)


def tolerance(ref: np.ndarray, rms=None) -> np.ndarray:
    """Per-element bound; `rms` over the whole output matrix, or None for the
    rms of `ref` (when `ref` is the whole output)."""
    if rms is None:
        rms = float(np.sqrt(np.mean(ref * ref))) if ref.size else 0.0
    return 2.0 ** -7 * np.abs(ref) + 2.0 ** -8 * rms


def full_rms_from_gpu(out: torch.Tensor) -> float:
    """rms over the whole GPU output, lowered by 2^-6 so the bound built on it
    is never looser than the one built on the whole ref (see above)."""
    rms = float(out.double().square().mean().sqrt())
    return rms * (1.0 - 2.0 ** -6)


# One record per passing check: (what, max err/tol, fraction of elements above
# half the tolerance, elements compared). The session summary prints the worst.
PARITY_LOG = []


def check_close(got: np.ndarray, ref: np.ndarray, what="", rms=None):
    tol = tolerance(ref, rms)
    err = np.abs(got - ref)
    bad = ~(err <= tol)          # also catches NaN
    if bad.any():
        idx = np.argwhere(bad)[:8]
        raise AssertionError(f"{what}: {int(bad.sum())} of {ref.size} elements out of tolerance; "
                             f"max err/tol {float(np.nanmax(err / np.maximum(tol, 1e-300))):.3g}; "
                             f"first {idx.tolist()} got {got[bad][:8]} want {ref[bad][:8]}")
    if not ref.size:
        return 0.0
    ratio = float(np.max(err / np.maximum(tol, 1e-300)))
    PARITY_LOG.append((what, ratio, float(np.mean(err > 0.5 * tol)), int(ref.size)))
    return ratio


def full_parity(p: workloads.Problem, tuning=None, what=""):
    out = run_gpu(p, tuning)
    ref, _ = oracle.bsgemm(p.layout, p.a, p.b, p.sa, p.sb, p.M, p.N, p.K, p.gran, p.a_fmt, p.b_fmt)
    return check_close(gpu_as_f64(out), ref, what or p.name), out


def sampled_parity(p: workloads.Problem, count=3000, tuning=None, seed=0, what=""):
    out = run_gpu(p, tuning)
    mi, ni = workloads.sample_indices(p.M, p.N, count, seed=seed)
    ref, _ = oracle.bsgemm_at(p.layout, p.a, p.b, p.sa, p.sb, p.M, p.N, p.K, p.gran, mi, ni,
                              p.a_fmt, p.b_fmt)
    got = gpu_as_f64(out[torch.from_numpy(mi).cuda(), torch.from_numpy(ni).cuda()])
    return check_close(got, ref, what or p.name, rms=full_rms_from_gpu(out)), out
