"""Shared helpers for the GPU parity tests (host<->device marshalling and the
row-wise tolerance check).  No method arithmetic lives here."""
import numpy as np
import torch

# Acceptance for floating-point outputs: for every row i,
#   max_j |gpu[i, j] - ref[i, j]| <= TOL * max_j |ref[i, j]|
# i.e. the max element error relative to the row's largest oracle magnitude.
# (This L-infinity reading of "relative to the fp64 oracle row norm" is the
# stricter one: max_j |ref[i, j]| <= ||ref[i, :]||_2.)
TOL = 2e-2


def bf16_dev(bits: np.ndarray) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
    return t.view(torch.bfloat16).cuda()


def f32_dev(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()


def bf16_host_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def bf16_host_f64(t: torch.Tensor) -> np.ndarray:
    bits = bf16_host_bits(t).astype(np.uint32) << 16
    return bits.view(np.float32).astype(np.float64)


def f32_host_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def rows_within(gpu: np.ndarray, ref: np.ndarray, tol: float = TOL, what: str = "") -> float:
    """Assert the row-wise bound; return the worst ratio err / (tol * rowmax)."""
    gpu = np.asarray(gpu, np.float64).reshape(ref.shape[0], -1)
    ref = np.asarray(ref, np.float64).reshape(ref.shape[0], -1)
    assert np.all(np.isfinite(gpu)), f"{what}: non-finite GPU output"
    err = np.abs(gpu - ref).max(axis=1)
    scale = np.abs(ref).max(axis=1)
    zero = scale == 0
    assert np.all(err[zero] == 0), f"{what}: rows that are exactly zero in the oracle must be zero"
    ratio = np.zeros_like(err)
    ratio[~zero] = err[~zero] / (tol * scale[~zero])
    worst = float(ratio.max()) if ratio.size else 0.0
    assert worst <= 1.0, f"{what}: row error {worst:.3f} x tolerance (row {int(ratio.argmax())})"
    return worst


def within_one_bf16_ulp(gpu_bits: np.ndarray, ref_bits: np.ndarray, what: str = "", ulps: int = 1,
                        abs_extra=0.0, mag_extra=None):
    """|gpu - ref| <= ulps * (bf16 spacing at the larger of the two magnitudes) + abs_extra.

    abs_extra carries the fp32 error of the GPU's rank-r product before the one
    rounding to bf16 (it matters only where W' + s B A cancels to a value far
    smaller than its terms)."""
    g = (gpu_bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    r = (ref_bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    mag = np.maximum(np.abs(r), np.abs(g))
    if mag_extra is not None:
        mag = np.maximum(mag, np.abs(mag_extra))
    mag = mag.astype(np.float32)
    ulp = np.spacing(mag).astype(np.float64) * 65536.0
    ulp = np.maximum(ulp, 2.0 ** -133) * ulps + abs_extra
    bad = np.abs(g - r) > ulp
    assert not bad.any(), f"{what}: {int(bad.sum())} elements beyond 1 bf16 ulp"
