"""Helpers shared by the GPU parity tests: device upload and the comparison rules."""
from __future__ import annotations

import numpy as np
import torch

# North-star gate on floating-point outputs: normwise relative error
# max_i |y_i - r_i| / max_i |r_i| <= 2e-3 with fp32 outputs (reading of "relative error
# against a float32 reference", paper §3.4).
NORMWISE_TOL = 2e-3
# fp32-accumulated GEMV with exact fp32 operands: the rounding error of a length-n sum is
# far below sqrt(n) * 2^-24 * max|y| for n <= 2^15, so any error above 1e-4 is a bug.
GEMV_F32_TOL = 1e-4


def normwise(got: np.ndarray, ref: np.ndarray) -> float:
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    den = np.abs(ref).max()
    return float(np.abs(got - ref).max() / (den if den > 0 else 1.0))


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


def ulp16(ref: np.ndarray, dtype: torch.dtype) -> np.ndarray:
    """Unit in the last place of each value rounded to the 16-bit type."""
    r = torch.from_numpy(np.asarray(ref, np.float64)).to(dtype).double().abs().numpy()
    mant = 10 if dtype == torch.float16 else 7
    tiny = 2.0 ** -24 if dtype == torch.float16 else 2.0 ** -133
    e = np.floor(np.log2(np.maximum(r, 1e-300)))
    return np.maximum(2.0 ** (e - mant), tiny)


def assert_out(got: torch.Tensor, ref: np.ndarray, f32_tol: float = GEMV_F32_TOL):
    """fp32 outputs: normwise error <= f32_tol (and the 2e-3 gate).  16-bit outputs: each
    element within one ulp of the oracle rounded to that type, plus the fp32 error."""
    g = to_np(got)
    assert g.shape == ref.shape, (g.shape, ref.shape)
    assert np.isfinite(g).all()
    if got.dtype == torch.float32:
        e = normwise(g, ref)
        assert e <= min(f32_tol, NORMWISE_TOL), e
    else:
        slack = f32_tol * np.abs(ref).max()
        bad = np.abs(g - ref) > ulp16(ref, got.dtype) + slack
        assert not bad.any(), (np.argwhere(bad)[:5], g[bad][:5], ref[bad][:5])


def x_tensor(xbits: np.ndarray, dtype_code: int, device="cuda") -> torch.Tensor:
    from workloads import F16, BF16

    if dtype_code == F16:
        return torch.from_numpy(xbits.view(np.int16)).to(device).view(torch.float16)
    if dtype_code == BF16:
        return torch.from_numpy(xbits.view(np.int16)).to(device).view(torch.bfloat16)
    return torch.from_numpy(xbits).to(device)
