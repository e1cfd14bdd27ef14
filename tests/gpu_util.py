"""Helpers shared by the GPU parity tests: upload seeded numpy inputs, read
results back, and compare against the float64 oracle with the tolerances the
method's statement fixes.

Tolerances (per element, NaN and +-inf positions must match exactly):
  fp32 inputs   loss, lse  |d| <= 1e-5 |ref| + 1e-6 (the absolute floor keeps
                           losses near 0, where float rounding of lse - z_y is
                           ~1e-7 absolute, from failing a purely relative test)
                gradient   |d| <= 1e-6
  bf16/fp16     loss, lse  |d| <= 2e-3 |ref| + 1e-6
                gradient   |d| <= 1e-4 with float output; with a 16-bit output,
                           against the oracle rounded to that format:
                           |d| <= max(1e-4, one unit in the last place of ref)
The gradient bounds are stated for the VJP of a unit upstream gradient,
dz = softmax - onehot, whose entries lie in [-1, 1]. With an upstream
gradient g_i the exact row is g_i times that, and so is its rounding error:
the absolute bound of row i is scaled by max(1, |g_i|) (every parity test
takes this reading; g may be a scalar or one value per row).
"""
from __future__ import annotations

import numpy as np
import pytest

torch = pytest.importorskip("torch")

from softmax_cross_entropy_lse_b200 import workloads as wl  # noqa: E402


def dev():
    return torch.device("cuda", 0)


def upload(arr: np.ndarray, dtype: str = "f32"):
    """numpy storage array (float32, bf16 bits as uint16, float16, ints) -> cuda tensor."""
    if dtype == "bf16":
        t = torch.from_numpy(np.ascontiguousarray(arr).view(np.int16)).to(dev())
        return t.view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(arr)).to(dev())


def f32(t) -> np.ndarray:
    return t.detach().float().cpu().numpy()


def bf16_round(x64: np.ndarray) -> np.ndarray:
    """float64 -> nearest bf16 value (as float64), ties to even, via float32."""
    return wl.f32_from_bf16_bits(wl.bf16_bits_from_f32(x64.astype(np.float32))).astype(np.float64)


def f16_round(x64: np.ndarray) -> np.ndarray:
    return x64.astype(np.float32).astype(np.float16).astype(np.float64)


def _special_match(got, ref, what):
    gn, rn = np.isnan(got), np.isnan(ref)
    assert (gn == rn).all(), f"{what}: NaN positions differ ({(gn != rn).sum()} entries)"
    gi, ri = np.isinf(got), np.isinf(ref)
    assert (gi == ri).all(), f"{what}: inf positions differ"
    assert (got[gi] == ref[ri]).all(), f"{what}: inf signs differ"
    return ~(rn | ri)


def assert_close(got, ref, rtol, atol, what="value"):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    ok = _special_match(got, ref, what)
    d = np.abs(got[ok] - ref[ok])
    bound = rtol * np.abs(ref[ok]) + atol
    bad = d > bound
    if bad.any():
        i = np.argmax(d - bound)
        raise AssertionError(f"{what}: {bad.sum()} of {d.size} outside tolerance; worst "
                             f"got {got[ok][i]!r} ref {ref[ok][i]!r} |d|={d[i]:.3e} "
                             f"bound={bound[i]:.3e}")


def loss_tol(dtype: str):
    return (1e-5, 1e-6) if dtype == "f32" else (2e-3, 1e-6)


def grad_scale(g, shape) -> np.ndarray:
    """max(1, |g_i|) broadcast over the rows of a gradient of `shape`."""
    gs = np.maximum(1.0, np.abs(np.asarray(1.0 if g is None else g, np.float64)))
    if gs.ndim == 1:
        gs = gs.reshape((-1,) + (1,) * (len(shape) - 1))
    return np.broadcast_to(gs, shape)


def assert_grad_close(got, ref64, in_dtype: str, out_dtype: str, what="dlogits", g=None):
    got = np.asarray(got, np.float64)
    scale = grad_scale(g, got.shape)
    if out_dtype == "f32":
        atol = 1e-6 if in_dtype == "f32" else 1e-4
        ref64 = np.asarray(ref64, np.float64)
        ok = _special_match(got, ref64, what)
        d = np.abs(got[ok] - ref64[ok])
        bound = atol * scale[ok]
        bad = d > bound
        if bad.any():
            i = np.argmax(d - bound)
            raise AssertionError(f"{what}: {bad.sum()} of {d.size} outside tolerance; worst "
                                 f"got {got[ok][i]!r} ref {ref64[ok][i]!r} |d|={d[i]:.3e} "
                                 f"bound={bound[i]:.3e}")
        return
    rounded = bf16_round(ref64) if out_dtype == "bf16" else f16_round(ref64)
    got = np.asarray(got, np.float64)
    ok = _special_match(got, rounded, what)
    mant = 7 if out_dtype == "bf16" else 10
    with np.errstate(divide="ignore"):
        ulp = np.where(rounded[ok] == 0, 0.0,
                       2.0 ** (np.floor(np.log2(np.abs(rounded[ok]))) - mant))
    bound = np.maximum(1e-4 * scale[ok], ulp)
    d = np.abs(got[ok] - rounded[ok])
    bad = d > bound
    if bad.any():
        i = np.argmax(d - bound)
        raise AssertionError(f"{what}: {bad.sum()} entries off; worst got {got[ok][i]} "
                             f"ref {rounded[ok][i]} |d|={d[i]:.3e}")
