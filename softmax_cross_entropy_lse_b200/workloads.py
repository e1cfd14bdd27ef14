"""Seeded synthetic inputs shared by the tests, the smoke check and the bench.

This module draws random numbers and encodes them into storage dtypes. It
holds none of the cross-entropy arithmetic, so both the CUDA path and the
float64 oracle can be fed the identical bytes it produces.

Recipes (numpy PCG64 via ``default_rng``; bf16 values are float32 draws
rounded to nearest-even; fp16 values use numpy's round-to-nearest-even cast):

  c1   4096 x 1024 fp32 ~N(0,1), int32 targets U[0,1024); plus V=2 rows of
       equal logits [v, v] and offset rows [2, -1] + c
  c2   1,048,576 x 128 fp32 ~N(0,1), targets U[0,128), 10% of rows (picked by
       the generator) set to ignore_index=-100, label smoothing 0.1
  c3a  8192 x 32000 bf16 ~N(0, std 2), targets U[0,V)
  c3b  2048 x 151,936 bf16 ~N(0, std 2), targets U[0,V)
  c4a  x (10, 119, 151,936) fp32 ~N(0,1), t (10, 119) int32 U[0,V); the loss
       is taken on the views x[:, :-1] and t[:, 1:]
  c4b  (2^27 + 2^20) x 8 fp32 ~N(0,1), targets U[0,8), drawn in 2^22-row
       chunks with one seed per chunk
  c5   H (8192, 4096) bf16 ~N(0,1), W (151,936, 4096) bf16 ~N(0, std 0.02),
       targets U[0,V)
"""
from __future__ import annotations

import numpy as np

IGNORE_INDEX = -100


# -- storage encodings --------------------------------------------------------
def bf16_bits_from_f32(x: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16 (nearest, ties to even); returns uint16 bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    rounding = ((u >> 16) & 1) + np.uint32(0x7FFF)
    out = ((u + rounding) >> 16).astype(np.uint16)
    nan = np.isnan(x)
    if nan.any():
        out[nan] = np.uint16(0x7FC0)
    return out


def f32_from_bf16_bits(b: np.ndarray) -> np.ndarray:
    """Widen bfloat16 bits to float32 exactly."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def encode(x32: np.ndarray, dtype: str):
    """Return (storage array, exact float32 copy of the stored values)."""
    if dtype == "f32":
        x = np.ascontiguousarray(x32, dtype=np.float32)
        return x, x
    if dtype == "bf16":
        b = bf16_bits_from_f32(x32)
        return b, f32_from_bf16_bits(b)
    if dtype == "f16":
        h = np.asarray(x32, dtype=np.float32).astype(np.float16)
        return h, h.astype(np.float32)
    raise ValueError(dtype)


# -- generic draws -------------------------------------------------------------
def rows(N: int, V: int, dtype: str = "f32", seed: int = 0, std: float = 1.0,
         ignore_frac: float = 0.0, ignore_index: int = IGNORE_INDEX):
    """(N, V) logits ~N(0, std^2) in `dtype`, int32 targets U[0, V)."""
    rng = np.random.default_rng(seed)
    z32 = rng.standard_normal((N, V), dtype=np.float32)
    if std != 1.0:
        z32 *= np.float32(std)
    y = rng.integers(0, V, size=N, dtype=np.int32)
    if ignore_frac > 0:
        k = int(round(ignore_frac * N))
        idx = rng.choice(N, size=k, replace=False)
        y[idx] = ignore_index
    z, zf = encode(z32, dtype)
    return z, zf, y


def special_rows_equal(magnitudes=(1e0, 1e4, 1e6, 1e8), repeat: int = 4):
    """V=2 rows [v, v] with target 0 (each magnitude `repeat` times)."""
    vals = np.repeat(np.asarray(magnitudes, dtype=np.float64), repeat)
    z = np.stack([vals, vals], axis=1)
    y = np.zeros(len(vals), dtype=np.int32)
    return z, y


def special_rows_offset(offsets=(0.0, 1e4, 1e6, 1e8)):
    """V=2 rows [2, -1] + c with target 0."""
    c = np.asarray(offsets, dtype=np.float64)[:, None]
    z = np.array([[2.0, -1.0]]) + c
    y = np.zeros(len(offsets), dtype=np.int32)
    return z, y


# -- named configurations --------------------------------------------------------
def c1(seed: int = 0):
    return rows(4096, 1024, "f32", seed)


def c2(seed: int = 0, N: int = 1 << 20):
    return rows(N, 128, "f32", seed, ignore_frac=0.1)


C2_EPS = 0.1


def c3a(seed: int = 0, N: int = 8192):
    return rows(N, 32000, "bf16", seed, std=2.0)


def c3b(seed: int = 0, N: int = 2048):
    return rows(N, 151936, "bf16", seed, std=2.0)


def c4a(seed: int = 0, B: int = 10, L: int = 119, V: int = 151936):
    """Full (B, L, V) fp32 tensor and (B, L) int32 targets; the loss is taken
    on x[:, :-1] against t[:, 1:]."""
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((B, L, V), dtype=np.float32)
    t = rng.integers(0, V, size=(B, L), dtype=np.int32)
    return x, t


C4B_ROWS = (1 << 27) + (1 << 20)
C4B_CHUNK = 1 << 22


def c4b_chunk(k: int, seed: int = 0, V: int = 8, chunk: int = C4B_CHUNK,
              total: int = C4B_ROWS):
    """Chunk k (rows [k*chunk, min((k+1)*chunk, total))) of the huge-N workload."""
    n = min(chunk, total - k * chunk)
    rng = np.random.default_rng([seed, k])
    z = rng.standard_normal((n, V), dtype=np.float32)
    y = rng.integers(0, V, size=n, dtype=np.int32)
    return z, y


def c5(seed: int = 0, N: int = 8192, V: int = 151936, D: int = 4096,
       w_std: float = 0.02):
    """bf16 bits of H (N, D) and W (V, D), their exact float32 values, targets."""
    rng = np.random.default_rng(seed)
    h32 = rng.standard_normal((N, D), dtype=np.float32)
    w32 = rng.standard_normal((V, D), dtype=np.float32)
    w32 *= np.float32(w_std)
    y = rng.integers(0, V, size=N, dtype=np.int32)
    hb, hf = encode(h32, "bf16")
    wb, wf = encode(w32, "bf16")
    return hb, hf, wb, wf, y
