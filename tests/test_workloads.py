"""The seeded input generators against the recipes they state: storage
encodings bit for bit against PyTorch's CPU conversions (round to nearest,
ties to even), and each named configuration's shapes, ranges, ignored-row
share, spread and chunking. Both the CUDA path and the oracle are fed these
bytes, so a wrong draw would not show as a parity failure."""
from __future__ import annotations

import numpy as np
import pytest

from softmax_cross_entropy_lse_b200 import workloads as wl

torch = pytest.importorskip("torch")


def special_f32():
    """Ties, near-ties, overflow, subnormals, signed zeros, infinities, NaN."""
    bits = np.array([
        0x3F808000,  # 1.00390625: a tie, even below -> stays
        0x3F818000,  # a tie, odd below -> rounds up
        0x3F808001,  # just above a tie -> up
        0x3F807FFF,  # just below a tie -> down
        0x7F7FFFFF,  # largest float -> rounds to +inf in bf16
        0x7F7F7FFF,  # largest float that stays finite
        0x00000001,  # smallest subnormal
        0x00408000,  # subnormal tie
        0x00000000, 0x80000000,  # +0, -0
        0x7F800000, 0xFF800000,  # +inf, -inf
        0x7FC00000, 0xFFC00001, 0x7F800001,  # NaNs (quiet, negative, signalling)
        0xBF818000, 0xC2F68000,  # negative ties
    ], dtype=np.uint32)
    return bits.view(np.float32)


def test_bf16_encoding_matches_torch():
    rng = np.random.default_rng(0)
    x = np.concatenate([
        special_f32(),
        rng.standard_normal(20000).astype(np.float32) * np.float32(3.0),
        (rng.standard_normal(20000) * 10.0 ** rng.uniform(-40, 38, 20000)).astype(np.float32),
        rng.integers(0, 2 ** 32, 20000, dtype=np.uint64).astype(np.uint32).view(np.float32),
    ])
    ours = wl.bf16_bits_from_f32(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    nan = np.isnan(x)
    assert np.array_equal(ours[~nan], ref[~nan])
    # every NaN becomes one quiet NaN (torch's own NaN bits vary by code path)
    assert np.all(ours[nan] == 0x7FC0)
    assert np.all((ref[nan] & 0x7F80) == 0x7F80) and np.all((ref[nan] & 0x7F) != 0)
    # widening is exact and agrees with torch's
    wide = wl.f32_from_bf16_bits(ours)
    ref_wide = torch.from_numpy(ours.view(np.int16)).view(torch.bfloat16).float().numpy()
    assert np.array_equal(wide.view(np.uint32)[~nan], ref_wide.view(np.uint32)[~nan])
    assert np.all(np.isnan(wide[nan]))


def test_f16_encoding_matches_torch():
    rng = np.random.default_rng(1)
    x = np.concatenate([special_f32(), rng.standard_normal(20000).astype(np.float32) * 300,
                        (rng.standard_normal(5000) * 1e-5).astype(np.float32)])
    with np.errstate(over="ignore"):  # the largest floats overflow to inf, as intended
        h, h32 = wl.encode(x, "f16")
    ref = torch.from_numpy(x).to(torch.float16).numpy()
    nan = np.isnan(x)
    assert np.array_equal(h.view(np.uint16)[~nan], ref.view(np.uint16)[~nan])
    assert np.array_equal(h32[~nan], h[~nan].astype(np.float32))


def test_rows_recipe():
    z, z32, y = wl.rows(4000, 300, "f32", seed=5, std=2.0, ignore_frac=0.1)
    assert z.shape == (4000, 300) and z.dtype == np.float32 and y.dtype == np.int32
    assert abs(float(z.std()) - 2.0) < 0.02 and abs(float(z.mean())) < 0.01
    ign = y == wl.IGNORE_INDEX
    assert ign.sum() == 400
    assert y[~ign].min() >= 0 and y[~ign].max() < 300
    # the same seed gives the same bytes; another seed does not
    z2, _, y2 = wl.rows(4000, 300, "f32", seed=5, std=2.0, ignore_frac=0.1)
    assert np.array_equal(z, z2) and np.array_equal(y, y2)
    z3, _, _ = wl.rows(4000, 300, "f32", seed=6, std=2.0, ignore_frac=0.1)
    assert not np.array_equal(z, z3)
    # bf16 storage holds the rounded draw; the float32 copy is its exact value
    b, b32, _ = wl.rows(50, 300, "bf16", seed=5, std=2.0)
    assert b.dtype == np.uint16 and np.array_equal(b32, wl.f32_from_bf16_bits(b))


def test_named_configurations():
    z, z32, y = wl.c2(N=1 << 14)
    assert z.shape == (1 << 14, 128) and (y == -100).sum() == round(0.1 * (1 << 14))
    assert wl.C2_EPS == 0.1
    b, b32, y = wl.c3a(N=16)
    assert b.shape == (16, 32000) and b.dtype == np.uint16 and y.max() < 32000
    assert abs(float(b32.std()) - 2.0) < 0.02
    b, b32, y = wl.c3b(N=4)
    assert b.shape == (4, 151936) and abs(float(b32.std()) - 2.0) < 0.02
    x, t = wl.c4a(B=3, L=7, V=40)
    assert x.shape == (3, 7, 40) and t.shape == (3, 7) and t.max() < 40
    hb, hf, wb, wf, y = wl.c5(N=64, V=3000, D=128)
    assert hb.shape == (64, 128) and wb.shape == (3000, 128) and y.max() < 3000
    assert abs(float(hf.std()) - 1.0) < 0.03 and abs(float(wf.std()) - 0.02) < 0.0005
    assert np.array_equal(wf, wl.f32_from_bf16_bits(wb))


def test_c4b_chunking():
    # the full size: 33 chunks of 2^22 rows, the last one 2^20
    assert wl.C4B_ROWS == 2 ** 27 + 2 ** 20 and wl.C4B_CHUNK == 2 ** 22
    nchunks = -(-wl.C4B_ROWS // wl.C4B_CHUNK)
    assert nchunks == 33
    z, y = wl.c4b_chunk(nchunks - 1)
    assert z.shape == (2 ** 20, 8) and y.shape == (2 ** 20,) and 0 <= y.min() and y.max() < 8
    # chunks are independent of one another and cover the rows exactly once
    sizes = [len(wl.c4b_chunk(k, chunk=1000, total=3500)[1]) for k in range(4)]
    assert sizes == [1000, 1000, 1000, 500]
    a = wl.c4b_chunk(2, chunk=1000, total=3500)
    b = wl.c4b_chunk(2, chunk=1000, total=3500)
    c = wl.c4b_chunk(1, chunk=1000, total=3500)
    assert np.array_equal(a[0], b[0]) and not np.array_equal(a[0], c[0])
