"""ce_forward_backward (forward and VJP in one call) on the GPU, through the
C ABI, against the float64 oracle and against ce_forward + ce_backward."""
from __future__ import annotations

import numpy as np
import pytest

from tests.gpu_util import assert_close, assert_grad_close, f32, loss_tol, torch, upload

import softmax_cross_entropy_lse_b200 as ce
from softmax_cross_entropy_lse_b200 import workloads as wl

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    ce.lib()
    yield
    assert ce.get_error() == 0


def close_ulps(a, b, g=1.0):
    """dz of the fused call vs the two-call path: the exponent argument may be
    evaluated by different instruction schedules, so entries may differ by a
    few float ulps of g * p; bound the difference by 1e-6 |g| (the float
    gradient tolerance), NaNs in the same places."""
    gmax = float(torch.as_tensor(g).abs().max()) if not isinstance(g, float) else abs(g)
    if not torch.equal(torch.isnan(a), torch.isnan(b)):
        return False
    d = (a.double() - b.double()).nan_to_num(0.0).abs().max().item()
    return d <= 1e-6 * max(gmax, 1e-30)


def separate(zt, yt, g, eps, ignore=-100, out_dtype=None):
    r = ce.ce_forward(zt, yt, eps, ignore, return_argmax=True)
    dz = ce.ce_backward(g, zt, yt, r.lse, r.lse_lo, eps, ignore, out_dtype=out_dtype)
    return r, dz


def check_oracle(orc, r, dz, z64, y, g, eps, ignore, in_dt, out_dt):
    loss, lse, am = orc.ce_forward(z64, y, eps, ignore)
    rt, at = loss_tol(in_dt)
    assert_close(f32(r.loss), loss, rt, at, "loss")
    assert_close(f32(r.lse), lse, rt, at, "lse")
    np.testing.assert_array_equal(r.argmax.cpu().numpy(), am)
    ref = orc.ce_backward(z64, y, g, eps, ignore)
    assert_grad_close(f32(dz).reshape(z64.shape), ref, in_dt, out_dt, g=g)


def test_c2_fused_matches_separate(orc):
    """1,048,576 x 128 fp32, 10% ignore_index, eps 0.1, g = 1/count."""
    z, z32, y = wl.c2()
    zt, yt = upload(z), upload(y)
    g = torch.full((1,), 1.0 / float((y != -100).sum()), device="cuda")
    rf, dzf = ce.ce_forward_backward(zt, yt, g, wl.C2_EPS, return_argmax=True)
    rs, dzs = separate(zt, yt, g, wl.C2_EPS)
    torch.cuda.synchronize()
    for a, b in zip(rf, rs):
        assert torch.equal(a, b)
    assert close_ulps(dzf, dzs, float(g.item()))
    check_oracle(orc, rf, dzf, z32.astype(np.float64), y, float(g.item()), wl.C2_EPS, -100,
                 "f32", "f32")


@pytest.mark.parametrize("V", [1, 2, 3, 8, 9, 100, 127, 128, 1000, 1023, 1024])
def test_short_rows(orc, V):
    z, z32, y = wl.rows(777, V, "f32", seed=V + 50, ignore_frac=0.1)
    gv = np.random.default_rng(V).standard_normal(777).astype(np.float32)
    zt, yt, gt = upload(z), upload(y), upload(gv)
    for eps in (0.0, 0.2):
        rf, dzf = ce.ce_forward_backward(zt, yt, gt, eps, return_argmax=True)
        rs, dzs = separate(zt, yt, gt, eps)
        torch.cuda.synchronize()
        assert torch.equal(rf.loss, rs.loss) and torch.equal(rf.lse, rs.lse)
        assert torch.equal(rf.lse_lo, rs.lse_lo) and torch.equal(rf.argmax, rs.argmax)
        assert close_ulps(dzf, dzs, gt)
        check_oracle(orc, rf, dzf, z32.astype(np.float64), y, gv.astype(np.float64), eps, -100,
                     "f32", "f32")


@pytest.mark.parametrize("out", ["bf16", "f32"])
def test_bf16_short_and_long_rows(orc, out):
    od = torch.bfloat16 if out == "bf16" else torch.float32
    for V in (1000, 4097, 32000):  # the last two take the forward-then-VJP path
        z, z32, y = wl.rows(300, V, "bf16", seed=V, std=2.0)
        zt, yt = upload(z, "bf16"), upload(y)
        rf, dzf = ce.ce_forward_backward(zt, yt, torch.ones(1, device="cuda"), 0.1,
                                         return_argmax=True, out_dtype=od)
        torch.cuda.synchronize()
        check_oracle(orc, rf, dzf, z32.astype(np.float64), y, 1.0, 0.1, -100, "bf16", out)


def test_tiny_rows_many(orc):
    """Rows of 8 classes (the huge-row-count shape), fewer rows."""
    z, y = wl.c4b_chunk(0, chunk=1 << 20)
    zt, yt = upload(z), upload(y)
    g = torch.full((1,), 1.0 / z.shape[0], device="cuda")
    rf, dzf = ce.ce_forward_backward(zt, yt, g, return_argmax=True)
    rs, dzs = separate(zt, yt, g, 0.0)
    torch.cuda.synchronize()
    assert torch.equal(rf.loss, rs.loss) and close_ulps(dzf, dzs, 1.0 / z.shape[0])
    check_oracle(orc, rf, dzf, z.astype(np.float64), y, 1.0 / z.shape[0], 0.0, -100, "f32", "f32")


def test_in_place_and_strided(orc):
    x, t = wl.c4a(B=6, L=33, V=500)
    xt, tt = upload(x), upload(t)
    zv, yv = xt[:, :-1], tt[:, 1:]
    ref_r, ref_dz = separate(zv, yv, torch.ones(1, device="cuda"), 0.0)
    ref_dz = ref_dz.clone()
    rf, dzf = ce.ce_forward_backward(zv, yv, torch.ones(1, device="cuda"), dlogits=zv,
                                     return_argmax=True)
    torch.cuda.synchronize()
    assert dzf.data_ptr() == zv.data_ptr()
    assert torch.equal(rf.loss, ref_r.loss)
    assert close_ulps(zv, ref_dz)


def test_bad_targets_and_nonfinite(orc):
    V = 300
    rng = np.random.default_rng(3)
    z = rng.standard_normal((16, V)).astype(np.float32)
    y = rng.integers(0, V, size=16).astype(np.int32)
    y[2] = V + 5
    z[4, 7] = np.nan
    z[5, :] = -np.inf
    z[6, 11] = -np.inf
    rf, dzf = ce.ce_forward_backward(upload(z), upload(y), torch.ones(1, device="cuda"), 0.1,
                                     return_argmax=True)
    torch.cuda.synchronize()
    assert ce.get_error() == 5
    check_oracle(orc, rf, dzf, z.astype(np.float64), y, 1.0, 0.1, -100, "f32", "f32")


# -- rows held in shared memory (one CTA, or a cluster of 2, 4 or 8 per row) ----------------
def _padded(N, V, pad, dtype, seed, std=2.0, ignore_frac=0.1):
    """Logits (N, V) as a view of an (N, V + pad) buffer, so rows stay 16-byte
    aligned when V is not a multiple of the vector width (a ragged tail)."""
    z, z32, y = wl.rows(N, V + pad, dtype, seed=seed, std=std, ignore_frac=ignore_frac)
    y = np.where(y >= V, y % V, y).astype(y.dtype)  # targets inside the view
    return z, z32[:, :V], y


@pytest.mark.parametrize("V,N,dt", [
    (2048, 400, "bf16"),       # shared memory, one CTA, 2 chunks
    (32000, 600, "bf16"),      # shared memory, the 8192 x 32000 row shape
    (33000, 300, "f16"),       # shared memory, partial last chunk
    (57344, 300, "bf16"),      # shared memory, the largest row (56 chunks, 112 KB)
    (57352, 300, "bf16"),      # one vector more: an L2 slice, cluster of 1
    (100000, 200, "bf16"),     # L2 slices, cluster of 2
    (151936, 160, "bf16"),     # L2 slices, cluster of 4, the 2048 x 151,936 row shape
    (20000, 300, "f32"),       # shared memory, fp32
    (100000, 80, "f32"),       # L2 slices, cluster of 4, fp32
    (151936, 40, "f32"),       # L2 slices, cluster of 8 (608 KB rows)
    (151936, 30, "bf16"),      # too few rows for every SM: the forward, then the VJP
    (524288, 24, "bf16"),      # the largest L2-slice row: 8 slices of exactly 128 KB
    (524296, 24, "bf16"),      # one vector more: the forward, then the VJP
    (600000, 12, "bf16"),      # beyond 8 slices of 128 KB: the forward, then the VJP
])
def test_smem_rows_vs_oracle(orc, V, N, dt):
    z, z32, y = wl.rows(N, V, dt, seed=V % 997 + N, std=2.0, ignore_frac=0.1)
    gv = np.random.default_rng(V).standard_normal(N).astype(np.float32)
    zt, yt, gt = upload(z, dt), upload(y), upload(gv)
    for eps, am in ((0.0, False), (0.1, True)):
        rf, dzf = ce.ce_forward_backward(zt, yt, gt, eps, return_argmax=am)
        torch.cuda.synchronize()
        assert ce.get_error() == 0
        loss, lse, amx = orc.ce_forward(z32.astype(np.float64), y, eps)
        rt, at = loss_tol(dt)
        assert_close(f32(rf.loss), loss, rt, at, "loss")
        assert_close(f32(rf.lse), lse, rt, at, "lse")
        if am:
            np.testing.assert_array_equal(rf.argmax.cpu().numpy(), amx)
        ref = orc.ce_backward(z32.astype(np.float64), y, gv.astype(np.float64), eps)
        assert_grad_close(f32(dzf), ref, dt, dt, g=gv)
        # the same lse as the separate forward, up to the order of the sum
        rs = ce.ce_forward(zt, yt, eps)
        assert_close(f32(rf.lse), f32(rs.lse).astype(np.float64), 2e-6, 0.0, "lse vs ce_forward")


@pytest.mark.parametrize("out", ["bf16", "f32"])
@pytest.mark.parametrize("V", [32005, 100005])
def test_smem_rows_ragged_tail_views(orc, out, V):
    """V = 32005 (shared memory) and 100005 (L2 slices, cluster of 2): 5
    columns past the last 16-byte vector, rows of a padded buffer; dlogits is
    a padded view too, in bf16 or float."""
    N, pad = 300, 3
    z, z32, y = _padded(N, V, pad, "bf16", seed=5)
    zt = upload(z, "bf16")[:, :V]
    yt = upload(y)
    od = torch.bfloat16 if out == "bf16" else torch.float32
    dbuf = torch.empty((N, V + pad), dtype=od, device="cuda")
    dv = dbuf[:, :V]
    rf, dzf = ce.ce_forward_backward(zt, yt, torch.ones(1, device="cuda"), 0.2,
                                     return_argmax=True, dlogits=dv)
    torch.cuda.synchronize()
    assert dzf.data_ptr() == dbuf.data_ptr()
    check_oracle(orc, rf, dzf, z32.astype(np.float64), y, 1.0, 0.2, -100, "bf16", out)


def test_long_rows_strided_3d_view(orc):
    """The (B, L, V) view x[:, :-1] at V = 151,936 fp32 (rows of 607,744 bytes:
    L2 slices, cluster of 8), targets t[:, 1:]."""
    x, t = wl.c4a(B=3, L=21, V=151936)
    xt, tt = upload(x), upload(t)
    zv, yv = xt[:, :-1], tt[:, 1:]
    g = torch.full((1,), 0.5, device="cuda")
    rf, dzf = ce.ce_forward_backward(zv, yv, g, 0.0, return_argmax=True, dlogits=zv.clone())
    torch.cuda.synchronize()
    z64 = x[:, :-1].reshape(-1, x.shape[-1]).astype(np.float64)
    y = t[:, 1:].reshape(-1)
    check_oracle(orc, rf, dzf.reshape(-1, x.shape[-1]), z64, y, 0.5, 0.0, -100, "f32", "f32")


@pytest.mark.parametrize("V", [32000, 151936])
def test_smem_rows_in_place_and_repeatable(V):
    """Shared memory (32000) and L2 slices (151,936): two calls give the same
    bits, and so does a call that writes dlogits over its own logits."""
    z, z32, y = wl.rows(300, V, "bf16", seed=9, std=2.0, ignore_frac=0.2)
    zt, yt = upload(z, "bf16"), upload(y)
    g = torch.ones(1, device="cuda")
    r1, d1 = ce.ce_forward_backward(zt, yt, g, 0.1, return_argmax=True)
    r2, d2 = ce.ce_forward_backward(zt, yt, g, 0.1, return_argmax=True)
    zc = zt.clone()
    r3, d3 = ce.ce_forward_backward(zc, yt, g, 0.1, return_argmax=True, dlogits=zc)
    torch.cuda.synchronize()
    for a, b in zip(r1, r2):
        assert torch.equal(a, b)
    assert torch.equal(d1, d2)
    for a, b in zip(r1, r3):
        assert torch.equal(a, b)
    assert d3.data_ptr() == zc.data_ptr() and torch.equal(d1, zc)


@pytest.mark.parametrize("V", [20000, 40000])
def test_smem_rows_bad_targets_and_nonfinite(orc, V):
    """fp32 rows in shared memory (20000) and in L2 slices (40000, cluster of
    2): bad and ignored targets, NaN, -inf and huge logits."""
    N = 200
    rng = np.random.default_rng(7)
    z32 = rng.standard_normal((N, V)).astype(np.float32)
    y = rng.integers(0, V, size=N).astype(np.int32)
    y[3] = V
    y[4] = -7
    y[5] = -100
    z32[6, 12345] = np.nan
    z32[7, :] = -np.inf
    z32[8, 100:200] = -np.inf
    z32[9, y[9]] = -np.inf
    z32[10, :] = 1e30
    rf, dzf = ce.ce_forward_backward(upload(z32), upload(y), torch.ones(1, device="cuda"), 0.0,
                                     return_argmax=True)
    torch.cuda.synchronize()
    assert ce.get_error() == 5
    check_oracle(orc, rf, dzf, z32.astype(np.float64), y, 1.0, 0.0, -100, "f32", "f32")


# -- tiny rows (one or two 16-byte vectors): one lane per row --------------------------------
@pytest.mark.parametrize("V,dt,out", [(4, "f32", "f32"), (8, "f32", "f32"), (8, "bf16", "bf16"),
                                      (16, "bf16", "f32"), (8, "f16", "f16"), (16, "f16", "f16")])
def test_tiny_rows_fused(orc, V, dt, out):
    N = 3000 + V
    z, z32, y = wl.rows(N, V, dt, seed=40 + V, std=2.0, ignore_frac=0.1)
    y = y.copy()
    y[3] = -5                     # bad target
    y[9] = 0
    z32 = z32.copy()
    z32[4, 1] = np.nan
    z32[5, :] = -np.inf
    z32[6, 0] = -np.inf
    z32[9, :] = 1e4
    z, z32 = wl.encode(z32, dt)
    gv = np.random.default_rng(V).standard_normal(N).astype(np.float32)
    zt, yt, gt = upload(z, dt), upload(y), upload(gv)
    od = {"f32": torch.float32, "bf16": torch.bfloat16, "f16": torch.float16}[out]
    for eps, am in ((0.0, True), (0.1, False)):
        rf, dzf = ce.ce_forward_backward(zt, yt, gt, eps, return_argmax=am, out_dtype=od)
        rs = ce.ce_forward(zt, yt, eps, return_argmax=am)
        torch.cuda.synchronize()
        assert ce.get_error() == 5
        for a, b in zip(rf, rs):  # bit for bit, NaN rows included
            assert (a is None and b is None) or torch.equal(a.view(torch.int32), b.view(torch.int32))
        loss, lse, amx = orc.ce_forward(z32.astype(np.float64), y, eps)
        rt, at = loss_tol(dt)
        assert_close(f32(rf.loss), loss, rt, at, "loss")
        assert_close(f32(rf.lse), lse, rt, at, "lse")
        if am:
            np.testing.assert_array_equal(rf.argmax.cpu().numpy(), amx)
        ref = orc.ce_backward(z32.astype(np.float64), y, gv.astype(np.float64), eps)
        assert_grad_close(f32(dzf), ref, dt, out, g=gv)


def test_tiny_rows_fused_in_place_view(orc):
    """In place on the (B, L, 8) view x[:, :-1]."""
    x, t = wl.c4a(B=5, L=97, V=8)
    xt, tt = upload(x), upload(t)
    zv, yv = xt[:, :-1], tt[:, 1:]
    rf, dzf = ce.ce_forward_backward(zv, yv, torch.ones(1, device="cuda"), 0.1, dlogits=zv)
    torch.cuda.synchronize()
    assert dzf.data_ptr() == zv.data_ptr()
    z64 = x[:, :-1].reshape(-1, 8).astype(np.float64)
    y = t[:, 1:].reshape(-1)
    loss, _, _ = orc.ce_forward(z64, y, 0.1)
    assert_close(f32(rf.loss), loss, 1e-5, 1e-6, "loss")
    ref = orc.ce_backward(z64, y, 1.0, 0.1)
    assert_grad_close(f32(zv).reshape(-1, 8), ref, "f32", "f32")
