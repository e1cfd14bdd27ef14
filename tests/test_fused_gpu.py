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
    assert_grad_close(f32(dz).reshape(z64.shape), ref, in_dt, out_dt)


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
    rf, dzf = ce.ce_forward_backward(zv, yv, torch.ones(1, device="cuda"), dlogits=zv)
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
