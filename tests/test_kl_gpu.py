"""KL divergence of a student distribution from a teacher's on the GPU,
through the C ABI, against the float64 oracle; and the self-check of "One
barrier short": repeated calls on one large input return the same bytes."""
from __future__ import annotations

import numpy as np
import pytest

from tests.gpu_util import assert_close, assert_grad_close, f32, torch, upload

import softmax_cross_entropy_lse_b200 as ce
from softmax_cross_entropy_lse_b200 import workloads as wl

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    ce.lib()
    yield


def pair(N, V, dt, seed, scale=4.0):
    """Student and teacher logits ~N(0, scale^2) (the page's draw is scale 4)."""
    rng = np.random.default_rng(seed)
    q, q32 = wl.encode(rng.standard_normal((N, V), dtype=np.float32) * scale, dt)
    p, p32 = wl.encode(rng.standard_normal((N, V), dtype=np.float32) * scale, dt)
    return q, q32, p, p32


def check(orc, r, dq, q32, p32, g, dt, od, rows=None):
    rows = np.arange(q32.shape[0]) if rows is None else rows
    loss, lq, lp = orc.kl_forward(q32.astype(np.float64), p32.astype(np.float64))
    # the loss is W / sp - (lse_p - lse_q), float sums of terms the size of
    # the logits: the page's bar of 1e-4 relative
    assert_close(f32(r.loss)[rows], loss, 1e-4, 1e-5, "loss")
    assert_close(f32(r.lse_student)[rows], lq, 1e-5, 1e-6, "student lse")
    assert_close(f32(r.lse_teacher)[rows], lp, 1e-5, 1e-6, "teacher lse")
    ref = orc.kl_backward(q32.astype(np.float64), p32.astype(np.float64), g)
    assert_grad_close(f32(dq).reshape(-1, q32.shape[1])[rows], ref, dt, od, g=g)


@pytest.mark.parametrize("V", [1, 7, 100, 1000, 4099, 32000])
@pytest.mark.parametrize("dt", ["f32", "bf16", "f16"])
def test_kl_rows_vs_oracle(orc, V, dt):
    N = 256 if V >= 4000 else 700
    q, q32, p, p32 = pair(N, V, dt, seed=V + 11, scale=4.0 if dt != "f16" else 2.0)
    # per-row upstream gradients ~N(0, 1); the gradient bound of row i scales
    # with max(1, |g_i|), as in every parity test
    gv = np.random.default_rng(V).standard_normal(N).astype(np.float32)
    qt, pt, gt = upload(q, dt), upload(p, dt), upload(gv)
    r = ce.kl_forward(qt, pt)
    dq = ce.kl_backward(gt, qt, pt, r)
    torch.cuda.synchronize()
    check(orc, r, dq, q32, p32, gv.astype(np.float64), dt, dt)


def test_kl_page_shape_sampled_and_repeatable(orc):
    """512 x 151,936 fp32, both ~N(0, 16): sampled rows against the oracle,
    and 20 calls on the same input give the same bytes for the loss and the
    gradient (the self-check "One barrier short" recommends)."""
    N, V = 512, 151936
    q, q32, p, p32 = pair(N, V, "f32", seed=0)
    qt, pt = upload(q), upload(p)
    g = torch.ones(1, device="cuda")
    r0 = ce.kl_forward(qt, pt)
    d0 = ce.kl_backward(g, qt, pt, r0)
    torch.cuda.synchronize()
    rows = np.array([0, 1, 77, 255, 256, 400, 511])
    check(orc, ce.KlResult(*(x[rows] for x in r0)), d0[rows], q32[rows], p32[rows], 1.0, "f32", "f32")
    losses = {r0.loss.cpu().numpy().tobytes()}
    grads = {d0.sum(1).cpu().numpy().tobytes()}
    for _ in range(19):
        r = ce.kl_forward(qt, pt)
        d = ce.kl_backward(g, qt, pt, r)
        torch.cuda.synchronize()
        losses.add(r.loss.cpu().numpy().tobytes())
        assert torch.equal(d, d0)
        grads.add(d.sum(1).cpu().numpy().tobytes())
    assert len(losses) == 1 and len(grads) == 1


def test_kl_equal_distributions_and_shift(orc):
    """Student equal to the teacher: loss 0 and a zero gradient, exactly.
    A constant added to a row changes neither."""
    q, q32, _, _ = pair(300, 2000, "f32", seed=2)
    qt = upload(q)
    r = ce.kl_forward(qt, qt.clone())
    d = ce.kl_backward(torch.ones(1, device="cuda"), qt, qt.clone(), r)
    torch.cuda.synchronize()
    assert torch.count_nonzero(r.loss).item() == 0 and torch.count_nonzero(d).item() == 0
    # exact shifts on a 1/64 grid
    rng = np.random.default_rng(3)
    zq = (rng.integers(-512, 512, size=(300, 1000)) / 64.0).astype(np.float32)
    zp = (rng.integers(-512, 512, size=(300, 1000)) / 64.0).astype(np.float32)
    a = ce.kl_forward(upload(zq), upload(zp))
    b = ce.kl_forward(upload(zq + 256.0), upload(zp - 128.0))
    torch.cuda.synchronize()
    assert_close(f32(b.loss), f32(a.loss).astype(np.float64), 0.0, 2e-4, "shifted loss")


def test_kl_strided_views_in_place_and_bf16_to_f32(orc):
    B, L, V = 3, 41, 3000
    rng = np.random.default_rng(4)
    xq, xq32 = wl.encode(rng.standard_normal((B, L, V), dtype=np.float32) * 3, "bf16")
    xp, xp32 = wl.encode(rng.standard_normal((B, L, V), dtype=np.float32) * 3, "bf16")
    qt, pt = upload(xq, "bf16"), upload(xp, "bf16")
    qv, pv = qt[:, :-1], pt[:, 1:]
    r = ce.kl_forward(qv, pv)
    dq = ce.kl_backward(torch.ones(1, device="cuda"), qv, pv, r, out_dtype=torch.float32)
    torch.cuda.synchronize()
    q64 = xq32[:, :-1].reshape(-1, V)
    p64 = xp32[:, 1:].reshape(-1, V)
    check(orc, r, dq, q64, p64, 1.0, "bf16", "f32")
    qc = qv.clone()
    d2 = ce.kl_backward(torch.ones(1, device="cuda"), qc, pv, r, dstudent=qc)
    torch.cuda.synchronize()
    assert d2.data_ptr() == qc.data_ptr()
    assert_grad_close(f32(qc).reshape(-1, V), orc.kl_backward(q64, p64, 1.0), "bf16", "bf16")


def test_kl_nonfinite_rows(orc):
    V = 500
    rng = np.random.default_rng(5)
    zq = rng.standard_normal((5, V)).astype(np.float32)
    zp = rng.standard_normal((5, V)).astype(np.float32)
    zp[0, 3] = -np.inf
    zq[0, 3] = -np.inf       # no teacher mass over a student -inf: finite
    zq[1, 7] = -np.inf       # teacher mass over a student -inf: +inf
    zq[2, 9] = np.nan        # NaN row
    zp[3, :] = -np.inf       # teacher all -inf: NaN
    r = ce.kl_forward(upload(zq), upload(zp))
    dq = ce.kl_backward(torch.ones(1, device="cuda"), upload(zq), upload(zp), r)
    torch.cuda.synchronize()
    check(orc, r, dq, zq, zp, 1.0, "f32", "f32")
