"""Cross-entropy against probability (soft) targets on the GPU, through the C
ABI, against the float64 oracle (the targets the oracle sees are the decoded
values of the stored ones)."""
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


def draw(N, V, dt, tdt, seed, kind="dist"):
    """Logits ~N(0, 2) in dt and targets in tdt: a distribution per row
    ("dist"), unnormalised non-negative weights ("raw"), or a distribution
    with most classes at exactly zero ("sparse")."""
    rng = np.random.default_rng(seed)
    z, z32 = wl.encode(rng.standard_normal((N, V), dtype=np.float32) * 2, dt)
    t = rng.random((N, V), dtype=np.float32)
    if kind == "sparse":
        t[rng.random((N, V)) < 0.9] = 0.0
    if kind in ("dist", "sparse"):
        t /= np.maximum(t.sum(1, keepdims=True), 1e-30)
    t, t32 = wl.encode(t, tdt)
    return z, z32, t, t32


def check(orc, r, dz, z32, t32, g, eps, dt, od):
    loss, lse = orc.ce_soft_forward(z32.astype(np.float64), t32.astype(np.float64), eps)
    rt, at = loss_tol(dt)
    assert_close(f32(r.loss), loss, rt, at, "loss")
    assert_close(f32(r.lse), lse, rt, at, "lse")
    np.testing.assert_allclose(f32(r.target_sum), t32.astype(np.float64).sum(1), rtol=1e-5, atol=1e-6)
    ref = orc.ce_soft_backward(z32.astype(np.float64), t32.astype(np.float64), g, eps)
    assert_grad_close(f32(dz).reshape(ref.shape), ref, dt, od, g=g)


@pytest.mark.parametrize("V", [1, 3, 8, 100, 1000, 1023, 4099, 32000])
@pytest.mark.parametrize("dt,tdt", [("f32", "f32"), ("bf16", "bf16"), ("bf16", "f32"), ("f16", "f16")])
def test_soft_rows_vs_oracle(orc, V, dt, tdt):
    N = 300 if V >= 4000 else 777
    z, z32, t, t32 = draw(N, V, dt, tdt, seed=V + 7)
    gv = np.random.default_rng(V).standard_normal(N).astype(np.float32)
    zt, tt, gt = upload(z, dt), upload(t, tdt), upload(gv)
    for eps in (0.0, 0.1):
        r = ce.ce_soft_forward(zt, tt, eps)
        dz = ce.ce_soft_backward(gt, zt, tt, r.lse, r.lse_lo, r.target_sum, eps)
        torch.cuda.synchronize()
        check(orc, r, dz, z32, t32, gv.astype(np.float64), eps, dt, dt)


@pytest.mark.parametrize("kind", ["raw", "sparse"])
def test_soft_unnormalised_and_sparse_targets(orc, kind):
    z, z32, t, t32 = draw(500, 2000, "bf16", "f32", seed=3, kind=kind)
    zt, tt = upload(z, "bf16"), upload(t)
    g = torch.ones(1, device="cuda")
    r = ce.ce_soft_forward(zt, tt, 0.05)
    dz = ce.ce_soft_backward(g, zt, tt, r.lse, r.lse_lo, r.target_sum, 0.05, out_dtype=torch.float32)
    torch.cuda.synchronize()
    check(orc, r, dz, z32, t32, 1.0, 0.05, "bf16", "f32")


def test_soft_normalised_targets_without_target_sum(orc):
    """target_sum None: the backward takes every row of t to sum to 1."""
    z, z32, t, t32 = draw(400, 777, "f32", "f32", seed=4)
    zt, tt = upload(z), upload(t)
    g = torch.full((1,), 0.5, device="cuda")
    r = ce.ce_soft_forward(zt, tt)
    dz = ce.ce_soft_backward(g, zt, tt, r.lse, r.lse_lo, None)
    torch.cuda.synchronize()
    ref = orc.ce_soft_backward(z32.astype(np.float64), t32.astype(np.float64), 0.5)
    # the rows of t32 sum to 1 up to float rounding: within that of the exact T
    np.testing.assert_allclose(f32(dz), ref, rtol=0, atol=2e-6)


def test_soft_strided_views_and_in_place(orc):
    """Logits x[:, :-1] of a (B, L, V) tensor and targets t[:, 1:] of another,
    gradient written in place over the logits view."""
    B, L, V = 4, 37, 1000
    rng = np.random.default_rng(5)
    x = rng.standard_normal((B, L, V), dtype=np.float32)
    tfull = rng.random((B, L, V), dtype=np.float32)
    tfull /= tfull.sum(-1, keepdims=True)
    xt, tt = upload(x), upload(tfull)
    zv, tv = xt[:, :-1], tt[:, 1:]
    r = ce.ce_soft_forward(zv, tv, 0.1)
    dz = ce.ce_soft_backward(torch.ones(1, device="cuda"), zv, tv, r.lse, r.lse_lo, r.target_sum, 0.1,
                             dlogits=zv)
    torch.cuda.synchronize()
    assert dz.data_ptr() == zv.data_ptr()
    z64 = x[:, :-1].reshape(-1, V).astype(np.float64)
    t64 = tfull[:, 1:].reshape(-1, V).astype(np.float64)
    loss, lse = orc.ce_soft_forward(z64, t64, 0.1)
    assert_close(f32(r.loss), loss, 1e-5, 1e-6, "loss")
    ref = orc.ce_soft_backward(z64, t64, 1.0, 0.1)
    assert_grad_close(f32(zv).reshape(-1, V), ref, "f32", "f32")


def test_soft_one_hot_equals_hard_targets(orc):
    z, z32, y = wl.rows(600, 3000, "bf16", seed=6, std=2.0)
    t = np.zeros((600, 3000), np.float32)
    t[np.arange(600), y] = 1.0
    zt, tt, yt = upload(z, "bf16"), upload(t), upload(y)
    for eps in (0.0, 0.2):
        rs = ce.ce_soft_forward(zt, tt, eps)
        rh = ce.ce_forward(zt, yt, eps)
        torch.cuda.synchronize()
        assert_close(f32(rs.loss), f32(rh.loss).astype(np.float64), 2e-6, 1e-6, "soft vs hard loss")
        assert_close(f32(rs.lse), f32(rh.lse).astype(np.float64), 1e-6, 0.0, "soft vs hard lse")


def test_soft_nonfinite_rows(orc):
    V = 700
    rng = np.random.default_rng(8)
    z = rng.standard_normal((6, V)).astype(np.float32)
    t = rng.random((6, V)).astype(np.float32)
    t /= t.sum(1, keepdims=True)
    z[0, 5] = -np.inf
    t[0, 5] = 0.0            # zero mass on a -inf logit: finite
    z[1, 9] = -np.inf        # mass on a -inf logit: +inf
    z[2, 100] = np.nan       # NaN row
    z[3, :] = -np.inf        # all -inf
    z[4, :] = 1e30           # equal huge logits: loss log V
    r = ce.ce_soft_forward(upload(z), upload(t))
    dz = ce.ce_soft_backward(torch.ones(1, device="cuda"), upload(z), upload(t), r.lse, r.lse_lo,
                             r.target_sum)
    torch.cuda.synchronize()
    check(orc, r, dz, z, t, 1.0, 0.0, "f32", "f32")
    assert abs(r.loss[4].item() - np.log(V)) < 1e-5 * np.log(V)


def test_soft_rejects_mismatched_shapes():
    z = torch.zeros((4, 10), device="cuda")
    with pytest.raises(ValueError):
        ce.ce_soft_forward(z, torch.zeros((4, 11), device="cuda"))
    with pytest.raises(ce.CEError):
        ce.ce_soft_forward(z.to(torch.bfloat16), torch.zeros((4, 10), dtype=torch.float16, device="cuda"))
