"""Row cross-entropy on the GPU, through the C ABI, against the float64 oracle.

Every input is a seeded synthetic draw from softmax_cross_entropy_lse_b200.workloads;
the oracle sees the identical values. Configurations follow the workloads of
the pages (the strided next-token view, the huge row count, LM vocabularies)
at full size where the oracle can follow, and on sampled rows where it cannot
hold the whole problem.
"""
from __future__ import annotations

import numpy as np
import pytest

from tests.gpu_util import (assert_close, assert_grad_close, f32, loss_tol, torch, upload)

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


def run_fwd_bwd(z_t, y_t, eps=0.0, ignore=-100, g=None, out_dtype=None, argmax=True):
    r = ce.ce_forward(z_t, y_t, eps, ignore, return_argmax=argmax)
    N = r.loss.numel()
    if g is None:
        g = torch.ones(1, dtype=torch.float32, device=z_t.device)
    dz = ce.ce_backward(g, z_t, y_t, r.lse, r.lse_lo, eps, ignore, out_dtype=out_dtype)
    torch.cuda.synchronize()
    return r, dz


def check_rows(orc, r, dz, z64, y, eps, ignore, in_dtype, out_dtype, g=1.0, rows=None):
    rows = np.arange(z64.shape[0]) if rows is None else rows
    loss, lse, am = orc.ce_forward(z64, y, eps, ignore)
    rt, at = loss_tol(in_dtype)
    assert_close(f32(r.loss)[rows], loss, rt, at, "loss")
    assert_close(f32(r.lse)[rows], lse, rt, at, "lse")
    if r.argmax is not None:
        np.testing.assert_array_equal(r.argmax.cpu().numpy()[rows], am)
    ref = orc.ce_backward(z64, y, g, eps, ignore)
    assert_grad_close(f32(dz).reshape(-1, z64.shape[1])[rows], ref, in_dtype, out_dtype, g=g)


# ---------------------------------------------------------------------------
# c1: 4096 x 1024 fp32, and the equal-logit / offset rows of MLX PR #4188
def test_c1_full(orc):
    z, z32, y = wl.c1()
    r, dz = run_fwd_bwd(upload(z), upload(y))
    check_rows(orc, r, dz, z32.astype(np.float64), y, 0.0, -100, "f32", "f32")
    # lse_lo is the float residual of the exact lse
    hi, lo = f32(r.lse).astype(np.float64), f32(r.lse_lo).astype(np.float64)
    _, lse64, _ = orc.ce_forward(z32.astype(np.float64), y)
    assert np.abs((hi + lo) - lse64).max() < 2e-6
    assert np.abs(lo).max() <= np.spacing(np.abs(hi).astype(np.float32)).max()


@pytest.mark.parametrize("eps", [0.0, 0.1, 0.5])
def test_c1_equal_logits_any_magnitude(orc, eps):
    """[v, v] with target 0: loss log 2 and gradient [-1/2, 1/2] (scaled by
    the smoothing) at every float32 magnitude up to 1e36."""
    z64, y = wl.special_rows_equal(tuple(10.0 ** k for k in range(0, 37, 2)) + (1e8, -1e8), 4)
    z = z64.astype(np.float32)
    r, dz = run_fwd_bwd(upload(z), upload(y), eps)
    loss = f32(r.loss)
    assert np.abs(loss - np.log(2.0)).max() <= 1e-6
    g = f32(dz)
    assert np.abs(g[:, 0] - (-0.5 + 0.5 * eps)).max() <= 1e-6
    assert np.abs(g[:, 1] - (0.5 - 0.5 * eps)).max() <= 1e-6
    check_rows(orc, r, dz, z.astype(np.float64), y, eps, -100, "f32", "f32")


def test_c1_shared_offset(orc):
    """[2, -1] + c: the float32 input keeps the gap up to c = 1e6 (loss
    0.04858735); at 1e8 the float32 values are equal and the exact loss of
    the stored input is log 2. Both must come out right."""
    z64, y = wl.special_rows_offset((0.0, 1e4, 1e6, 1e8, -1e8, 3e5))
    z = z64.astype(np.float32)
    r, dz = run_fwd_bwd(upload(z), upload(y))
    check_rows(orc, r, dz, z.astype(np.float64), y, 0.0, -100, "f32", "f32")
    loss = f32(r.loss)
    assert np.abs(loss[:3] - np.log1p(np.exp(-3.0))).max() <= 1e-6


@pytest.mark.parametrize("c", [1e4, 1e6, 1e7])
def test_random_rows_large_offset(orc, c):
    rng = np.random.default_rng(4)
    z = (rng.standard_normal((64, 1000)) + c).astype(np.float32)
    y = rng.integers(0, 1000, size=64).astype(np.int32)
    for eps in (0.0, 0.1):
        r, dz = run_fwd_bwd(upload(z), upload(y), eps)
        check_rows(orc, r, dz, z.astype(np.float64), y, eps, -100, "f32", "f32")


# ---------------------------------------------------------------------------
# c2: 1,048,576 x 128 fp32, 10% ignore_index, label smoothing 0.1
def test_c2_full(orc):
    z, z32, y = wl.c2()
    g = torch.full((1,), 1.0 / float((y != -100).sum()), device="cuda")
    r, dz = run_fwd_bwd(upload(z), upload(y), wl.C2_EPS, -100, g)
    check_rows(orc, r, dz, z32.astype(np.float64), y, wl.C2_EPS, -100, "f32", "f32",
               g=float(g.item()))
    assert (f32(r.loss)[y == -100] == 0).all()
    assert (f32(dz)[y == -100] == 0).all()


# ---------------------------------------------------------------------------
# c3: LM vocabularies in bf16 (std 2), float accumulation, bf16 or float dz
@pytest.mark.parametrize("V", [32000, 151936, 4097, 50257])
@pytest.mark.parametrize("out", ["bf16", "f32"])
def test_c3_bf16_reduced(orc, V, out):
    z, z32, y = wl.rows(300, V, "bf16", seed=V, std=2.0)
    od = torch.bfloat16 if out == "bf16" else torch.float32
    r, dz = run_fwd_bwd(upload(z, "bf16"), upload(y), out_dtype=od)
    check_rows(orc, r, dz, z32.astype(np.float64), y, 0.0, -100, "bf16", out)


@pytest.mark.parametrize("cfg", ["c3a", "c3b"])
def test_c3_full_size_sampled_rows(orc, cfg):
    z, z32, y = getattr(wl, cfg)()
    r, dz = run_fwd_bwd(upload(z, "bf16"), upload(y), out_dtype=torch.bfloat16)
    rows = np.random.default_rng(1).choice(z.shape[0], 96, replace=False)
    rows.sort()
    check_rows(orc, r, dz, z32[rows].astype(np.float64), y[rows], 0.0, -100, "bf16", "bf16",
               rows=rows)
    assert np.isfinite(f32(r.loss)).all()


def test_fp16_rows(orc):
    z, z32, y = wl.rows(513, 3001, "f16", seed=3, std=2.0)
    for out in ("f16", "f32"):
        od = torch.float16 if out == "f16" else torch.float32
        r, dz = run_fwd_bwd(upload(z), upload(y), 0.1, out_dtype=od)
        check_rows(orc, r, dz, z32.astype(np.float64), y, 0.1, -100, "f16", out)


# ---------------------------------------------------------------------------
# c4a: x (10, 119, 151936) fp32, CE on x[:, :-1] vs t[:, 1:], no copy
def test_c4a_strided_view(orc):
    x, t = wl.c4a()
    xd, td = upload(x), upload(t)
    zv, yv = xd[:, :-1], td[:, 1:]
    assert not zv.is_contiguous()
    r = ce.ce_forward(zv, yv, return_argmax=True)
    dx = torch.full_like(xd, float("nan"))
    ce.ce_backward(torch.ones(1, device="cuda"), zv, yv, r.lse, r.lse_lo, dlogits=dx[:, :-1])
    # same values made contiguous: bit-identical results
    zc, yc = zv.contiguous(), yv.contiguous()
    rc = ce.ce_forward(zc, yc, return_argmax=True)
    dc = ce.ce_backward(torch.ones(1, device="cuda"), zc, yc, rc.lse, rc.lse_lo)
    torch.cuda.synchronize()
    assert torch.equal(r.loss, rc.loss) and torch.equal(r.lse, rc.lse)
    assert torch.equal(r.argmax, rc.argmax)
    assert torch.equal(dx[:, :-1], dc)
    # the last position of each sequence was never written
    assert torch.isnan(dx[:, -1]).all()
    # oracle on sampled rows
    z = x[:, :-1].reshape(-1, x.shape[2])
    y = t[:, 1:].reshape(-1)
    rows = np.random.default_rng(2).choice(z.shape[0], 64, replace=False)
    rows.sort()
    check_rows(orc, r, dc.reshape(-1, x.shape[2]), z[rows].astype(np.float64), y[rows], 0.0,
               -100, "f32", "f32", rows=rows)
    # the issue's statistical expectation: grad norm ~ sqrt(1180)
    gn = torch.linalg.vector_norm(dc.double()).item()
    assert abs(gn - np.sqrt(1180)) < 0.05


# ---------------------------------------------------------------------------
# c4b: 2^27 + 2^20 rows x 8 fp32: no grid wrap, 64-bit row indexing
def test_c4b_huge_rows(orc):
    """Protocol of MLX PR #4776 ("Test and reproduction"): the whole batch of
    2^27 + 2^20 rows against a float64 reference computed in 2^22-row chunks,
    a row counted wrong when its loss or any entry of its gradient is off by
    more than 1e-3; the wrong-row count, the first wrong row and the largest
    errors are reported, and every row must also meet the fp32 tolerances.
    Outputs start as NaN, so an unwritten row shows as wrong."""
    n, V, C = wl.C4B_ROWS, 8, wl.C4B_CHUNK
    nchunks = (n + C - 1) // C
    z_d = torch.empty((n, V), dtype=torch.float32, device="cuda")
    y_d = torch.empty(n, dtype=torch.int32, device="cuda")
    for k in range(nchunks):
        zc, yc = wl.c4b_chunk(k)
        z_d[k * C:k * C + len(yc)].copy_(torch.from_numpy(zc))
        y_d[k * C:k * C + len(yc)].copy_(torch.from_numpy(yc))
    r = ce.ce_forward(z_d, y_d)
    dz = torch.full_like(z_d, float("nan"))
    ce.ce_backward(torch.ones(1, device="cuda"), z_d, y_d, r.lse, r.lse_lo, dlogits=dz)
    torch.cuda.synchronize()
    assert ce.get_error() == 0
    wrong, first_wrong, max_loss_err, max_grad_err = 0, None, 0.0, 0.0
    for k in range(nchunks):
        zc, yc = wl.c4b_chunk(k)  # the same seeded draw, regenerated
        lo = k * C
        z64 = zc.astype(np.float64)
        loss, lse, _ = orc.ce_forward(z64, yc)
        ref = orc.ce_backward(z64, yc, 1.0)
        gl = f32(r.loss[lo:lo + len(yc)]).astype(np.float64)
        gg = f32(dz[lo:lo + len(yc)]).astype(np.float64)
        le = np.abs(gl - loss)
        ge = np.abs(gg - ref).max(axis=1)
        bad = ~(le <= 1e-3) | ~(ge <= 1e-3)  # NaN counts as wrong
        if bad.any() and first_wrong is None:
            first_wrong = lo + int(np.argmax(bad))
        wrong += int(bad.sum())
        max_loss_err = max(max_loss_err, float(np.nan_to_num(le, nan=np.inf).max()))
        max_grad_err = max(max_grad_err, float(np.nan_to_num(ge, nan=np.inf).max()))
        assert_close(gl, loss, 1e-5, 1e-6, f"loss chunk {k}")
        assert_close(f32(r.lse[lo:lo + len(yc)]), lse, 1e-5, 1e-6, f"lse chunk {k}")
        assert_close(gg, ref, 0.0, 1e-6, f"dz chunk {k}")
    summary = (f"{n} rows: {wrong} wrong, first wrong row {first_wrong}, max error "
               f"{max_loss_err:.2e} (loss), {max_grad_err:.2e} (gradient)")
    print(summary)
    assert wrong == 0, summary
    del z_d, dz


# ---------------------------------------------------------------------------
# long rows with few of them: the vocabulary is split across CTAs and merged
@pytest.mark.parametrize("N,V,dt", [(3, 151936, "bf16"), (37, 151936, "bf16"),
                                    (5, 1 << 20, "f32"), (2, 262147, "f32")])
def test_split_vocabulary(orc, N, V, dt):
    z, z32, y = wl.rows(N, V, dt, seed=N + V, std=2.0)
    assert ce.ce_workspace_size(N, V, torch.bfloat16 if dt == "bf16" else torch.float32) > 0
    # the row max sits in the last split on row 0, tied with an earlier copy on row 1
    z32 = z32.copy()
    z32[0, V - 3] = 40.0
    if N > 1:
        z32[1, 5] = 40.0
        z32[1, V - 2] = 40.0
    z, z32 = wl.encode(z32, dt)
    od = torch.bfloat16 if dt == "bf16" else torch.float32
    r, dz = run_fwd_bwd(upload(z, dt), upload(y), 0.1, out_dtype=od)
    check_rows(orc, r, dz, z32.astype(np.float64), y, 0.1, -100, dt, dt)
    assert r.argmax[0].item() == V - 3
    if N > 1:
        assert r.argmax[1].item() == 5


# ---------------------------------------------------------------------------
# edge cases
@pytest.mark.parametrize("V", [1, 2, 3, 5, 8, 9, 31, 33, 127, 129, 255, 1023, 1025, 2049, 4095])
def test_ragged_widths(orc, V):
    z, z32, y = wl.rows(257, V, "f32", seed=V)
    for eps in (0.0, 0.1):
        r, dz = run_fwd_bwd(upload(z), upload(y), eps)
        check_rows(orc, r, dz, z32.astype(np.float64), y, eps, -100, "f32", "f32")


def test_empty_batch():
    z = torch.empty((0, 17), device="cuda")
    y = torch.empty(0, dtype=torch.int32, device="cuda")
    r = ce.ce_forward(z, y)
    dz = ce.ce_backward(torch.ones(1, device="cuda"), z, y, r.lse)
    assert r.loss.numel() == 0 and dz.shape == (0, 17)


def test_misaligned_and_strided_columns(orc):
    rng = np.random.default_rng(8)
    base = rng.standard_normal((301, 1003)).astype(np.float32)
    y = rng.integers(0, 1000, size=300).astype(np.int32)
    bd = upload(base)
    # rows that start off a 16-byte boundary: scalar path
    zv = bd[1:, 3:]
    r, dz = run_fwd_bwd(zv, upload(y))
    check_rows(orc, r, dz, base[1:, 3:].astype(np.float64), y, 0.0, -100, "f32", "f32")
    # columns with a stride (a transposed view)
    t = upload(np.ascontiguousarray(base[:, :300].T))  # (300, 301) contiguous
    zt = t.t()  # (301, 300), s_col = 301
    y2 = rng.integers(0, 300, size=301).astype(np.int32)
    r, dz = run_fwd_bwd(zt, upload(y2))
    check_rows(orc, r, dz, base[:, :300].astype(np.float64), y2, 0.0, -100, "f32", "f32")


def test_int64_targets_custom_ignore(orc):
    z, z32, y = wl.rows(1000, 777, "f32", seed=12)
    y64 = y.astype(np.int64)
    y64[::3] = 5
    r, dz = run_fwd_bwd(upload(z), upload(y64), 0.2, ignore=5)
    check_rows(orc, r, dz, z32.astype(np.float64), y64, 0.2, 5, "f32", "f32")


def test_bad_targets_flagged(orc):
    z, z32, y = wl.rows(64, 300, "f32", seed=13)
    y = y.copy()
    y[3] = 300
    y[7] = -1
    assert ce.get_error() == 0
    r, dz = run_fwd_bwd(upload(z), upload(y))
    assert ce.get_error() == 5
    assert ce.get_error() == 0  # cleared by the read
    check_rows(orc, r, dz, z32.astype(np.float64), y, 0.0, -100, "f32", "f32")


def test_nonfinite_inputs(orc):
    V = 600
    rng = np.random.default_rng(14)
    z = rng.standard_normal((8, V)).astype(np.float32)
    y = rng.integers(0, V, size=8).astype(np.int32)
    z[0, 17] = np.nan              # NaN row
    z[1, :] = -np.inf              # all -inf
    z[2, 5] = -np.inf              # one -inf, not the target
    y[2] = 6
    z[3, y[3]] = -np.inf           # target at -inf
    z[4, 100] = np.inf             # +inf
    z[5, [3, 400]] = 9.0           # argmax tie
    for eps in (0.0, 0.3):
        r, dz = run_fwd_bwd(upload(z), upload(y), eps)
        check_rows(orc, r, dz, z.astype(np.float64), y, eps, -100, "f32", "f32")
    assert ce.get_error() == 0


def test_in_place_backward(orc):
    z, z32, y = wl.rows(500, 5000, "bf16", seed=15, std=2.0)
    zt = upload(z, "bf16")
    r = ce.ce_forward(zt, upload(y))
    ref = ce.ce_backward(torch.ones(1, device="cuda"), zt, upload(y), r.lse, r.lse_lo)
    out = ce.ce_backward(torch.ones(1, device="cuda"), zt, upload(y), r.lse, r.lse_lo, dlogits=zt)
    torch.cuda.synchronize()
    assert out.data_ptr() == zt.data_ptr()
    assert torch.equal(zt, ref)


def test_grad_per_row_and_broadcast(orc):
    z, z32, y = wl.rows(700, 300, "f32", seed=16)
    g = np.random.default_rng(16).standard_normal(700).astype(np.float32)
    zt, yt = upload(z), upload(y)
    r = ce.ce_forward(zt, yt)
    dz = ce.ce_backward(upload(g), zt, yt, r.lse, r.lse_lo)
    torch.cuda.synchronize()
    ref = orc.ce_backward(z32.astype(np.float64), y, g.astype(np.float64))
    assert_grad_close(f32(dz), ref, "f32", "f32", "dz per-row g", g=g)
    # a strided grad_out view
    g2 = upload(np.repeat(g, 2))[::2]
    dz2 = ce.ce_backward(g2, zt, yt, r.lse, r.lse_lo)
    torch.cuda.synchronize()
    assert torch.equal(dz, dz2)


def test_repeat_calls_bitwise_identical():
    """One barrier short: call twice on the same large input and compare the
    bytes. Vocabulary-sized rows (128 x 151,936 fp32), ten calls."""
    z, _, y = wl.rows(128, 151936, "f32", seed=17, std=4.0)
    zt, yt = upload(z), upload(y)
    first = None
    for _ in range(10):
        r = ce.ce_forward(zt, yt, 0.1, return_argmax=True)
        dz = ce.ce_backward(torch.ones(1, device="cuda"), zt, yt, r.lse, r.lse_lo, 0.1)
        cur = (r.loss.clone(), r.lse.clone(), r.argmax.clone(), dz)
        if first is None:
            first = cur
        else:
            for a, b in zip(first, cur):
                assert torch.equal(a, b)
    # and through the split path
    z, _, y = wl.rows(4, 1 << 20, "f32", seed=18, std=4.0)
    zt, yt = upload(z), upload(y)
    outs = [ce.ce_forward(zt, yt, 0.1, return_argmax=True) for _ in range(10)]
    for o in outs[1:]:
        assert torch.equal(o.loss, outs[0].loss) and torch.equal(o.lse, outs[0].lse)


# ---------------------------------------------------------------------------
# tiny rows (one or two 16-byte vectors per row): one lane per row
@pytest.mark.parametrize("V,dt", [(4, "f32"), (8, "f32"), (8, "bf16"), (16, "bf16"),
                                  (8, "f16"), (16, "f16")])
def test_tiny_rows(orc, V, dt):
    N = 1000 + V  # not a multiple of the rows one block takes per step
    z, z32, y = wl.rows(N, V, dt, seed=300 + V, std=2.0, ignore_frac=0.1)
    y = y.copy()
    y[7] = V          # bad target
    y[14] = 1
    z32 = z32.copy()
    z32[11, 1] = np.nan
    z32[12, :] = -np.inf
    z32[13, 0] = -np.inf
    z32[14, :] = 3e36 if dt != "f16" else 6e4   # equal logits at a huge magnitude
    z32[15, [0, V - 1]] = 5.0                    # argmax tie
    z, z32 = wl.encode(z32, dt)
    od = {"f32": None, "bf16": torch.bfloat16, "f16": torch.float16}[dt]
    for eps, am in ((0.0, True), (0.1, False), (0.2, True)):
        r, dz = run_fwd_bwd(upload(z, dt), upload(y), eps, out_dtype=od, argmax=am)
        assert ce.get_error() == 5
        check_rows(orc, r, dz, z32.astype(np.float64), y, eps, -100, dt, dt)
        assert abs(r.loss[14].item() - np.log(V)) < 1e-5 * np.log(V) + 1e-6


def test_tiny_rows_strided_view_matches_copy(orc):
    """x[:, :-1] of a (B, L, 8) tensor (rows 32 bytes apart inside a batch,
    a jump between batches) equals the contiguous copy bit for bit."""
    x, t = wl.c4a(B=7, L=301, V=8)
    xt, tt = upload(x), upload(t)
    r1, d1 = run_fwd_bwd(xt[:, :-1], tt[:, 1:], 0.1)
    r2, d2 = run_fwd_bwd(xt[:, :-1].contiguous(), tt[:, 1:].contiguous(), 0.1)
    for a, b in zip(r1, r2):
        assert torch.equal(a, b)
    assert torch.equal(d1, d2)
    z64 = x[:, :-1].reshape(-1, 8).astype(np.float64)
    check_rows(orc, r1, d1, z64, t[:, 1:].reshape(-1), 0.1, -100, "f32", "f32")


@pytest.mark.parametrize("V,dt", [(4, "f32"), (8, "f32"), (16, "bf16")])
def test_tiny_rows_backward_per_row_g_and_in_place(orc, V, dt):
    """Tiny-row VJP with a per-row upstream gradient read through a strided
    view, and written over the logits it reads."""
    N = 3001
    z, z32, y = wl.rows(N, V, dt, seed=40 + V, std=2.0, ignore_frac=0.1)
    g = np.random.default_rng(V).standard_normal(N).astype(np.float32)
    zt, yt = upload(z, dt), upload(y)
    r = ce.ce_forward(zt, yt, 0.1)
    g2 = upload(np.repeat(g, 3))[::3]
    dz = ce.ce_backward(g2, zt, yt, r.lse, r.lse_lo, 0.1)
    torch.cuda.synchronize()
    ref = orc.ce_backward(z32.astype(np.float64), y, g.astype(np.float64), 0.1)
    assert_grad_close(f32(dz), ref, dt, dt, g=g)
    out = ce.ce_backward(g2, zt, yt, r.lse, r.lse_lo, 0.1, dlogits=zt)
    torch.cuda.synchronize()
    assert out.data_ptr() == zt.data_ptr()
    assert torch.equal(zt, dz)


def test_tiny_rows_forward_matches_fused():
    z, _, y = wl.rows(5000, 8, "f32", seed=2, ignore_frac=0.1)
    zt, yt = upload(z), upload(y)
    g = torch.full((1,), 0.25, device="cuda")
    for eps, am in ((0.0, False), (0.1, True)):
        rs = ce.ce_forward(zt, yt, eps, return_argmax=am)
        rf, _ = ce.ce_forward_backward(zt, yt, g, eps, return_argmax=am)
        torch.cuda.synchronize()
        for a, b in zip(rs, rf):
            assert (a is None and b is None) or torch.equal(a, b)


def test_forward_into_caller_outputs():
    """out=: the per-row results land in the caller's tensors, bit for bit the
    same as freshly allocated ones, for the forward and the fused call."""
    z, _, y = wl.rows(700, 3000, "bf16", seed=21, std=2.0, ignore_frac=0.1)
    zt, yt = upload(z, "bf16"), upload(y)
    out = ce.ForwardResult(*(torch.full((700,), float("nan"), device="cuda") for _ in range(3)),
                           torch.full((700,), -1, dtype=torch.int32, device="cuda"))
    ref = ce.ce_forward(zt, yt, 0.1, return_argmax=True)
    got = ce.ce_forward(zt, yt, 0.1, return_argmax=True, out=out)
    torch.cuda.synchronize()
    for a, b, c in zip(ref, got, out):
        assert b.data_ptr() == c.data_ptr() and torch.equal(a, b)
    g = torch.ones(1, device="cuda")
    ref2, _ = ce.ce_forward_backward(zt, yt, g, 0.1, return_argmax=True)
    got2, _ = ce.ce_forward_backward(zt, yt, g, 0.1, return_argmax=True, out=out)
    torch.cuda.synchronize()
    for a, b, c in zip(ref2, got2, out):
        assert b.data_ptr() == c.data_ptr() and torch.equal(a, b)
