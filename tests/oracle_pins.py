"""Pins that tie the float64 oracle to facts other than itself.

Each pin takes an ``oracle.Oracle`` and raises AssertionError when the oracle
disagrees with what the pages or the mathematics fix. The same battery runs
against the real oracle (every pin must pass) and against copies of the
oracle with a planted mistake (at least one pin must fail), which shows that
the battery can see a dropped term, a flipped sign, a wrong index or a wrong
operand anywhere in the oracle.

Sources of truth used here:
  * MLX PR #4188 "Shift by the max in cross_entropy" (Proposed changes):
    printed values for equal logits and for a shared offset.
  * Closed forms: uniform rows, two-logit rows, gradient rows summing to 0.
  * Brute force in 50-digit arithmetic (mpmath) from the unshifted textbook
    definition, on tiny rows.
  * PyTorch's float64 cross_entropy with label_smoothing and ignore_index,
    and its autograd, as an independent library special case.
  * Central finite differences of the oracle's own forward.
  * numpy float64 matmul for Z = H W^T and for G W, G^T H (library step).
  * For probability targets: the hard-target oracle at one-hot targets, PyTorch's
    float64 cross_entropy with probability targets, closed forms, shift
    invariance and finite differences.
  * For the KL divergence: PyTorch's float64 kl_div and its autograd, zero at
    equal distributions, the two-class closed form, shift invariance, Gibbs'
    inequality, zero-sum gradient rows and finite differences.
"""
from __future__ import annotations

import math
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _read_golden_pr4188():
    out = []
    with open(os.path.join(GOLDEN, "shift_by_max_pr4188.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            kind, mag, val, tol = line.split()
            out.append((kind, float(mag), float(val), float(tol)))
    return out


def pin_pr4188_printed_values(orc):
    """Equal logits give log 2 and [2,-1]+c gives the printed 0.04858734."""
    for kind, mag, val, tol in _read_golden_pr4188():
        z = np.array([[mag, mag]]) if kind == "equal" else np.array([[2.0, -1.0]]) + mag
        loss, lse, _ = orc.ce_forward(z, np.array([0]))
        assert abs(loss[0] - val) <= tol, (kind, mag, loss[0], val)


def pin_equal_logits_closed_form(orc):
    """[v, v] -> loss log 2, lse v + log 2, grad [-1/2, 1/2], v up to 1e36."""
    mags = [10.0 ** k for k in range(0, 37)] + [-1e8, -1e36]
    z = np.array([[v, v] for v in mags])
    y = np.zeros(len(mags), np.int64)
    for eps in (0.0, 0.1, 0.5):
        loss, lse, am = orc.ce_forward(z, y, eps=eps)
        # eps spreads over both classes equally: the smoothed loss is still log 2
        np.testing.assert_allclose(loss, math.log(2.0), rtol=1e-15, atol=0)
        np.testing.assert_allclose(lse, np.array(mags) + math.log(2.0), rtol=1e-15)
        assert (am == 0).all()
        dz = orc.ce_backward(z, y, 1.0, eps=eps)
        # p = [1/2, 1/2]: dz_0 = 1/2 - (1-eps) - eps/2, dz_1 = 1/2 - eps/2
        np.testing.assert_allclose(dz[:, 0], -0.5 + 0.5 * eps, rtol=1e-14)
        np.testing.assert_allclose(dz[:, 1], 0.5 - 0.5 * eps, rtol=1e-14)


def pin_two_logit_offset_closed_form(orc):
    """[2,-1]+c: loss log(1+e^-3); grad -/+ e^-3/(1+e^-3) (exact in double)."""
    offs = [0.0, 1e4, 1e6, 1e8, -1e8]
    z = np.array([[2.0, -1.0]]) + np.array(offs)[:, None]
    y = np.zeros(len(offs), np.int64)
    loss, lse, _ = orc.ce_forward(z, y)
    np.testing.assert_allclose(loss, math.log1p(math.exp(-3.0)), rtol=1e-12)
    np.testing.assert_allclose(lse - z[:, 0], math.log1p(math.exp(-3.0)), rtol=1e-7)
    dz = orc.ce_backward(z, y, 1.0)
    q = math.exp(-3.0) / (1.0 + math.exp(-3.0))
    np.testing.assert_allclose(dz[:, 0], -q, rtol=1e-12)
    np.testing.assert_allclose(dz[:, 1], q, rtol=1e-12)
    # target on the smaller logit: loss 3 + log(1+e^-3)
    loss1, _, _ = orc.ce_forward(z, np.ones(len(offs), np.int64))
    np.testing.assert_allclose(loss1, 3.0 + math.log1p(math.exp(-3.0)), rtol=1e-12)


def pin_uniform_rows_closed_form(orc):
    """V equal values: loss log V (any eps), lse v + log V, grad 1/V - onehot."""
    for V in (1, 3, 128, 1000):
        for v in (0.0, -7.5, 3e5):
            z = np.full((2, V), v)
            y = np.array([0, V - 1])
            for eps in (0.0, 0.1):
                loss, lse, am = orc.ce_forward(z, y, eps=eps)
                np.testing.assert_allclose(loss, math.log(V), rtol=1e-13, atol=1e-13)
                np.testing.assert_allclose(lse, v + math.log(V), rtol=1e-13, atol=1e-13)
                assert (am == 0).all()
                dz = orc.ce_backward(z, y, 2.0, eps=eps)
                ref = np.full((2, V), 2.0 * (1.0 / V - eps / V))
                ref[0, 0] -= 2.0 * (1 - eps)
                ref[1, V - 1] -= 2.0 * (1 - eps)
                np.testing.assert_allclose(dz, ref, rtol=1e-12, atol=1e-15)


def pin_bruteforce_mpmath(orc):
    """Tiny rows against the unshifted textbook formulas in 50-digit arithmetic."""
    import mpmath
    mpmath.mp.dps = 50
    rng = np.random.default_rng(1234)
    for V in range(1, 9):
        z = rng.standard_normal((6, V)) * rng.choice([0.1, 1.0, 10.0, 50.0], size=(6, 1))
        y = rng.integers(0, V, size=6)
        g = rng.standard_normal(6)
        for eps in (0.0, 0.1, 0.5):
            loss, lse, am = orc.ce_forward(z, y, eps=eps)
            dz = orc.ce_backward(z, y, g, eps=eps)
            for i in range(6):
                zi = [mpmath.mpf(float(v)) for v in z[i]]
                L = mpmath.log(mpmath.fsum(mpmath.exp(v) for v in zi))
                mean = mpmath.fsum(zi) / V
                ref_loss = (1 - eps) * (L - zi[y[i]]) + eps * (L - mean)
                assert abs(lse[i] - float(L)) <= 1e-14 * max(1.0, abs(float(L)))
                assert abs(loss[i] - float(ref_loss)) <= 1e-13 * max(1.0, abs(float(ref_loss)))
                assert am[i] == int(np.argmax(z[i]))
                for j in range(V):
                    p = mpmath.exp(zi[j] - L)
                    ref = g[i] * (p - (1 - eps) * (1 if j == y[i] else 0) - eps / V)
                    assert abs(dz[i, j] - float(ref)) <= 1e-14 * max(1.0, abs(g[i]))


def pin_torch_float64(orc):
    """PyTorch float64 cross_entropy (reduction none), label smoothing and
    ignore_index, and its autograd for sum_i g_i loss_i."""
    import torch
    rng = np.random.default_rng(7)
    N, V = 64, 50
    z = rng.standard_normal((N, V)) * 3.0
    y = rng.integers(0, V, size=N)
    y[::7] = -100
    g = rng.standard_normal(N)
    for eps in (0.0, 0.1, 0.5):
        zt = torch.tensor(z, dtype=torch.float64, requires_grad=True)
        lt = torch.nn.functional.cross_entropy(zt, torch.tensor(y), reduction="none",
                                               label_smoothing=eps, ignore_index=-100)
        (lt * torch.tensor(g)).sum().backward()
        loss, lse, _ = orc.ce_forward(z, y, eps=eps, ignore_index=-100)
        np.testing.assert_allclose(loss, lt.detach().numpy(), rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(lse, torch.logsumexp(zt, 1).detach().numpy(), rtol=1e-13)
        dz = orc.ce_backward(z, y, g, eps=eps, ignore_index=-100)
        np.testing.assert_allclose(dz, zt.grad.numpy(), rtol=1e-11, atol=1e-14)


def pin_grad_rows_sum_to_zero(orc):
    """sum_j (p_j - (1-eps)[j=y] - eps/V) = 0; ignored rows are all zero."""
    rng = np.random.default_rng(3)
    z = rng.standard_normal((40, 300)) * 4
    y = rng.integers(0, 300, size=40)
    y[5] = -100
    for eps in (0.0, 0.25):
        dz = orc.ce_backward(z, y, rng.standard_normal(40), eps=eps)
        assert np.abs(dz.sum(1)).max() < 1e-13
        assert (dz[5] == 0).all()


def pin_finite_differences(orc):
    """Central differences of sum_i g_i loss_i match the VJP (V <= 16)."""
    rng = np.random.default_rng(11)
    N, V, h = 3, 7, 1e-6
    z = rng.standard_normal((N, V))
    y = rng.integers(0, V, size=N)
    g = rng.standard_normal(N)
    for eps in (0.0, 0.3):
        dz = orc.ce_backward(z, y, g, eps=eps)
        fd = np.zeros_like(z)
        for i in range(N):
            for j in range(V):
                zp = z.copy(); zp[i, j] += h
                zm = z.copy(); zm[i, j] -= h
                lp = orc.ce_forward(zp, y, eps=eps)[0] @ g
                lm = orc.ce_forward(zm, y, eps=eps)[0] @ g
                fd[i, j] = (lp - lm) / (2 * h)
        np.testing.assert_allclose(dz, fd, rtol=0, atol=2e-8)


def pin_neg_inf(orc):
    """-inf entries: drop out of the sum at eps=0; make the loss +inf with eps>0
    or as the target; an all -inf row has lse -inf and NaN loss and grad."""
    z = np.array([[1.0, -np.inf, 0.5, 2.0]])
    zr = np.array([[1.0, 0.5, 2.0]])
    l, lse, am = orc.ce_forward(z, np.array([3]))
    lr, lser, _ = orc.ce_forward(zr, np.array([2]))
    np.testing.assert_allclose(l, lr, rtol=1e-15)
    np.testing.assert_allclose(lse, lser, rtol=1e-15)
    assert am[0] == 3
    dz = orc.ce_backward(z, np.array([3]), 1.0)
    dzr = orc.ce_backward(zr, np.array([2]), 1.0)
    assert dz[0, 1] == 0.0
    np.testing.assert_allclose(dz[0, [0, 2, 3]], dzr[0], rtol=1e-15)
    # eps > 0: the mean logit is -inf
    l, _, _ = orc.ce_forward(z, np.array([3]), eps=0.1)
    assert l[0] == np.inf
    dz = orc.ce_backward(z, np.array([3]), 1.0, eps=0.1)
    assert dz[0, 1] == -0.1 / 4
    # target at -inf
    l, _, _ = orc.ce_forward(z, np.array([1]))
    assert l[0] == np.inf
    # every entry -inf
    zi = np.full((1, 3), -np.inf)
    l, lse, _ = orc.ce_forward(zi, np.array([0]))
    assert np.isnan(l[0]) and lse[0] == -np.inf
    assert np.isnan(orc.ce_backward(zi, np.array([0]), 1.0)).all()


def pin_nan_and_argmax(orc):
    """NaN rows give NaN loss/lse and argmax at the first NaN; ties resolve to
    the lowest index (numpy's first-occurrence argmax)."""
    z = np.array([[0.0, np.nan, 5.0, np.nan], [1.0, 3.0, 3.0, -2.0]])
    l, lse, am = orc.ce_forward(z, np.array([0, 0]))
    assert np.isnan(l[0]) and np.isnan(lse[0]) and am[0] == 1
    assert am[1] == 1
    rng = np.random.default_rng(5)
    zz = rng.integers(-3, 3, size=(200, 17)).astype(np.float64)  # many ties
    _, _, am = orc.ce_forward(zz, np.zeros(200, np.int64))
    np.testing.assert_array_equal(am, np.argmax(zz, axis=1))


def pin_ignore_and_bad_targets(orc):
    """ignore_index rows: loss 0, lse still the row's log-sum-exp, zero grad.
    Targets outside [0, V): NaN loss and NaN grad row."""
    rng = np.random.default_rng(9)
    z = rng.standard_normal((4, 10))
    y = np.array([-100, 3, 10, -1])
    loss, lse, _ = orc.ce_forward(z, y, ignore_index=-100)
    assert loss[0] == 0.0
    np.testing.assert_allclose(lse, np.log(np.exp(z).sum(1)), rtol=1e-14)
    assert np.isfinite(loss[1]) and np.isnan(loss[2]) and np.isnan(loss[3])
    dz = orc.ce_backward(z, y, 1.0, ignore_index=-100)
    assert (dz[0] == 0).all() and np.isfinite(dz[1]).all()
    assert np.isnan(dz[2]).all() and np.isnan(dz[3]).all()
    # a different ignore_index value is honoured; -100 is then out of range
    loss, _, _ = orc.ce_forward(z, np.array([7, 3, 7, 7]), ignore_index=7)
    assert loss[0] == 0.0 and loss[2] == 0.0 and np.isfinite(loss[1])


def pin_offset_invariance(orc):
    """loss(z + c) = loss(z) for random rows and shared offsets up to 1e8."""
    rng = np.random.default_rng(21)
    z = rng.standard_normal((16, 64)) * 2
    y = rng.integers(0, 64, size=16)
    for eps in (0.0, 0.1):
        base, _, _ = orc.ce_forward(z, y, eps=eps)
        gbase = orc.ce_backward(z, y, 1.0, eps=eps)
        for c in (1e4, 1e6, 1e8, -1e8):
            l, lse, _ = orc.ce_forward(z + c, y, eps=eps)
            # z + c rounds z to the ulp of c in double (1.5e-8 at 1e8)
            np.testing.assert_allclose(l, base, rtol=0, atol=1e-6)
            np.testing.assert_allclose(orc.ce_backward(z + c, y, 1.0, eps=eps), gbase,
                                       rtol=0, atol=1e-7)


def pin_linear_vs_numpy(orc):
    """Fused-linear oracle = row oracle on numpy's float64 Z = H W^T; its dH,
    dW = numpy's G W and G^T H with G from the row VJP."""
    rng = np.random.default_rng(17)
    N, V, D = 24, 37, 19
    H = rng.standard_normal((N, D)).astype(np.float32)
    W = (rng.standard_normal((V, D)) * 0.3).astype(np.float32)
    y = rng.integers(0, V, size=N)
    y[4] = -100
    g = rng.standard_normal(N)
    for eps in (0.0, 0.1):
        Z = H.astype(np.float64) @ W.astype(np.float64).T
        lz, lsez, _ = orc.ce_forward(Z, y, eps=eps)
        lf, lsef = orc.linear_ce_forward_rows(H, W, y, eps=eps)
        np.testing.assert_allclose(lf, lz, rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(lsef, lsez, rtol=1e-13)
        G = orc.ce_backward(Z, y, g, eps=eps)
        dH, dW, G2 = orc.linear_ce_backward(H, W, y, g, eps=eps)
        np.testing.assert_allclose(G2, G, rtol=1e-12, atol=1e-15)
        np.testing.assert_allclose(dH, G @ W.astype(np.float64), rtol=1e-11, atol=1e-14)
        np.testing.assert_allclose(dW, G.T @ H.astype(np.float64), rtol=1e-11, atol=1e-14)
        rows = np.array([0, 4, 23, 9])
        dHr = orc.linear_ce_dh_rows(H, W, y, g, rows, eps=eps)
        np.testing.assert_allclose(dHr, dH[rows], rtol=1e-12, atol=1e-15)
        # dW rows from single columns of Z, given numpy's lse of every row
        cols = np.array([0, int(y[0]), 36, 17, int(y[5])])
        dWr = orc.linear_ce_dw_rows(H, W, y, g, cols, lsez, eps=eps)
        np.testing.assert_allclose(dWr, (G.T @ H.astype(np.float64))[cols], rtol=1e-11,
                                   atol=1e-14)
        # the chunked float64 lse of every row: numpy's lse over the whole Z
        np.testing.assert_allclose(orc.linear_lse_all(H, W, chunk=8), lsez, rtol=1e-14)
        lr, _ = orc.linear_ce_forward_rows(H, W, y, rows=rows, eps=eps)
        np.testing.assert_allclose(lr, lf[rows], rtol=1e-15)


def pin_linear_finite_differences(orc):
    """Central differences of sum_i g_i loss_i with respect to H and W. Inputs
    are multiples of 1/64 and the step is 2^-12, so every perturbed value is
    exact in float32."""
    rng = np.random.default_rng(23)
    N, V, D = 3, 5, 4
    H = (rng.integers(-64, 64, size=(N, D)) / 64.0).astype(np.float32)
    W = (rng.integers(-64, 64, size=(V, D)) / 64.0).astype(np.float32)
    y = rng.integers(0, V, size=N)
    g = rng.standard_normal(N)
    h = 2.0 ** -12
    for eps in (0.0, 0.2):
        dH, dW, _ = orc.linear_ce_backward(H, W, y, g, eps=eps)

        def f(Hx, Wx):
            return orc.linear_ce_forward_rows(Hx, Wx, y, eps=eps)[0] @ g

        for (A, dA, which) in ((H, dH, 0), (W, dW, 1)):
            fd = np.zeros(A.shape)
            for idx in np.ndindex(A.shape):
                Ap = A.copy(); Ap[idx] += h
                Am = A.copy(); Am[idx] -= h
                fp = f(Ap, W) if which == 0 else f(H, Ap)
                fm = f(Am, W) if which == 0 else f(H, Am)
                fd[idx] = (fp - fm) / (2 * h)
            np.testing.assert_allclose(dA, fd, rtol=0, atol=5e-7)
        # the dW rows of single Z columns against the same differences
        _, lse = orc.linear_ce_forward_rows(H, W, y, eps=eps)
        cols = np.arange(V)
        np.testing.assert_allclose(orc.linear_ce_dw_rows(H, W, y, g, cols, lse, eps=eps), dW,
                                   rtol=0, atol=1e-12)


# ---- probability (soft) targets ---------------------------------------------------
def _soft_draw(rng, N, V, normalised=True):
    z = rng.standard_normal((N, V))
    t = rng.random((N, V))
    if normalised:
        t /= t.sum(1, keepdims=True)
    return z, t


def pin_soft_onehot_matches_hard(orc):
    """A one-hot target distribution is the hard target: same loss, lse and
    gradient, with and without label smoothing."""
    rng = np.random.default_rng(31)
    N, V = 9, 13
    z = rng.standard_normal((N, V)) * 3
    y = rng.integers(0, V, size=N)
    t = np.zeros((N, V))
    t[np.arange(N), y] = 1.0
    g = rng.standard_normal(N)
    for eps in (0.0, 0.3):
        ls, lses = orc.ce_soft_forward(z, t, eps)
        lh, lseh, _ = orc.ce_forward(z, y, eps)
        np.testing.assert_allclose(ls, lh, rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(lses, lseh, rtol=1e-15)
        np.testing.assert_allclose(orc.ce_soft_backward(z, t, g, eps), orc.ce_backward(z, y, g, eps),
                                   rtol=1e-12, atol=1e-15)


def pin_soft_torch_float64(orc):
    """PyTorch's float64 cross_entropy with probability targets (and its
    label smoothing, which mixes the targets with the uniform distribution),
    and its autograd, as an independent library special case; targets need
    not sum to 1."""
    torch = __import__("torch")
    import torch.nn.functional as F
    rng = np.random.default_rng(32)
    for normalised in (True, False):
        z, t = _soft_draw(rng, 7, 11, normalised)
        g = rng.standard_normal(7)
        for eps in (0.0, 0.25):
            zt = torch.tensor(z, dtype=torch.float64, requires_grad=True)
            ref = F.cross_entropy(zt, torch.tensor(t), reduction="none", label_smoothing=eps)
            (ref * torch.tensor(g)).sum().backward()
            loss, _ = orc.ce_soft_forward(z, t, eps)
            np.testing.assert_allclose(loss, ref.detach().numpy(), rtol=1e-12, atol=1e-14)
            np.testing.assert_allclose(orc.ce_soft_backward(z, t, g, eps), zt.grad.numpy(),
                                       rtol=1e-11, atol=1e-14)


def pin_soft_closed_forms(orc):
    """Equal logits against any distribution: loss = log V (t sums to 1).
    Two logits [x, 0] against [1, 0]: log(1 + e^-x); against [a, 1-a] on
    equal logits: log 2. Uniform targets with eps keep the loss."""
    V = 10
    t = np.random.default_rng(33).random((1, V)); t /= t.sum()
    for c in (0.0, 1e4, 1e8):
        loss, lse = orc.ce_soft_forward(np.full((1, V), c), t)
        assert abs(loss[0] - math.log(V)) <= 1e-12 * math.log(V)
        assert abs(lse[0] - (c + math.log(V))) <= 1e-15 * max(1.0, abs(c))
    for x in (0.5, 3.0, -2.0):
        loss, _ = orc.ce_soft_forward(np.array([[x, 0.0]]), np.array([[1.0, 0.0]]))
        assert abs(loss[0] - math.log1p(math.exp(-x))) <= 1e-15
    loss, _ = orc.ce_soft_forward(np.array([[5.0, 5.0]]), np.array([[0.3, 0.7]]))
    assert abs(loss[0] - math.log(2.0)) <= 1e-15
    z = np.array([[1.0, -2.0, 0.5, 3.0]])
    u = np.full((1, 4), 0.25)
    assert abs(orc.ce_soft_forward(z, u, 0.4)[0][0] - orc.ce_soft_forward(z, u, 0.0)[0][0]) <= 1e-15


def pin_soft_grad_rows_sum_to_zero_and_shift(orc):
    """Each gradient row sums to g (T' - T') = 0; shifting a row by c leaves
    the loss unchanged for any targets (inputs on a 1/64 grid, so the shift
    is exact)."""
    rng = np.random.default_rng(34)
    z = rng.integers(-256, 256, size=(6, 17)) / 64.0
    t = rng.random((6, 17)) * 2 - 0.5
    g = rng.standard_normal(6)
    for eps in (0.0, 0.1):
        dz = orc.ce_soft_backward(z, t, g, eps)
        assert np.abs(dz.sum(1)).max() <= 1e-13 * (np.abs(dz).max() + 1)
        l0, _ = orc.ce_soft_forward(z, t, eps)
        l1, _ = orc.ce_soft_forward(z + 1024.0, t, eps)
        np.testing.assert_allclose(l1, l0, rtol=1e-12, atol=1e-12)


def pin_soft_finite_differences(orc):
    """Central differences of sum_i g_i loss_i with respect to z."""
    rng = np.random.default_rng(35)
    z, t = _soft_draw(rng, 3, 6, normalised=False)
    g = rng.standard_normal(3)
    h = 1e-6
    for eps in (0.0, 0.2):
        dz = orc.ce_soft_backward(z, t, g, eps)
        fd = np.zeros_like(z)
        for idx in np.ndindex(z.shape):
            zp = z.copy(); zp[idx] += h
            zm = z.copy(); zm[idx] -= h
            fd[idx] = (orc.ce_soft_forward(zp, t, eps)[0] @ g - orc.ce_soft_forward(zm, t, eps)[0] @ g) / (2 * h)
        np.testing.assert_allclose(dz, fd, rtol=0, atol=1e-8)


def pin_soft_nonfinite(orc):
    """A -inf logit with zero target mass contributes nothing (0 log 0 = 0);
    with target mass the loss is +inf; NaN rows and all -inf rows give NaN
    losses and NaN gradient rows, with lse NaN and -inf."""
    z = np.array([[1.0, -np.inf, 0.5], [1.0, -np.inf, 0.5], [1.0, np.nan, 0.5],
                  [-np.inf, -np.inf, -np.inf]])
    t = np.array([[0.5, 0.0, 0.5], [0.5, 0.25, 0.25], [0.3, 0.3, 0.4], [0.2, 0.3, 0.5]])
    loss, lse = orc.ce_soft_forward(z, t)
    ref0 = 0.5 * (math.log(math.e + math.exp(0.5)) - 1.0) + 0.5 * (math.log(math.e + math.exp(0.5)) - 0.5)
    assert abs(loss[0] - ref0) <= 1e-15
    assert loss[1] == math.inf
    assert math.isnan(loss[2]) and math.isnan(lse[2])
    assert math.isnan(loss[3]) and lse[3] == -math.inf
    dz = orc.ce_soft_backward(z, t, 1.0)
    assert np.isfinite(dz[:2]).all() and dz[0, 1] == 0.0
    assert np.isnan(dz[2:]).all()


# ---- KL divergence of a student from a teacher ("One barrier short") ----------------
def pin_kl_torch_float64(orc):
    """PyTorch float64 kl_div on log-softmaxes (log_target) and its autograd
    with respect to the student logits, as an independent library case."""
    torch = __import__("torch")
    import torch.nn.functional as F
    rng = np.random.default_rng(41)
    zq = rng.standard_normal((6, 13)) * 4
    zp = rng.standard_normal((6, 13)) * 4
    g = rng.standard_normal(6)
    qt = torch.tensor(zq, requires_grad=True)
    ref = F.kl_div(F.log_softmax(qt, -1), F.log_softmax(torch.tensor(zp), -1), reduction="none",
                   log_target=True).sum(-1)
    (ref * torch.tensor(g)).sum().backward()
    loss, _, _ = orc.kl_forward(zq, zp)
    np.testing.assert_allclose(loss, ref.detach().numpy(), rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(orc.kl_backward(zq, zp, g), qt.grad.numpy(), rtol=1e-11, atol=1e-14)


def pin_kl_closed_forms(orc):
    """Identical distributions: 0 and a zero gradient. Two classes:
    a log(a/b) + (1-a) log((1-a)/(1-b)). Shifting either row by a constant
    changes nothing; the loss is never negative (Gibbs)."""
    rng = np.random.default_rng(42)
    z = rng.standard_normal((4, 9))
    loss, _, _ = orc.kl_forward(z, z)
    assert np.abs(loss).max() <= 1e-15
    assert np.abs(orc.kl_backward(z, z, 1.0)).max() == 0.0
    for (x, y) in ((0.7, -1.2), (3.0, 0.0), (-2.0, 2.5)):
        a = 1.0 / (1.0 + math.exp(-x))     # teacher p = softmax([x, 0])
        b = 1.0 / (1.0 + math.exp(-y))     # student q = softmax([y, 0])
        ref = a * math.log(a / b) + (1 - a) * math.log((1 - a) / (1 - b))
        loss, _, _ = orc.kl_forward(np.array([[y, 0.0]]), np.array([[x, 0.0]]))
        assert abs(loss[0] - ref) <= 1e-14 * max(1.0, ref)
    zq = rng.integers(-256, 256, size=(5, 11)) / 64.0
    zp = rng.integers(-256, 256, size=(5, 11)) / 64.0
    l0, lq0, lp0 = orc.kl_forward(zq, zp)
    l1, lq1, lp1 = orc.kl_forward(zq + 512.0, zp - 256.0)
    np.testing.assert_allclose(l1, l0, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(lq1 - lq0, 512.0, rtol=1e-15)
    np.testing.assert_allclose(lp1 - lp0, -256.0, rtol=1e-15)
    assert (l0 >= 0).all()


def pin_kl_grad_and_finite_differences(orc):
    """Gradient rows sum to 0; central differences of sum_i g_i loss_i with
    respect to the student logits."""
    rng = np.random.default_rng(43)
    zq = rng.standard_normal((3, 7)) * 2
    zp = rng.standard_normal((3, 7)) * 2
    g = rng.standard_normal(3)
    d = orc.kl_backward(zq, zp, g)
    assert np.abs(d.sum(1)).max() <= 1e-15
    h = 1e-6
    fd = np.zeros_like(zq)
    for idx in np.ndindex(zq.shape):
        a = zq.copy(); a[idx] += h
        b = zq.copy(); b[idx] -= h
        fd[idx] = (orc.kl_forward(a, zp)[0] @ g - orc.kl_forward(b, zp)[0] @ g) / (2 * h)
    np.testing.assert_allclose(d, fd, rtol=0, atol=1e-8)


def pin_kl_nonfinite(orc):
    """Teacher -inf (p_j = 0) adds nothing, even over a student -inf; a
    student -inf under teacher mass is +inf; NaN and all -inf rows give NaN."""
    zq = np.array([[1.0, -np.inf, 0.5], [1.0, -np.inf, 0.5], [1.0, np.nan, 0.5], [0.0, 1.0, 2.0]])
    zp = np.array([[0.5, -np.inf, 1.0], [0.5, 0.0, 1.0], [0.2, 0.3, 0.4], [-np.inf] * 3])
    loss, lq, lp = orc.kl_forward(zq, zp)
    lp0 = math.log(math.exp(0.5) + math.e)
    lq0 = math.log(math.e + math.exp(0.5))
    ref0 = (math.exp(0.5 - lp0) * ((0.5 - lp0) - (1.0 - lq0)) +
            math.exp(1.0 - lp0) * ((1.0 - lp0) - (0.5 - lq0)))
    assert abs(loss[0] - ref0) <= 1e-15
    assert loss[1] == math.inf
    assert math.isnan(loss[2]) and math.isnan(lq[2])
    assert math.isnan(loss[3]) and lp[3] == -math.inf
    d = orc.kl_backward(zq, zp, 1.0)
    assert np.isfinite(d[:2]).all() and np.isnan(d[2:]).all()


# Ordered: cheap first. The planted-mistake test runs every entry.
BATTERY = [
    pin_pr4188_printed_values,
    pin_equal_logits_closed_form,
    pin_two_logit_offset_closed_form,
    pin_uniform_rows_closed_form,
    pin_grad_rows_sum_to_zero,
    pin_neg_inf,
    pin_nan_and_argmax,
    pin_ignore_and_bad_targets,
    pin_offset_invariance,
    pin_bruteforce_mpmath,
    pin_torch_float64,
    pin_finite_differences,
    pin_linear_vs_numpy,
    pin_linear_finite_differences,
    pin_soft_onehot_matches_hard,
    pin_soft_closed_forms,
    pin_soft_grad_rows_sum_to_zero_and_shift,
    pin_soft_nonfinite,
    pin_soft_torch_float64,
    pin_soft_finite_differences,
    pin_kl_closed_forms,
    pin_kl_nonfinite,
    pin_kl_torch_float64,
    pin_kl_grad_and_finite_differences,
]
