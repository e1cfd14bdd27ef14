"""Bounded pipeline waits on the GPU: a wait that runs out ends the kernel
with an error status, and the context stays usable.

The kernels that stream their operands through mbarrier pipelines (the
tensor-core GEMM engine of the fused-linear calls, the bulk-copy ring of the
long-row forward, and the slices of the one-call forward + VJP, which also
wait on their cluster peers' states) give up a wait after a time limit, raise the timeout
bit of the device error word, let the copies and MMAs they started complete,
free their tensor memory and return. These tests make such a wait run out
without any fault: the testing hook sets a short limit and starves the
launches of their copies, so each consumer waits on a barrier that nothing
completes. Nothing asynchronous is in flight when the kernel returns.
ce_get_error must then report CE_ETIMEOUT (not a bad target), and the next
call on the same stream must give the correct result.
"""
from __future__ import annotations

import numpy as np
import pytest

from tests.gpu_util import assert_close, f32, loss_tol, torch, upload

import softmax_cross_entropy_lse_b200 as ce
from softmax_cross_entropy_lse_b200 import workloads as wl

pytestmark = pytest.mark.gpu

CE_ETIMEOUT = 7
LIMIT_NS = 50_000_000  # 50 ms: far above any wait of a correct pipeline here


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    ce.lib()
    assert ce.get_error() == 0
    yield
    ce.testing_set_wait(0, False)
    assert ce.get_error() == 0


def starved(fn):
    """Runs fn with every copy of the waiting kernels withheld; returns the
    status ce_get_error reports afterwards."""
    ce.testing_set_wait(LIMIT_NS, True)
    try:
        fn()
        return ce.get_error()
    finally:
        ce.testing_set_wait(0, False)


def bf16_dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def test_gemm_engine_wait_runs_out(orc):
    N, V, D = 256, 1500, 256
    hb, hf, wb, wf, y = wl.c5(seed=11, N=N, V=V, D=D, w_std=0.05)
    H, W, yt = bf16_dev(hb), bf16_dev(wb), torch.from_numpy(y).cuda()
    good_loss, good_lse = ce.linear_ce_forward(H, W, yt)
    assert ce.get_error() == 0
    # forward: the MMA thread's first wait for a stage runs out
    assert starved(lambda: ce.linear_ce_forward(H, W, yt)) == CE_ETIMEOUT
    loss, lse = ce.linear_ce_forward(H, W, yt)
    assert ce.get_error() == 0
    assert torch.equal(loss, good_loss) and torch.equal(lse, good_lse)
    ref_loss, ref_lse = orc.linear_ce_forward_rows(hf, wf, y)
    assert_close(f32(loss), ref_loss, 5e-3, 0.0, "loss after a timeout")
    # backward: each of its GEMMs (gradient, dW and dH epilogues) runs out too
    g = torch.full((1,), 1.0 / N, device="cuda")
    good = ce.linear_ce_backward(g, H, W, yt, lse, dH_dtype=torch.float32,
                                 dW_dtype=torch.float32)
    assert ce.get_error() == 0
    assert starved(lambda: ce.linear_ce_backward(g, H, W, yt, lse)) == CE_ETIMEOUT
    dH, dW = ce.linear_ce_backward(g, H, W, yt, lse, dH_dtype=torch.float32,
                                   dW_dtype=torch.float32)
    assert ce.get_error() == 0
    assert torch.equal(dH, good[0]) and torch.equal(dW, good[1])


def test_bulk_copy_ring_wait_runs_out(orc):
    """bf16 rows of 32000 classes take the long-row forward with per-warp
    bulk-copy rings."""
    z, z32, y = wl.rows(300, 32000, "bf16", seed=12, std=2.0)
    zt, yt = upload(z, "bf16"), upload(y)
    good = ce.ce_forward(zt, yt)
    assert ce.get_error() == 0
    assert starved(lambda: ce.ce_forward(zt, yt)) == CE_ETIMEOUT
    r = ce.ce_forward(zt, yt)
    assert ce.get_error() == 0
    assert torch.equal(r.loss, good.loss) and torch.equal(r.lse, good.lse)
    loss, lse, _ = orc.ce_forward(z32.astype(np.float64), y)
    rt, at = loss_tol("bf16")
    assert_close(f32(r.loss), loss, rt, at, "loss after a timeout")
    assert_close(f32(r.lse), lse, rt, at, "lse after a timeout")


@pytest.mark.parametrize("N,V", [(600, 32000), (160, 151936)])
def test_fused_slices_wait_runs_out(orc, N, V):
    """The one-call forward + VJP of long rows: 32000-wide rows wait for their
    bulk copies into shared memory, 151,936-wide rows (L2 slices over a 4-CTA
    cluster) for the states their peers push; starved, both waits run out."""
    z, z32, y = wl.rows(N, V, "bf16", seed=14, std=2.0)
    zt, yt = upload(z, "bf16"), upload(y)
    g = torch.ones(1, device="cuda")
    good_r, good_dz = ce.ce_forward_backward(zt, yt, g)
    assert ce.get_error() == 0
    assert starved(lambda: ce.ce_forward_backward(zt, yt, g)) == CE_ETIMEOUT
    r, dz = ce.ce_forward_backward(zt, yt, g)
    assert ce.get_error() == 0
    assert torch.equal(r.loss, good_r.loss) and torch.equal(r.lse, good_r.lse)
    assert torch.equal(dz, good_dz)
    loss, lse, _ = orc.ce_forward(z32.astype(np.float64), y)
    rt, at = loss_tol("bf16")
    assert_close(f32(r.loss), loss, rt, at, "loss after a timeout")


def test_timeout_outranks_bad_target():
    """A launch that both saw a bad target and gave up a wait reports the
    timeout: its outputs are not valid at all."""
    z, _, y = wl.rows(64, 32000, "bf16", seed=13, std=2.0)
    y = y.copy()
    y[5] = 32000
    zt, yt = upload(z, "bf16"), upload(y)
    ce.ce_forward(zt, yt)
    assert ce.get_error() == 5
    assert starved(lambda: ce.ce_forward(zt, yt)) == CE_ETIMEOUT
