"""ce_forward_noalloc: the forward for callers that cannot allocate device
memory (plugins inside a host application that owns all device memory
through its own pool, loops with a memory budget fixed at start-up, C callers
without an allocator; cudaMalloc may also synchronise the device).

It runs the vocabulary-split forward with its scratch in a library-owned
static device array instead of a caller workspace. These tests call it
through the C ABI with raw pointers and compare it with ce_forward given a
workspace, on two calls in a row (the array keeps the previous call's
contents, which must not leak into the next result).

This file is collected last on purpose: if it fails, a run that stops at the
first failure has already run every other test.
"""
import numpy as np
import pytest

import softmax_cross_entropy_lse_b200 as ce
from softmax_cross_entropy_lse_b200 import ce_layout, workloads as wl


def _plain(N, V):
    return ce_layout(N, 0, V, 1)


def test_noalloc_rejects_oversized_shape_on_host():
    L = ce.lib()
    # a shape whose split scratch exceeds the fixed array: rejected before
    # any device work (fake pointers are never touched)
    N, V = 33, 1 << 20
    assert L.ce_workspace_size(N, V, ce.CE_F32, 148) > ce.NOALLOC_SCRATCH_BYTES
    st = L.ce_forward_noalloc(0x1000000, ce.CE_F32, _plain(N, V), N, V, 0x2000000, ce.CE_I32,
                              ce_layout(N, 0, 1, 0), 0.0, -100, 0x3000000, 0x4000000, None, None,
                              None)
    assert st == 3  # CE_EWORKSPACE
    assert L.ce_forward_noalloc(None, 9, _plain(4, 4), 4, 4, None, 0, ce_layout(4, 0, 1, 0), 0.0,
                                -100, None, None, None, None, None) == 1


@pytest.mark.gpu
def test_noalloc_matches_workspace_forward(orc):
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    L = ce.lib()
    dev = torch.device("cuda", 0)
    stream = torch.cuda.current_stream(dev).cuda_stream
    cases = [(37, 151936, "bf16", 0.1), (5, 1 << 20, "f32", 0.0)]
    for call, (N, V, dt, eps) in enumerate(cases * 2):
        z, z32, y = wl.rows(N, V, dt, seed=100 + call, std=2.0)
        code = ce.CE_BF16 if dt == "bf16" else ce.CE_F32
        need = L.ce_workspace_size(N, V, code, 0)
        assert 0 < need <= ce.NOALLOC_SCRATCH_BYTES  # the split path, with scratch
        if dt == "bf16":
            zt = torch.from_numpy(z.view(np.int16)).to(dev)
        else:
            zt = torch.from_numpy(z).to(dev)
        yt = torch.from_numpy(y).to(dev)
        outs = {}
        for kind in ("noalloc", "workspace"):
            loss = torch.full((N,), float("nan"), device=dev)
            lse = torch.full((N,), float("nan"), device=dev)
            lo = torch.full((N,), float("nan"), device=dev)
            am = torch.full((N,), -7, dtype=torch.int32, device=dev)
            args = (zt.data_ptr(), code, _plain(N, V), N, V, yt.data_ptr(), ce.CE_I32,
                    ce_layout(N, 0, 1, 0), eps, -100, loss.data_ptr(), lse.data_ptr(),
                    lo.data_ptr(), am.data_ptr())
            if kind == "noalloc":
                st = L.ce_forward_noalloc(*args, stream)
            else:
                ws = torch.empty(need, dtype=torch.uint8, device=dev)
                st = L.ce_forward(*args, ws.data_ptr(), need, stream)
            assert st == 0, (kind, st)
            torch.cuda.synchronize()
            outs[kind] = (loss.cpu().numpy(), lse.cpu().numpy(), lo.cpu().numpy(),
                          am.cpu().numpy())
        a, b = outs["noalloc"], outs["workspace"]
        rt, at = (1e-5, 1e-6) if dt == "f32" else (2e-3, 1e-6)
        for x, r in zip(a[:3], b[:3]):
            assert np.all(np.abs(x - r) <= rt * np.abs(r) + at)
        np.testing.assert_array_equal(a[3], b[3])
        # the same kernels in the same order: bit-identical results
        for x, r in zip(a, b):
            np.testing.assert_array_equal(x, r)
        # and both match the oracle
        loss64, _, am64 = orc.ce_forward(z32.astype(np.float64), y, eps)
        assert np.all(np.abs(a[0] - loss64) <= rt * np.abs(loss64) + at)
        np.testing.assert_array_equal(a[3], am64)
    assert L.ce_get_error(stream) == 0
