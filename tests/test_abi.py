"""C ABI checks that need no GPU: the library loads, exports every function
the header declares, and rejects bad arguments on the host before any launch."""
import ctypes
import os
import re

import pytest

import softmax_cross_entropy_lse_b200 as ce
from softmax_cross_entropy_lse_b200 import ce_layout

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_functions():
    names = set()
    for h in os.listdir(os.path.join(ROOT, "include")):
        if not h.endswith(".h"):
            continue
        text = open(os.path.join(ROOT, "include", h)).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        for m in re.finditer(r"^\s*(?:const\s+)?[a-z_0-9]+\s*\*?\s+([a-z_0-9]+)\s*\(", text, re.M):
            names.add(m.group(1))
    return sorted(names)


@pytest.fixture(scope="module")
def L():
    from softmax_cross_entropy_lse_b200 import build
    build.build()
    return ce.lib()


def test_every_declared_symbol_is_exported(L):
    names = header_functions()
    assert len(names) >= 9, names
    for n in names:
        assert hasattr(L, n), f"{n} declared in include/ but not exported"
    assert sorted(ce.EXPORTED) == names


def test_status_strings(L):
    for s in range(8):
        assert L.ce_status_string(s)
    assert L.ce_status_string(99) == b"unknown status"
    assert b"bounded wait" in L.ce_status_string(7)


def test_wait_hook_validates_and_resets(L):
    """The testing hook of the bounded waits takes starve 0 or 1 only; the
    settings are host state, so this needs no GPU."""
    assert L.ce_testing_set_wait(0, 2) == 1
    assert L.ce_testing_set_wait(0, -1) == 1
    assert L.ce_testing_set_wait(10_000_000, 1) == 0
    assert L.ce_testing_set_wait(0, 0) == 0


def lay(N, ld, s_col=1):
    return ce_layout(N, 0, ld, s_col)


# Fake, never-dereferenced addresses: validation must reject these calls on
# the host, so nothing reaches the device.
Z = 0x10000000
T = 0x20000000
OUT = 0x30000000


def fwd(L, z=Z, dt=0, lg=None, N=8, V=16, t=T, tdt=0, tg=None, eps=0.0, ign=-100,
        loss=OUT, lse=OUT + 4096, lse_lo=None, am=None, ws=None, ws_bytes=0):
    lg = lg or lay(N, V)
    tg = tg or ce_layout(N, 0, 1, 0)
    return L.ce_forward(z, dt, lg, N, V, t, tdt, tg, eps, ign, loss, lse, lse_lo, am, ws,
                        ws_bytes, None)


def test_forward_rejects_bad_arguments(L):
    assert fwd(L, N=-1) == 1
    assert fwd(L, V=0) == 1
    assert fwd(L, V=2**31) == 1
    assert fwd(L, dt=7) == 1
    assert fwd(L, tdt=5) == 1
    assert fwd(L, eps=-0.1) == 1
    assert fwd(L, eps=1.5) == 1
    assert fwd(L, eps=float("nan")) == 1
    assert fwd(L, z=None) == 1
    assert fwd(L, t=None) == 1
    assert fwd(L, loss=None) == 1
    assert fwd(L, lse=None) == 1
    assert fwd(L, lg=ce_layout(0, 0, 16, 1)) == 1
    # N = 0 is a no-op that succeeds without touching the device
    assert fwd(L, N=0, z=None, t=None, loss=None, lse=None) == 0


def test_forward_rejects_aliasing(L):
    # loss overlapping the logits
    assert fwd(L, loss=Z + 64) == 2
    # lse overlapping loss
    assert fwd(L, lse=OUT + 16) == 2
    # argmax overlapping the targets
    assert fwd(L, am=T) == 2
    # lse_lo overlapping lse
    assert fwd(L, lse_lo=OUT + 4096 + 4) == 2


def test_forward_rejects_short_workspace(L):
    # few long rows: the plan splits the vocabulary and needs a workspace
    N, V = 4, 1 << 20
    need = L.ce_workspace_size(N, V, 0, 148)
    assert need > 0
    big = ce_layout(N, 0, V, 1)
    assert fwd(L, N=N, V=V, lg=big, loss=0x90000000, lse=0x90001000) == 3
    assert fwd(L, N=N, V=V, lg=big, loss=0x90000000, lse=0x90001000, ws=0xA0000000,
               ws_bytes=need - 1) == 3
    # misaligned workspace
    assert fwd(L, N=N, V=V, lg=big, loss=0x90000000, lse=0x90001000, ws=0xA0000004,
               ws_bytes=need + 64) == 3


def test_workspace_sizes(L):
    # short rows never split
    assert L.ce_workspace_size(1 << 20, 128, 0, 148) == 0
    assert L.ce_workspace_size(4096, 1024, 0, 148) == 0
    # plenty of long rows (several full waves of CTAs): no split
    assert L.ce_workspace_size(8192, 32000, 1, 148) == 0
    assert L.ce_workspace_size(2048, 151936, 1, 148) == 0
    # few very long rows split, 16 bytes per partial
    ws = L.ce_workspace_size(64, 151936, 1, 148)
    assert ws % (16 * 64) == 0 and ws >= 2 * 16 * 64
    assert L.ce_workspace_size(0, 100, 0, 148) == 0
    assert L.ce_workspace_size(10, 100, 9, 148) == 0


def bwd(L, g=OUT, gs=1, z=Z, dt=0, lg=None, N=8, V=16, t=T, tdt=0, tg=None, lse=OUT + 4096,
        lse_lo=None, eps=0.0, ign=-100, dz=0x40000000, ddt=0, dl=None):
    lg = lg or lay(N, V)
    tg = tg or ce_layout(N, 0, 1, 0)
    dl = dl or lay(N, V)
    return L.ce_backward(g, gs, z, dt, lg, N, V, t, tdt, tg, lse, lse_lo, eps, ign, dz, ddt, dl,
                         None)


def test_backward_rejects_bad_arguments(L):
    assert bwd(L, N=-1) == 1
    assert bwd(L, V=0) == 1
    assert bwd(L, dt=3) == 1
    assert bwd(L, dt=0, ddt=1) == 6  # fp32 logits into bf16 dlogits: not provided
    assert bwd(L, g=None) == 1
    assert bwd(L, lse=None) == 1
    assert bwd(L, dz=None) == 1
    assert bwd(L, eps=2.0) == 1


def test_backward_aliasing_rules(L):
    # dlogits overlapping logits but not identical: rejected (the VJP bug of
    # MLX issue #4686 came from an output aliasing a temporary copy)
    assert bwd(L, dz=Z + 4) == 2
    assert bwd(L, dz=Z, dl=lay(8, 32)) == 2
    assert bwd(L, dz=Z, ddt=0, dt=1) == 6 or bwd(L, dz=Z, ddt=0, dt=1) == 2
    # dlogits over lse / grad / targets
    assert bwd(L, dz=OUT + 4096) == 2
    assert bwd(L, dz=T) == 2
    assert bwd(L, dz=OUT) == 2


def test_linear_entry_points_exist(L):
    assert L.linear_ce_workspace_size(8, 16, 64, 148) >= 0
    assert L.linear_ce_backward_workspace_size(8, 16, 64, 148) >= 0


def test_linear_backward_workspace_is_one_vocabulary_chunk(L):
    """The backward holds one 8192-column chunk of the logits' gradient (bf16,
    row-major) and the float dH accumulator, nothing transposed, so its
    workspace does not grow with V past one chunk."""
    N, V, D = 8192, 151936, 4096
    chunk = 8192
    want = N * chunk * 2 + N * D * 4
    assert L.linear_ce_backward_workspace_size(N, V, D, 148) == want == 268435456
    for v in (chunk, chunk + 1, 4 * V):
        assert L.linear_ce_backward_workspace_size(N, v, D, 148) == want
    # one chunk rounded up to the 256-column GEMM tile when V is smaller
    small = L.linear_ce_backward_workspace_size(512, 1000, 128, 148)
    assert small == 512 * 1024 * 2 + 512 * 128 * 4


def test_row_layout_marshalling():
    torch = pytest.importorskip("torch")
    x = torch.empty(10, 119, 64)
    N, lg = ce.row_layout(x[:, :-1], True)
    assert N == 1180 and (lg.inner, lg.s_outer, lg.s_inner, lg.s_col) == (118, 119 * 64, 64, 1)
    t = torch.empty(10, 119, dtype=torch.int32)
    N, tg = ce.row_layout(t[:, 1:], False)
    assert N == 1180 and (tg.inner, tg.s_outer, tg.s_inner) == (118, 119, 1)
    N, lg = ce.row_layout(x, True)  # contiguous 3-D merges to one level
    assert N == 1190 and lg.inner == 1190 and lg.s_inner == 64
    N, lg = ce.row_layout(x.view(1190, 64).t(), True)  # columns strided
    assert N == 64 and lg.s_inner == 1 and lg.s_col == 64
    with pytest.raises(ValueError):
        ce.row_layout(torch.empty(4, 5, 6, 7)[:, :-1, :-1], True)


def test_out_tensors_validated():
    """ce_forward(out=...) checks the caller's tensors before any launch."""
    import torch
    import softmax_cross_entropy_lse_b200 as ce
    good = ce.ForwardResult(*(torch.empty(5) for _ in range(3)), None)
    assert ce._row_outputs(5, torch.device("cpu"), False, good)[0] is good.loss
    for bad in (ce.ForwardResult(torch.empty(4), torch.empty(5), torch.empty(5), None),
                ce.ForwardResult(torch.empty(5, dtype=torch.float64), torch.empty(5), torch.empty(5), None),
                ce.ForwardResult(torch.empty(10)[::2], torch.empty(5), torch.empty(5), None)):
        with pytest.raises(ValueError):
            ce._row_outputs(5, torch.device("cpu"), False, bad)
    with pytest.raises(ValueError):
        ce._row_outputs(5, torch.device("cpu"), True, good)  # argmax requested, none given


def soft_fwd(L, z=Z, dt=0, N=8, V=16, t=T, tdt=0, tl=None, eps=0.0, loss=OUT, lse=OUT + 4096,
             lse_lo=None, tsum=None):
    tl = tl or lay(N, V)
    return L.ce_soft_forward(z, dt, lay(N, V), N, V, t, tdt, tl, eps, loss, lse, lse_lo, tsum, None)


def soft_bwd(L, g=OUT + 8192, z=Z, dt=0, N=8, V=16, t=T, tdt=0, lse=OUT, tsum=None, eps=0.0,
             dz=0x40000000, ddt=0):
    return L.ce_soft_backward(g, 0, z, dt, lay(N, V), N, V, t, tdt, lay(N, V), lse, None, tsum, eps,
                              dz, ddt, lay(N, V), None)


def test_soft_targets_reject_bad_arguments_and_aliasing(L):
    assert soft_fwd(L, N=-1) == 1
    assert soft_fwd(L, eps=2.0) == 1
    assert soft_fwd(L, t=None) == 1
    assert soft_fwd(L, dt=1, tdt=2) == 6      # f16 targets for bf16 logits: not supported
    assert soft_fwd(L, dt=0, tdt=1) == 6      # bf16 targets for f32 logits: not supported
    assert soft_fwd(L, N=0, z=None, t=None, loss=None, lse=None) == 0
    assert soft_fwd(L, loss=T + 32) == 2      # loss over the targets
    assert soft_fwd(L, tsum=OUT + 8) == 2     # target sums over loss
    assert soft_bwd(L, ddt=2) == 6            # f16 gradient of f32 logits
    assert soft_bwd(L, dz=T + 64) == 2        # gradient over the targets
    assert soft_bwd(L, dz=OUT) == 2           # gradient over lse
    assert soft_bwd(L, g=None) == 1


def test_kl_rejects_bad_arguments_and_aliasing(L):
    N, V = 8, 16

    def fwd_kl(q=Z, p=T, dt=0, loss=OUT, lq=OUT + 4096, lp=OUT + 8192, lq_lo=None, lp_lo=None, n=N):
        return L.ce_kl_forward(q, p, dt, lay(n, V), lay(n, V), n, V, loss, lq, lq_lo, lp, lp_lo, None)

    def bwd_kl(g=OUT + 16384, dq=0x40000000, ddt=0, dt=0):
        return L.ce_kl_backward(g, 0, Z, T, dt, lay(N, V), lay(N, V), N, V, OUT, None, OUT + 4096, None,
                                dq, ddt, lay(N, V), None)

    assert fwd_kl(dt=5) == 1
    assert fwd_kl(p=None) == 1
    assert fwd_kl(lp=None) == 1
    assert fwd_kl(n=0, q=None, p=None, loss=None, lq=None, lp=None) == 0
    assert fwd_kl(loss=T + 8) == 2          # loss over the teacher logits
    assert fwd_kl(lp=OUT + 4096 + 16) == 2  # teacher lse over the student lse
    assert bwd_kl(ddt=1) == 6               # bf16 gradient of f32 logits
    assert bwd_kl(dq=T) == 2                # gradient over the teacher
    assert bwd_kl(dq=OUT + 4096) == 2       # gradient over the teacher lse
    assert bwd_kl(g=None) == 1
