"""Float64 CPU oracle for fused softmax cross-entropy (ctypes wrapper).

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` may import this package; the product path never
does. The arithmetic lives in ``ce_oracle.c`` (plain C, double precision,
OpenMP over independent rows); this module only marshals numpy arrays.

Every entry point returns float64 results computed from inputs widened
exactly to float64 (row oracle) or to float32-held bf16 values widened to
double inside the dot products (linear oracle).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ce_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

_f64p = ctypes.POINTER(ctypes.c_double)
_f32p = ctypes.POINTER(ctypes.c_float)
_i64p = ctypes.POINTER(ctypes.c_int64)
_i64 = ctypes.c_int64


def build(src: str = _SRC, out: str = _LIB, force: bool = False) -> str:
    """Compile the oracle with gcc (-O2, OpenMP, no fast-math)."""
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(src):
        cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
               "-Wall", "-o", out, src, "-lm"]
        subprocess.run(cmd, check=True)
    return out


class Oracle:
    """Bindings to one compiled copy of the oracle library."""

    def __init__(self, lib_path: str | None = None):
        path = lib_path or build()
        self.lib = ctypes.CDLL(path)
        L = self.lib
        L.orc_ce_forward.argtypes = [_f64p, _i64, _i64, _i64p, ctypes.c_double, _i64,
                                     _f64p, _f64p, _i64p]
        L.orc_ce_backward.argtypes = [_f64p, _i64, _i64, _i64p, _f64p, ctypes.c_double,
                                      _i64, _f64p]
        L.orc_linear_ce_forward_rows.argtypes = [_f32p, _f32p, _i64, _i64, _i64p, _i64,
                                                 _i64p, ctypes.c_double, _i64, _f64p, _f64p]
        L.orc_linear_ce_dh_rows.argtypes = [_f32p, _f32p, _i64, _i64, _i64p, _i64, _i64p,
                                            _f64p, ctypes.c_double, _i64, _f64p]
        L.orc_linear_ce_dw_rows.argtypes = [_f32p, _f32p, _i64, _i64, _i64, _i64p, _i64, _i64p,
                                            _f64p, _f64p, ctypes.c_double, _i64, _f64p]
        L.orc_linear_ce_backward.argtypes = [_f32p, _f32p, _i64, _i64, _i64, _i64p, _f64p,
                                             ctypes.c_double, _i64, _f64p, _f64p, _f64p]
        L.orc_ce_soft_forward.argtypes = [_f64p, _f64p, _i64, _i64, ctypes.c_double, _f64p, _f64p]
        L.orc_ce_soft_backward.argtypes = [_f64p, _f64p, _i64, _i64, _f64p, ctypes.c_double, _f64p]
        L.orc_kl_forward.argtypes = [_f64p, _f64p, _i64, _i64, _f64p, _f64p, _f64p]
        L.orc_kl_backward.argtypes = [_f64p, _f64p, _i64, _i64, _f64p, _f64p]
        L.orc_num_threads.restype = ctypes.c_int

    # -- helpers -----------------------------------------------------------
    @staticmethod
    def _p(a, t):
        return a.ctypes.data_as(t)

    # -- row cross-entropy -------------------------------------------------
    def ce_forward(self, z, y, eps: float = 0.0, ignore_index: int = -100):
        """loss, lse (float64, N) and argmax (int64, N) of each row of z (N, V)."""
        z = np.ascontiguousarray(z, dtype=np.float64)
        y = np.ascontiguousarray(y, dtype=np.int64)
        N, V = z.shape
        loss = np.empty(N, np.float64)
        lse = np.empty(N, np.float64)
        am = np.empty(N, np.int64)
        self.lib.orc_ce_forward(self._p(z, _f64p), N, V, self._p(y, _i64p), float(eps),
                                int(ignore_index), self._p(loss, _f64p), self._p(lse, _f64p),
                                self._p(am, _i64p))
        return loss, lse, am

    def ce_backward(self, z, y, g, eps: float = 0.0, ignore_index: int = -100):
        """Gradient of sum_i g_i loss_i with respect to z, float64 (N, V)."""
        z = np.ascontiguousarray(z, dtype=np.float64)
        y = np.ascontiguousarray(y, dtype=np.int64)
        N, V = z.shape
        g = np.ascontiguousarray(np.broadcast_to(np.asarray(g, np.float64), (N,)))
        dz = np.empty((N, V), np.float64)
        self.lib.orc_ce_backward(self._p(z, _f64p), N, V, self._p(y, _i64p),
                                 self._p(g, _f64p), float(eps), int(ignore_index),
                                 self._p(dz, _f64p))
        return dz

    # -- probability (soft) targets ----------------------------------------
    def ce_soft_forward(self, z, t, eps: float = 0.0):
        """loss, lse (float64, N) of each row of z (N, V) against the target
        distribution t (N, V): loss = sum_j t'_j (lse - z_j)."""
        z = np.ascontiguousarray(z, dtype=np.float64)
        t = np.ascontiguousarray(t, dtype=np.float64)
        N, V = z.shape
        assert t.shape == (N, V)
        loss = np.empty(N, np.float64)
        lse = np.empty(N, np.float64)
        self.lib.orc_ce_soft_forward(self._p(z, _f64p), self._p(t, _f64p), N, V, float(eps),
                                     self._p(loss, _f64p), self._p(lse, _f64p))
        return loss, lse

    def ce_soft_backward(self, z, t, g, eps: float = 0.0):
        """Gradient of sum_i g_i loss_i with respect to z, float64 (N, V)."""
        z = np.ascontiguousarray(z, dtype=np.float64)
        t = np.ascontiguousarray(t, dtype=np.float64)
        N, V = z.shape
        g = np.ascontiguousarray(np.broadcast_to(np.asarray(g, np.float64), (N,)))
        dz = np.empty((N, V), np.float64)
        self.lib.orc_ce_soft_backward(self._p(z, _f64p), self._p(t, _f64p), N, V,
                                      self._p(g, _f64p), float(eps), self._p(dz, _f64p))
        return dz

    # -- KL divergence of the student from the teacher ----------------------
    def kl_forward(self, zq, zp):
        """loss = sum_j p_j (log p_j - log q_j), lse of the student and of the
        teacher (float64, N each); zq student, zp teacher logits (N, V)."""
        zq = np.ascontiguousarray(zq, dtype=np.float64)
        zp = np.ascontiguousarray(zp, dtype=np.float64)
        N, V = zq.shape
        assert zp.shape == (N, V)
        loss, lq, lp = (np.empty(N, np.float64) for _ in range(3))
        self.lib.orc_kl_forward(self._p(zq, _f64p), self._p(zp, _f64p), N, V, self._p(loss, _f64p),
                                self._p(lq, _f64p), self._p(lp, _f64p))
        return loss, lq, lp

    def kl_backward(self, zq, zp, g):
        """Gradient of sum_i g_i loss_i with respect to the student logits."""
        zq = np.ascontiguousarray(zq, dtype=np.float64)
        zp = np.ascontiguousarray(zp, dtype=np.float64)
        N, V = zq.shape
        g = np.ascontiguousarray(np.broadcast_to(np.asarray(g, np.float64), (N,)))
        d = np.empty((N, V), np.float64)
        self.lib.orc_kl_backward(self._p(zq, _f64p), self._p(zp, _f64p), N, V, self._p(g, _f64p),
                                 self._p(d, _f64p))
        return d

    # -- fused-linear cross-entropy ---------------------------------------
    def linear_ce_forward_rows(self, H, W, y, rows=None, eps: float = 0.0,
                               ignore_index: int = -100):
        """loss, lse of the listed rows of Z = H W^T (all rows if rows is None)."""
        H = np.ascontiguousarray(H, dtype=np.float32)
        W = np.ascontiguousarray(W, dtype=np.float32)
        y = np.ascontiguousarray(y, dtype=np.int64)
        N, D = H.shape
        V = W.shape[0]
        rows = np.arange(N, dtype=np.int64) if rows is None else \
            np.ascontiguousarray(rows, dtype=np.int64)
        loss = np.empty(len(rows), np.float64)
        lse = np.empty(len(rows), np.float64)
        self.lib.orc_linear_ce_forward_rows(self._p(H, _f32p), self._p(W, _f32p), V, D,
                                            self._p(rows, _i64p), len(rows),
                                            self._p(y, _i64p), float(eps), int(ignore_index),
                                            self._p(loss, _f64p), self._p(lse, _f64p))
        return loss, lse

    def linear_ce_dh_rows(self, H, W, y, g, rows, eps: float = 0.0,
                          ignore_index: int = -100):
        """Rows of dH = G W for the listed rows, float64 (len(rows), D)."""
        H = np.ascontiguousarray(H, dtype=np.float32)
        W = np.ascontiguousarray(W, dtype=np.float32)
        y = np.ascontiguousarray(y, dtype=np.int64)
        N, D = H.shape
        V = W.shape[0]
        g = np.ascontiguousarray(np.broadcast_to(np.asarray(g, np.float64), (N,)))
        rows = np.ascontiguousarray(rows, dtype=np.int64)
        dH = np.empty((len(rows), D), np.float64)
        self.lib.orc_linear_ce_dh_rows(self._p(H, _f32p), self._p(W, _f32p), V, D,
                                       self._p(rows, _i64p), len(rows), self._p(y, _i64p),
                                       self._p(g, _f64p), float(eps), int(ignore_index),
                                       self._p(dH, _f64p))
        return dH

    def linear_ce_dw_rows(self, H, W, y, g, cols, lse, eps: float = 0.0,
                          ignore_index: int = -100):
        """Rows of dW = G^T H for the listed vocabulary indices, float64
        (len(cols), D); lse (N,) is every row's log-sum-exp (float64)."""
        H = np.ascontiguousarray(H, dtype=np.float32)
        W = np.ascontiguousarray(W, dtype=np.float32)
        y = np.ascontiguousarray(y, dtype=np.int64)
        N, D = H.shape
        V = W.shape[0]
        g = np.ascontiguousarray(np.broadcast_to(np.asarray(g, np.float64), (N,)))
        lse = np.ascontiguousarray(lse, dtype=np.float64)
        assert lse.shape == (N,)
        cols = np.ascontiguousarray(cols, dtype=np.int64)
        dW = np.empty((len(cols), D), np.float64)
        self.lib.orc_linear_ce_dw_rows(self._p(H, _f32p), self._p(W, _f32p), N, V, D,
                                       self._p(cols, _i64p), len(cols), self._p(y, _i64p),
                                       self._p(g, _f64p), self._p(lse, _f64p), float(eps),
                                       int(ignore_index), self._p(dW, _f64p))
        return dW

    @staticmethod
    def linear_lse_all(H, W, chunk: int = 8192):
        """lse_i = m_i + log sum_j exp(Z_ij - m_i) of every row of Z = H W^T
        in float64, for problems too large for the row-by-row C loop (every
        row of the fused-linear workload). Z is formed one vocabulary chunk at
        a time by numpy's float64 matrix product (a library primitive); a
        first pass over the chunks takes the row maxima m_i, a second the sums
        of exp(Z_ij - m_i), chunk after chunk in vocabulary order."""
        Hd = np.asarray(H, dtype=np.float64)
        N = Hd.shape[0]
        V = W.shape[0]
        m = np.full(N, -np.inf)
        for v0 in range(0, V, chunk):
            Z = Hd @ np.asarray(W[v0:v0 + chunk], dtype=np.float64).T
            np.maximum(m, Z.max(axis=1), out=m)
        s = np.zeros(N)
        for v0 in range(0, V, chunk):
            Z = Hd @ np.asarray(W[v0:v0 + chunk], dtype=np.float64).T
            s += np.exp(Z - m[:, None]).sum(axis=1)
        return m + np.log(s)

    def linear_ce_backward(self, H, W, y, g, eps: float = 0.0, ignore_index: int = -100):
        """dH (N, D) and dW (V, D) in float64 for a small problem; also G (N, V)."""
        H = np.ascontiguousarray(H, dtype=np.float32)
        W = np.ascontiguousarray(W, dtype=np.float32)
        y = np.ascontiguousarray(y, dtype=np.int64)
        N, D = H.shape
        V = W.shape[0]
        g = np.ascontiguousarray(np.broadcast_to(np.asarray(g, np.float64), (N,)))
        G = np.empty((N, V), np.float64)
        dH = np.empty((N, D), np.float64)
        dW = np.empty((V, D), np.float64)
        self.lib.orc_linear_ce_backward(self._p(H, _f32p), self._p(W, _f32p), N, V, D,
                                        self._p(y, _i64p), self._p(g, _f64p), float(eps),
                                        int(ignore_index), self._p(G, _f64p),
                                        self._p(dH, _f64p), self._p(dW, _f64p))
        return dH, dW, G

    def num_threads(self) -> int:
        return int(self.lib.orc_num_threads())


_default: Oracle | None = None


def get() -> Oracle:
    """The oracle built from this directory's source (compiled on first use)."""
    global _default
    if _default is None:
        _default = Oracle()
    return _default
