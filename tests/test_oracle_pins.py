"""The oracle against its pins (CPU only)."""
import os
import shutil
import subprocess

import numpy as np
import pytest

import oracle
from tests import oracle_pins
from tests.oracle_pins import BATTERY, GOLDEN


@pytest.mark.parametrize("pin", BATTERY, ids=lambda f: f.__name__)
def test_pin(orc, pin):
    pin(orc)


def test_issue4686_statistical_pin(orc):
    """MLX issue #4686, Expected behavior: summed loss 12904.3 and gradient
    norm 34.352 on cross_entropy(x[:, :-1], y[:, 1:]) for x ~ N(0,1) of shape
    (10, 119, 32768). Our draw differs from the page's, so the pins are the
    statistical ones stated in the fixture."""
    vals = {}
    with open(os.path.join(GOLDEN, "vjp_grad_norm_issue4686.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                k, v = line.split()
                vals[k] = float(v)
    B, L, V = int(vals["B"]), int(vals["L"]), int(vals["V"])
    rng = np.random.default_rng(0)
    x = rng.standard_normal((B, L, V), dtype=np.float32)
    y = rng.integers(0, V, size=(B, L))
    z = x[:, :-1].reshape(-1, V)
    t = y[:, 1:].reshape(-1)
    loss, _, _ = orc.ce_forward(z, t)
    dz = orc.ce_backward(z, t, 1.0)
    assert abs(loss.sum() - vals["loss"]) <= vals["loss_tolerance"]
    assert abs(np.linalg.norm(dz) - vals["grad_norm"]) <= vals["grad_norm_tolerance"]


# Planted mistakes: (description, original text, replacement). Each must make
# at least one pin of the battery fail.
MUTANTS = [
    ("exp without the max shift", "s += exp(z[j] - m);", "s += exp(z[j]);"),
    ("lse drops m", "*lse = m + log(s);", "*lse = log(s);"),
    ("target term sign", "double l = log(s) - (1.0 - eps) * (z[y] - m);",
     "double l = log(s) + (1.0 - eps) * (z[y] - m);"),
    ("target term drops (1-eps)", "double l = log(s) - (1.0 - eps) * (z[y] - m);",
     "double l = log(s) - (z[y] - m);"),
    ("smoothing term sign", "l -= eps * (shifted_sum / (double)V);",
     "l += eps * (shifted_sum / (double)V);"),
    ("smoothing mean unshifted", "shifted_sum += (z[j] - m);", "shifted_sum += z[j];"),
    ("smoothing mean over V-1", "l -= eps * (shifted_sum / (double)V);",
     "l -= eps * (shifted_sum / (double)(V - 1));"),
    ("grad drops (1-eps)", "(1.0 - eps) * onehot", "onehot"),
    ("grad drops eps/V", " - eps / (double)V);", ");"),
    ("grad unnormalised", "double p = exp(z[j] - m) / s;", "double p = exp(z[j] - m);"),
    ("grad drops g", "dz[j] = g * (p", "dz[j] = (p"),
    ("grad one-hot off by one", "double onehot = (j == y) ? 1.0 : 0.0;",
     "double onehot = (j == y + 1) ? 1.0 : 0.0;"),
    ("argmax keeps last tie", "if (v > m) { m = v; am = j; }", "if (v >= m) { m = v; am = j; }"),
    ("ignore_index not honoured", "if (y == ignore_index) { *loss = 0.0; return; }", ""),
    ("ignored grad rows not zeroed",
     "        for (int64_t j = 0; j < V; ++j) dz[j] = 0.0;\n        return;",
     "        (void)0;"),
    ("linear row uses W^T indexing", "acc += (double)h[d] * (double)w[d];",
     "acc += (double)h[d] * (double)W[d * V + j];"),
    ("dW contracts with W", "acc += G[i * V + j] * (double)H[i * D + d];",
     "acc += G[i * V + j] * (double)W[j * D + d];"),
    ("dH contracts with H", "acc += G[i * V + j] * (double)W[j * D + d];\n            dH",
     "acc += G[i * V + j] * (double)H[i * D + d];\n            dH"),
    ("dh rows sign", "out[d] += gij * (double)w[d];", "out[d] -= gij * (double)w[d];"),
    ("dw rows contract with W", "out[d] += giv * (double)h[d];", "out[d] += giv * (double)w[d];"),
    ("dw rows drop eps/V", "- (1.0 - eps) * onehot - eps / (double)V);",
     "- (1.0 - eps) * onehot);"),
    ("dw rows one-hot on the row index", "const double onehot = (v == y[i]) ? 1.0 : 0.0;",
     "const double onehot = (i == y[i]) ? 1.0 : 0.0;"),
    ("dw rows keep ignored rows", "if (y[i] == ignore_index) {\n                giv = 0.0;",
     "if (0) {\n                giv = 0.0;"),
    ("soft lse drops m", "*lse = m + L;", "*lse = L;"),
    ("soft exp unshifted", "s += exp(z[j] - m);\n    const double L", "s += exp(z[j]);\n    const double L"),
    ("soft loss sign", "l += tj * (L - (z[j] - m));", "l += tj * (L + (z[j] - m));"),
    ("soft forward unsmoothed", "eps / (double)V;\n        if (tj", "0.0;\n        if (tj"),
    ("soft zero-mass terms kept", "if (tj != 0.0) l += ", "l += "),
    ("soft grad drops T", "d[j] = g[i] * (p * T - tj);", "d[j] = g[i] * (p - tj);"),
    ("soft grad drops g", "d[j] = g[i] * (p * T - tj);", "d[j] = (p * T - tj);"),
    ("soft grad unsmoothed target", "eps / (double)V;\n            d[j]", "0.0;\n            d[j]"),
    ("soft grad unnormalised", "const double p = exp(zr[j] - m) / s;", "const double p = exp(zr[j] - m);"),
    ("kl uses student lse for teacher", "const double lp = p[j] - lse_p[i];", "const double lp = p[j] - lse_q[i];"),
    ("kl sign of student term", "l += pj * (lp - (q[j] - lse_q[i]));", "l += pj * (lp + (q[j] - lse_q[i]));"),
    ("kl weights by student", "const double pj = exp(lp);", "const double pj = exp(q[j] - lse_q[i]);"),
    ("kl grad sign", "d[j] = g[i] * (exp(q[j] - lq) - exp(p[j] - lp));", "d[j] = g[i] * (exp(p[j] - lp) - exp(q[j] - lq));"),
    ("kl grad drops g", "d[j] = g[i] * (exp(q[j] - lq) - exp(p[j] - lp));", "d[j] = (exp(q[j] - lq) - exp(p[j] - lp));"),
    ("kl zero-mass terms kept", "if (pj != 0.0) l += ", "l += "),
]


@pytest.mark.parametrize("desc,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_planted_mistake_is_caught(tmp_path, desc, old, new):
    if shutil.which("gcc") is None:
        pytest.skip("gcc missing")
    src = open(os.path.join(os.path.dirname(oracle.__file__), "ce_oracle.c")).read()
    assert old in src, f"mutation anchor not found: {desc}"
    mutated = src.replace(old, new, 1)
    p = tmp_path / "mut.c"
    p.write_text(mutated)
    lib = str(tmp_path / "libmut.so")
    oracle.build(str(p), lib, force=True)
    mut = oracle.Oracle(lib)
    failures = 0
    for pin in oracle_pins.BATTERY:
        try:
            with np.errstate(all="ignore"):
                pin(mut)
        except AssertionError:
            failures += 1
        except (FloatingPointError, ValueError, IndexError):
            failures += 1
    assert failures > 0, f"no pin caught the planted mistake: {desc}"
